"""Pins of the fp64 oracle against facts that do not come from the oracle itself.

Each test is chosen so that a plausible slip in the oracle (a dropped term, a swapped
operand, a wrong index, a wrong sign, a wrong tie rule) fails at least one of them:

* a hand-derived worked example (tests/golden/worked_example.json), whose values
  follow from sigmoid(+-ln 3) in closed form;
* hand-decoded int4 group-32 rows (tests/golden/int4_groups.json);
* a k-subset enumeration for the top-k selection;
* a dense brute-force layer computed in another loop order with a full sort;
* special cases with closed forms (one dominant expert, zero routed experts);
* invariants (weights sum to one, relabelling the experts, stable grouping equals a
  library stable sort, int4 equals its dequantised fp32 copy).
"""

import itertools
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import moe_inputs as mi
import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


# ----------------------------------------------------------------- helpers
def _val(v):
    if isinstance(v, str):
        neg = v.startswith("-")
        base = v.lstrip("-")
        if base.startswith("ln"):
            r = math.log(float(base[2:]))
        else:
            r = float(Fraction(base))
        return -r if neg else r
    return float(v)


def _arr(a, dtype=np.float32):
    return np.vectorize(_val, otypes=[np.float64])(np.array(a, dtype=object)).astype(dtype)


def _frac(a):
    return np.vectorize(lambda s: float(Fraction(s)), otypes=[np.float64])(np.array(a, dtype=object))


def _tiny(shape, seed, T=None):
    L = mi.make_layer(shape, seed, "cpu")
    x = mi.make_x(shape, T if T is not None else 3, seed, "cpu")
    return mi.layer_to_numpy(L), mi.to_numpy(x)


def _golden_layer(g):
    s = g["shape"]
    shape = mi.LayerShape(H=s["H"], E=s["E"], k=s["k"], I=s["I"], Is=s["Is"], x_dtype="f32",
                          router_dtype="f32", expert_dtype="f32")
    lay = {name: _arr(v) for name, v in g["layer"].items()}
    return shape, lay


SHAPES = {
    "f32_E16_k2": mi.LayerShape(H=64, E=16, k=2, I=32, Is=32, x_dtype="f32", router_dtype="f32",
                                expert_dtype="f32", sigma=0.3, rms_norm_x=False),
    "bf16_E8_k3": mi.LayerShape(H=64, E=8, k=3, I=32, Is=64, sigma=0.2),
    "int4_E8_k2": mi.LayerShape(H=64, E=8, k=2, I=32, Is=32, expert_dtype="int4g32", sigma=0.2),
    "bf16_E12_k4_bias": mi.LayerShape(H=32, E=12, k=4, I=32, Is=32, sigma=0.3, zipf_s=1.1),
}


# ------------------------------------------------------------- worked example
@pytest.mark.parametrize("case_idx", [0, 1])
def test_hand_worked_example(case_idx):
    g = json.load(open(os.path.join(GOLDEN, "worked_example.json")))
    shape, lay = _golden_layer(g)
    case = g["cases"][case_idx]
    if case["router_bias"] is not None:
        lay["router_bias"] = _arr(case["router_bias"])
    x = _arr(g["x"])
    r = oracle.forward(lay, shape, x)
    np.testing.assert_array_equal(r["ids"], np.array(case["ids"]))
    # fp32 storage of ln n perturbs the closed forms at the 1e-7 relative level
    np.testing.assert_allclose(r["w"], _frac(case["w"]), rtol=1e-6, atol=0)
    np.testing.assert_allclose(r["s"], _frac(case["s"]), rtol=1e-6, atol=0)
    np.testing.assert_allclose(r["out"], _frac(case["out_over_ln3"]) * math.log(3.0), rtol=2e-6, atol=1e-7)
    counts, offsets, perm = oracle.route_build(r["ids"], shape.E)
    np.testing.assert_array_equal(counts, case["counts"])
    np.testing.assert_array_equal(offsets, case["offsets"])
    np.testing.assert_array_equal(perm, case["perm"])


# ----------------------------------------------------------------- int4 format
def test_int4_hand_decoded_rows():
    g = json.load(open(os.path.join(GOLDEN, "int4_groups.json")))
    r0 = g["rows"][0]
    got = oracle.dequant_int4(np.array([r0["bytes"]], np.uint8), np.array([r0["scales_bf16_bits"]], np.uint16))
    np.testing.assert_array_equal(got[0], np.array(r0["expected"]))
    r1 = g["rows"][1]
    got = oracle.dequant_int4(np.array([r1["bytes"]], np.uint8), np.array([r1["scales_bf16_bits"]], np.uint16))
    pat = r1["expected_pattern"]
    expect = np.array([pat[0][i % 2] for i in range(32)] + [pat[1][i % 2] for i in range(32)])
    np.testing.assert_array_equal(got[0], expect)


def test_int4_quantiser_roundtrip_and_extremes():
    g = torch.Generator().manual_seed(5)
    w = torch.randn(6, 96, generator=g) * 0.02
    w[2, 32:64] = 0.0                       # an all-zero group: scale 0, codes 0
    packed, scales = mi.quantize_int4g32(w)
    deq = oracle.dequant_int4(mi.to_numpy(packed), mi.to_numpy(scales))
    s = np.repeat(scales.float().numpy().astype(np.float64), 32, axis=1)
    err = np.abs(deq - w.double().numpy())
    assert np.all(err <= 0.5 * s * (1 + 1e-6))
    assert np.all(deq[2, 32:64] == 0.0)
    # the element of largest magnitude of a group sits at code +-7 (scale = bf16(amax / 7))
    grp = w.reshape(6, 3, 32)
    arg = grp.abs().argmax(dim=-1)
    for n in range(6):
        for gi in range(3):
            if n == 2 and gi == 1:
                continue
            c = gi * 32 + int(arg[n, gi])
            q = deq[n, c] / float(scales[n, gi].float())
            assert abs(abs(q) - 7.0) < 1e-12


def test_int4_layer_equals_its_dequantised_fp32_copy():
    shape = SHAPES["int4_E8_k2"]
    lay, x = _tiny(shape, 11)
    dq = dict(lay)
    for w_name, s_name in (("w_gate", "s_gate"), ("w_up", "s_up"), ("w_down", "s_down")):
        W, S = lay[w_name], lay[s_name]
        E, N = W.shape[0], W.shape[1]
        dq[w_name] = np.stack([oracle.dequant_int4(W[e], S[e]) for e in range(E)]).astype(np.float32)
        dq[s_name] = None
    for w_name, s_name in (("sh_gate", "sh_s_gate"), ("sh_up", "sh_s_up"), ("sh_down", "sh_s_down")):
        dq[w_name] = oracle.dequant_int4(lay[w_name], lay[s_name]).astype(np.float32)
        dq[s_name] = None
    # scale * code is exact in fp32, so the fp32 copy holds the same numbers
    shape32 = mi.LayerShape(**{**shape.__dict__, "expert_dtype": "f32"})
    a = oracle.forward(lay, shape, x)
    b = oracle.forward(dq, shape32, x)
    np.testing.assert_array_equal(a["ids"], b["ids"])
    np.testing.assert_array_equal(a["out"], b["out"])


# ----------------------------------------------------------------- int2 format
def test_int2_hand_decoded_rows():
    g = json.load(open(os.path.join(GOLDEN, "int2_groups.json")))
    r0 = g["rows"][0]
    got = oracle.dequant_int2(np.array([r0["bytes"]], np.uint8), np.array([r0["scales_bf16_bits"]], np.uint16))
    np.testing.assert_array_equal(got[0], np.array(r0["expected"]))
    r1 = g["rows"][1]
    got = oracle.dequant_int2(np.array([r1["bytes"]], np.uint8), np.array([r1["scales_bf16_bits"]], np.uint16))
    pat = r1["expected_pattern"]
    expect = np.array([pat[0][i % 4] for i in range(32)] + [pat[1][i % 4] for i in range(32)])
    np.testing.assert_array_equal(got[0], expect)


def test_int2_quantiser_roundtrip_and_extremes():
    g = torch.Generator().manual_seed(6)
    w = torch.randn(5, 64, generator=g) * 0.02
    w[1, 0:32] = 0.0                        # an all-zero group: scale 0, codes 2 (value 0)
    packed, scales = mi.quantize_int2g32(w)
    assert packed.shape == (5, 16) and scales.shape == (5, 2)
    assert np.all(mi.to_numpy(packed)[1, 0:8] == 0xAA)
    deq = oracle.dequant_int2(mi.to_numpy(packed), mi.to_numpy(scales))
    s = np.repeat(scales.float().numpy().astype(np.float64), 32, axis=1)
    # every value is -s, 0 or s, and it is the one nearest to w (scale = bf16(amax))
    q = np.where(s == 0, 0.0, deq / np.where(s == 0, 1.0, s))
    assert set(np.unique(q).tolist()) <= {-1.0, 0.0, 1.0}
    wd = w.double().numpy()
    assert np.all(np.abs(deq - wd) <= 0.5 * s * (1 + 1e-6) + np.maximum(0, np.abs(wd) - s))
    grp = w.reshape(5, 2, 32)
    arg = grp.abs().argmax(dim=-1)
    for n in range(5):
        for gi in range(2):
            if n == 1 and gi == 0:
                continue
            c = gi * 32 + int(arg[n, gi])
            assert abs(q[n, c]) == 1.0


def test_int2_layer_equals_its_dequantised_fp32_copy():
    shape = mi.LayerShape(H=64, E=8, k=2, I=32, Is=32, expert_dtype="int2g32", sigma=0.2)
    lay, x = _tiny(shape, 12)
    dq = dict(lay)
    for w_name, s_name in (("w_gate", "s_gate"), ("w_up", "s_up"), ("w_down", "s_down")):
        W, S = lay[w_name], lay[s_name]
        dq[w_name] = np.stack([oracle.dequant_int2(W[e], S[e]) for e in range(W.shape[0])]).astype(np.float32)
        dq[s_name] = None
    for w_name, s_name in (("sh_gate", "sh_s_gate"), ("sh_up", "sh_s_up"), ("sh_down", "sh_s_down")):
        dq[w_name] = oracle.dequant_int2(lay[w_name], lay[s_name]).astype(np.float32)
        dq[s_name] = None
    shape32 = mi.LayerShape(**{**shape.__dict__, "expert_dtype": "f32"})
    a = oracle.forward(lay, shape, x)
    b = oracle.forward(dq, shape32, x)
    np.testing.assert_array_equal(a["ids"], b["ids"])
    np.testing.assert_array_equal(a["out"], b["out"])


# ------------------------------------------------------------ top-k selection
@pytest.mark.parametrize("name", list(SHAPES))
def test_topk_is_best_k_subset(name):
    shape = SHAPES[name]
    lay, x = _tiny(shape, 3, T=6)
    r = oracle.router(lay, shape, x)
    for t in range(x.shape[0]):
        l = r["logits"][t]
        best = max(itertools.combinations(range(shape.E), shape.k), key=lambda c: sum(l[list(c)]))
        assert set(best) == set(r["ids"][t].tolist())
        # ordered by logit, largest first
        assert np.all(np.diff(l[r["ids"][t]]) <= 0)


def test_router_logits_match_a_matrix_product():
    shape = SHAPES["bf16_E12_k4_bias"]
    lay, x = _tiny(shape, 4, T=5)
    r = oracle.router(lay, shape, x)
    X = (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    W = (lay["router_w"].astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    G = (lay["shared_gate_w"].astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    np.testing.assert_allclose(r["logits"], X @ W.T + lay["router_bias"].astype(np.float64), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(r["s"], 1.0 / (1.0 + np.exp(-(X @ G))), rtol=1e-12)


@pytest.mark.parametrize("name", list(SHAPES))
def test_weights_positive_sum_to_one_and_equal_softmax_of_selected(name):
    shape = SHAPES[name]
    lay, x = _tiny(shape, 7, T=8)
    r = oracle.router(lay, shape, x)
    assert np.all(r["w"] > 0)
    np.testing.assert_allclose(r["w"].sum(axis=1), 1.0, rtol=0, atol=1e-15)
    np.testing.assert_allclose(r["probs"].sum(axis=1), 1.0, rtol=0, atol=1e-14)
    for t in range(x.shape[0]):
        sel = r["logits"][t][r["ids"][t]]
        alt = np.exp(sel - sel.max())
        np.testing.assert_allclose(r["w"][t], alt / alt.sum(), rtol=0, atol=1e-15)
        assert len(set(r["ids"][t].tolist())) == shape.k


def test_exact_tie_goes_to_lower_id():
    shape = mi.LayerShape(H=32, E=8, k=3, I=32, Is=32, x_dtype="f32", router_dtype="f32", expert_dtype="f32")
    lay, x = _tiny(shape, 9, T=2)
    lay["router_w"] = np.zeros_like(lay["router_w"])
    lay["router_w"][5] = 1.0                      # expert 5 leads; 0..4, 6, 7 tie at 0
    x = np.abs(x) + 0.1
    r = oracle.router(lay, shape, x)
    np.testing.assert_array_equal(r["ids"], [[5, 0, 1], [5, 0, 1]])


# --------------------------------------------------------------- brute force
@pytest.mark.parametrize("name", list(SHAPES))
def test_sparse_equals_dense_brute_force(name):
    shape = SHAPES[name]
    lay, x = _tiny(shape, 21, T=5)
    a = oracle.forward(lay, shape, x)
    b = oracle.brute(lay, shape, x)
    np.testing.assert_array_equal(a["ids"], b["ids"])
    np.testing.assert_allclose(a["w"], b["w"], rtol=1e-14, atol=0)
    scale = np.sqrt(np.mean(a["out"] ** 2))
    assert np.max(np.abs(a["out"] - b["out"])) <= 1e-13 * scale


# ------------------------------------------------------- closed-form special cases
def _as_f64(a, dtype):
    if dtype == "bf16":
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


def test_expert_ffn_equals_dense_matrix_formula():
    shape = SHAPES["bf16_E8_k3"]
    lay, x = _tiny(shape, 31, T=1)
    xd = _as_f64(x[0], "bf16")
    for e in (0, 5, -1):
        y = oracle.expert_ffn(lay, shape, e, xd)
        if e >= 0:
            Wg, Wu, Wd = (_as_f64(lay[n][e], "bf16") for n in ("w_gate", "w_up", "w_down"))
        else:
            Wg, Wu, Wd = (_as_f64(lay[n], "bf16") for n in ("sh_gate", "sh_up", "sh_down"))
        a = Wg @ xd
        ref = Wd @ (a / (1 + np.exp(-a)) * (Wu @ xd))
        np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-14)


def test_one_dominant_expert_reduces_to_that_expert():
    """A router row aligned with x and scaled so that every other softmax weight underflows:
    the layer output is exactly that single expert's SwiGLU (the shared expert is zeroed)."""
    shape = SHAPES["f32_E16_k2"]
    lay, x = _tiny(shape, 41, T=3)
    e_star = 9
    for name in ("sh_gate", "sh_up", "sh_down"):
        lay[name] = np.zeros_like(lay[name])
    for t in range(x.shape[0]):
        L = dict(lay)
        L["router_w"] = lay["router_w"].copy()
        L["router_w"][e_star] = (2000.0 * x[t] / np.dot(x[t], x[t])).astype(np.float32)
        r = oracle.forward(L, shape, x[t:t + 1])
        assert r["ids"][0, 0] == e_star
        assert r["w"][0, 0] == 1.0 and r["w"][0, 1] == 0.0
        y = oracle.expert_ffn(L, shape, e_star, x[t].astype(np.float64))
        np.testing.assert_array_equal(r["out"][0], y)


def test_zero_routed_experts_leave_shared_path_in_closed_form():
    """Zero routed experts; shared weights built so that a = ln 3, u = c_i and the down
    projection copies lane i: out[h] = sigmoid(ln 3) * (3/4) ln 3 * c_{h mod Is}."""
    shape = mi.LayerShape(H=256, E=16, k=2, I=64, Is=64, x_dtype="f32", router_dtype="f32", expert_dtype="f32")
    lay, _ = _tiny(shape, 51, T=2)
    ref_route = None
    x = np.ones((2, shape.H), np.float32)
    x[1, :] = 1.0
    ln3 = np.float32(math.log(3.0))
    for name in ("w_gate", "w_up", "w_down"):
        lay[name] = np.zeros_like(lay[name])
    c = np.linspace(-2.0, 2.0, shape.Is).astype(np.float32)
    lay["sh_gate"] = np.full((shape.Is, shape.H), ln3 / shape.H, np.float32)
    lay["sh_up"] = np.repeat((c / shape.H)[:, None], shape.H, axis=1).astype(np.float32)
    lay["sh_down"] = np.zeros((shape.H, shape.Is), np.float32)
    lay["sh_down"][np.arange(shape.H), np.arange(shape.H) % shape.Is] = 1.0
    lay["shared_gate_w"] = np.full((shape.H,), ln3 / shape.H, np.float32)
    r = oracle.forward(lay, shape, x)
    a = float(ln3)                                  # the H equal terms sum exactly
    u = (c.astype(np.float64) / shape.H) * shape.H   # likewise exact for H = 256
    s = 1.0 / (1.0 + math.exp(-a))
    expect = s * (a / (1.0 + math.exp(-a))) * u[np.arange(shape.H) % shape.Is]
    np.testing.assert_allclose(r["out"][0], expect, rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(r["s"], 0.75, rtol=1e-7)
    ref_route = oracle.router(lay, shape, x)
    np.testing.assert_array_equal(ref_route["ids"], r["ids"])


# ------------------------------------------------------------- invariances
@pytest.mark.parametrize("name", ["f32_E16_k2", "int4_E8_k2", "bf16_E12_k4_bias"])
def test_relabelling_experts_changes_nothing(name):
    shape = SHAPES[name]
    lay, x = _tiny(shape, 61, T=6)
    sigma = np.random.default_rng(0).permutation(shape.E)
    perm_lay = dict(lay)
    perm_lay["router_w"] = lay["router_w"][sigma]
    if lay.get("router_bias") is not None:
        perm_lay["router_bias"] = lay["router_bias"][sigma]
    for n in ("w_gate", "w_up", "w_down", "s_gate", "s_up", "s_down"):
        if lay.get(n) is not None:
            perm_lay[n] = lay[n][sigma]
    a = oracle.forward(lay, shape, x)
    b = oracle.forward(perm_lay, shape, x)
    # expert sigma[j] of the relabelled layer is expert j' = sigma[j] of the original
    np.testing.assert_array_equal(sigma[b["ids"]], a["ids"])
    np.testing.assert_allclose(b["w"], a["w"], rtol=1e-14, atol=0)
    scale = np.sqrt(np.mean(a["out"] ** 2))
    assert np.max(np.abs(a["out"] - b["out"])) <= 1e-14 * scale


# ----------------------------------------------------------- token->expert grouping
@pytest.mark.parametrize("T,k,E,zipf", [(1, 10, 512, None), (3, 10, 512, None), (37, 4, 16, 1.1),
                                        (2048, 10, 512, 1.1), (500, 8, 64, None), (0, 10, 512, None)])
def test_grouping_is_a_stable_sort_by_expert(T, k, E, zipf):
    ids = mi.random_topk_ids(T, k, E, seed=T * 7 + k, zipf_s=zipf).numpy()
    counts, offsets, perm = oracle.route_build(ids, E)
    flat = ids.reshape(-1)
    # a library stable sort of the row indices by expert id is the definition
    ref = np.array(sorted(range(T * k), key=lambda i: flat[i]), dtype=np.int32)
    np.testing.assert_array_equal(perm, ref)
    np.testing.assert_array_equal(counts, np.bincount(flat, minlength=E))
    assert offsets[0] == 0 and offsets[-1] == T * k
    np.testing.assert_array_equal(np.diff(offsets), counts)
    assert sorted(perm.tolist()) == list(range(T * k))
    for e in range(E):
        rows = perm[offsets[e]:offsets[e + 1]]
        assert np.all(flat[rows] == e)
        assert np.all(np.diff(rows // k) > 0)


def test_partial_expert_supply_is_enough_and_missing_is_reported():
    shape = SHAPES["bf16_E8_k3"]
    lay, x = _tiny(shape, 71, T=2)
    full = oracle.forward(lay, shape, x)
    used = sorted(set(full["ids"].reshape(-1).tolist()))
    part = dict(lay)
    for n in ("w_gate", "w_up", "w_down"):
        part[n] = {e: lay[n][e] for e in used}
    again = oracle.forward(part, shape, x)
    np.testing.assert_array_equal(again["out"], full["out"])
    missing = dict(part)
    missing["w_down"] = {e: lay["w_down"][e] for e in used[1:]}
    with pytest.raises(oracle.OracleError):
        oracle.forward(missing, shape, x)


# ------------------------------------------------------- renormalised subsets
# oracle.renorm gives the weights of an arbitrary k-subset of one token's experts; the
# parity checker uses it for tokens on a near-tie, where the valid id set is not unique.
LOGITS_WORKED = np.log(np.array([1.0, 2.0, 3.0, 4.0]))  # p = (1, 2, 3, 4) / 10


@pytest.mark.parametrize("ids,expected", [
    ((3, 2), (Fraction(4, 7), Fraction(3, 7))),   # the worked example's token 0
    ((0, 1), (Fraction(1, 3), Fraction(2, 3))),   # a subset the router would not pick
    ((1, 3), (Fraction(1, 3), Fraction(2, 3))),
    ((2,), (Fraction(1),)),                      # a single selection renormalises to 1
    ((0, 1, 2, 3), (Fraction(1, 10), Fraction(2, 10), Fraction(3, 10), Fraction(4, 10))),
])
def test_renorm_hand_derived_subsets(ids, expected):
    w = oracle.renorm(LOGITS_WORKED, np.array(ids, np.int32))
    np.testing.assert_allclose(w, [float(f) for f in expected], rtol=0, atol=1e-15)


def test_renorm_ignores_a_common_logit_shift():
    # softmax is shift-invariant: p_e / sum_sel p = exp(l_e) / sum_sel exp(l); a shift of
    # every logit by 700 must not change the weights (nor overflow); l + 700 is stored
    # with an absolute rounding of up to 2^-44, so the weights agree to about 1e-13
    ids = np.array([3, 0, 2], np.int32)
    np.testing.assert_allclose(oracle.renorm(LOGITS_WORKED + 700.0, ids),
                               [4 / 8, 1 / 8, 3 / 8], rtol=0, atol=1e-12)


@pytest.mark.parametrize("name", list(SHAPES))
def test_renorm_equals_router_weights_for_router_ids(name):
    shape = SHAPES[name]
    lay, x = _tiny(shape, 11, T=6)
    r = oracle.router(lay, shape, x)
    for t in range(x.shape[0]):
        np.testing.assert_allclose(oracle.renorm(r["logits"][t], r["ids"][t]), r["w"][t], rtol=0, atol=1e-15)
        # a reversed order gives the same weights, reversed
        np.testing.assert_allclose(oracle.renorm(r["logits"][t], r["ids"][t][::-1].copy()), r["w"][t][::-1],
                                   rtol=0, atol=1e-15)
