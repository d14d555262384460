"""Decode-size parity (1..4 token rows) of the CUDA path against the fp64 oracle, through
the C ABI. Layers are seeded synthetic layers with the workloads' shapes and dtypes."""

import numpy as np
import pytest
import torch

import moe_inputs as mi
import oracle
import sparse_moe_gemv_b200 as smg
from parity import assert_layer_parity, host_routing_layer, reference, tolerances

pytestmark = pytest.mark.gpu

QWEN = mi.LayerShape(H=2048, E=512, k=10, I=512, Is=512)
QWEN_INT4 = mi.LayerShape(H=2048, E=512, k=10, I=512, Is=512, expert_dtype="int4g32")
QWEN_INT2 = mi.LayerShape(H=2048, E=512, k=10, I=512, Is=512, expert_dtype="int2g32")
TINY = mi.WORKLOADS["tiny_f32"]["shape"]


def _dev_layer(shape, seed):
    return mi.make_layer(shape, seed, "cuda")


def _run(gpu_lib, shape, L, x):
    T = x.shape[0]
    lay = smg.Layer.from_shape(L, shape)
    ws = smg.new_workspace(lay, T)
    out = torch.full((T, shape.H), float("nan"), device="cuda")
    ids = torch.full((T, shape.k), -1, dtype=torch.int32, device="cuda")
    w = torch.full((T, shape.k), float("nan"), device="cuda")
    smg.redmoe_forward(lay, x, out, ids, w, ws)
    smg.redmoe_check_timeout(ws)
    return out, ids, w, ws, lay


@pytest.mark.parametrize("T", [1, 2, 3, 4])
def test_tiny_fp32(gpu_lib, T):
    shape = TINY
    L = mi.make_layer(shape, 0, "cpu")
    L = {k: (v.cuda() if v is not None else None) for k, v in L.items()}
    x = mi.make_x(shape, T, 0, "cpu").cuda()
    out, ids, w, _, _ = _run(gpu_lib, shape, L, x)
    ot, wt = tolerances(shape)
    assert_layer_parity(shape, L, x, out, ids, w, ot, wt, f"tiny T={T}")


@pytest.mark.parametrize("T", [1, 2, 3, 4])
def test_qwen_bf16(gpu_lib, T):
    shape = QWEN
    L = _dev_layer(shape, 1000 + T)
    x = mi.make_x(shape, T, 1000 + T, "cuda")
    out, ids, w, _, _ = _run(gpu_lib, shape, L, x)
    ot, wt = tolerances(shape)
    assert_layer_parity(shape, L, x, out, ids, w, ot, wt, f"bf16 T={T}")


@pytest.mark.parametrize("T", [1, 2, 3, 4])
def test_qwen_int4(gpu_lib, T):
    shape = QWEN_INT4
    L = _dev_layer(shape, 4000 + T)
    x = mi.make_x(shape, T, 4000 + T, "cuda")
    out, ids, w, _, _ = _run(gpu_lib, shape, L, x)
    ot, wt = tolerances(shape)
    assert_layer_parity(shape, L, x, out, ids, w, ot, wt, f"int4 T={T}")


def test_qwen_int2(gpu_lib):
    """The library's int2 group-32 experts, dequantised inside the one-row kernel."""
    shape = QWEN_INT2
    for seed in (6001, 6002):
        L = _dev_layer(shape, seed)
        x = mi.make_x(shape, 1, seed, "cuda")
        out, ids, w, _, _ = _run(gpu_lib, shape, L, x)
        ot, wt = tolerances(shape)
        assert_layer_parity(shape, L, x, out, ids, w, ot, wt, f"int2 seed={seed}")


@pytest.mark.parametrize("case", ["ties_in_topk", "ties_at_boundary", "all_equal"])
def test_router_ties_one_row(gpu_lib, case):
    """Exactly equal logits (duplicated router rows) go to the lower expert id first, in
    the selection and in its order: inside the top-k, across the k-th place, and with all
    E logits equal (every key reaches the selection threshold, so the one-row kernel takes
    its round-by-round fallback)."""
    shape = QWEN
    L = _dev_layer(shape, 1100)
    x = mi.make_x(shape, 1, 1100, "cuda")
    out, ids, w, _, _ = _run(gpu_lib, shape, L, x)
    top = ids[0].tolist()
    R = L["router_w"]
    if case == "ties_in_topk":
        # the 3rd-ranked expert's row copied to two lower and two higher ids
        src = top[2]
        for e in (0, 1, 510, 511):
            if e not in top:
                R[e] = R[src]
    elif case == "ties_at_boundary":
        # the 10th-ranked expert's row copied to four other experts: a 5-way tie that only
        # the lowest ids survive
        src = top[9]
        for e in (3, 77, 300, 509):
            if e not in top:
                R[e] = R[src]
    else:
        R[:] = R[0]
    out, ids, w, _, _ = _run(gpu_lib, shape, L, x)
    ot, wt = tolerances(shape)
    if case != "all_equal":
        ref = reference(shape, L, x)
        assert ids[0].tolist() == [int(e) for e in ref["ids"][0]], (ids[0].tolist(), ref["ids"][0])
        assert_layer_parity(shape, L, x, out, ids, w, ot, wt, f"ties {case}")
        return
    # every expert ties: the oracle's own routing (no near-tie enumeration, which would
    # list every k-subset of the 512) and its outputs for that routing
    xn = mi.to_numpy(x)
    r = oracle.router(host_routing_layer(L), shape, xn)
    assert r["ids"][0].tolist() == list(range(shape.k))
    assert ids[0].tolist() == list(range(shape.k))
    assert np.allclose(w[0].cpu().numpy(), 1.0 / shape.k, atol=1e-6)
    lay_e = mi.layer_to_numpy(L, experts=list(range(shape.k)))
    ref_out = oracle.experts(lay_e, shape, xn, r["ids"], r["w"], r["s"])
    rms = float(np.sqrt(np.mean(ref_out ** 2)))
    err = float(np.max(np.abs(out.cpu().numpy().astype(np.float64) - ref_out)))
    assert err <= ot * rms, (err, rms)


def test_int2_beyond_one_row_is_unsupported(gpu_lib):
    shape = QWEN_INT2
    L = _dev_layer(shape, 6003)
    x = mi.make_x(shape, 2, 6003, "cuda")
    with pytest.raises(smg.RedmoeError) as e:
        _run(gpu_lib, shape, L, x)
    assert e.value.status == 2  # REDMOE_ERR_UNSUPPORTED


@pytest.mark.parametrize("T,shape", [(1, QWEN), (1, QWEN_INT4), (1, QWEN_INT2), (2, QWEN)])
def test_repeat_calls_are_identical(gpu_lib, T, shape):
    """The decode path has no atomics: two calls give bit-identical outputs."""
    L = _dev_layer(shape, 1234)
    x = mi.make_x(shape, T, 1234, "cuda")
    out1, ids1, w1, ws, lay = _run(gpu_lib, shape, L, x)
    out2 = torch.empty_like(out1)
    ids2 = torch.empty_like(ids1)
    w2 = torch.empty_like(w1)
    smg.redmoe_forward(lay, x, out2, ids2, w2, ws)
    torch.cuda.synchronize()
    assert torch.equal(out1, out2) and torch.equal(ids1, ids2) and torch.equal(w1, w2)


@pytest.mark.parametrize("T,nl,shape", [(2, 4, QWEN), (3, 3, QWEN), (1, 6, QWEN_INT4), (1, 3, QWEN), (1, 4, QWEN_INT2), (4, 2, TINY)])
def test_stack_matches_per_layer_oracle(gpu_lib, T, nl, shape):
    layers = [_dev_layer(shape, 2000 + 17 * l) for l in range(nl)]
    xs = [mi.make_x(shape, T, 2000 + 17 * l, "cuda") for l in range(nl)]
    lays = [smg.Layer.from_shape(L, shape) for L in layers]
    ws = smg.new_workspace(lays[0], T)
    outs = [torch.full((T, shape.H), float("nan"), device="cuda") for _ in range(nl)]
    ids = [torch.full((T, shape.k), -1, dtype=torch.int32, device="cuda") for _ in range(nl)]
    wts = [torch.full((T, shape.k), float("nan"), device="cuda") for _ in range(nl)]
    smg.redmoe_forward_stack(lays, xs, outs, ids, wts, ws)
    smg.redmoe_check_timeout(ws)
    ot, wt = tolerances(shape)
    for l in range(nl):
        assert_layer_parity(shape, layers[l], xs[l], outs[l], ids[l], wts[l], ot, wt, f"stack layer {l}")


def test_empty_call_touches_nothing(gpu_lib):
    shape = QWEN
    L = _dev_layer(shape, 7)
    lay = smg.Layer.from_shape(L, shape)
    ws = smg.new_workspace(lay, 1)
    x = torch.empty(0, shape.H, dtype=torch.bfloat16, device="cuda")
    out = torch.empty(0, shape.H, device="cuda")
    ids = torch.empty(0, shape.k, dtype=torch.int32, device="cuda")
    w = torch.empty(0, shape.k, device="cuda")
    smg.redmoe_forward(lay, x, out, ids, w, ws)
    smg.redmoe_check_timeout(ws)


def test_router_entry_point(gpu_lib):
    shape = QWEN
    L = _dev_layer(shape, 99)
    for T in (1, 5, 37):
        x = mi.make_x(shape, T, 99 + T, "cuda")
        lay = smg.Layer.from_shape(L, shape)
        ws = smg.new_workspace(lay, T)
        ids = torch.empty(T, shape.k, dtype=torch.int32, device="cuda")
        w = torch.empty(T, shape.k, device="cuda")
        s = torch.empty(T, device="cuda")
        logits = torch.empty(T, shape.E, device="cuda")
        smg.redmoe_router(lay, x, ids, w, s, ws, logits=logits)
        torch.cuda.synchronize()
        import oracle
        r = oracle.router(mi.layer_to_numpy(L, experts=[]), shape, mi.to_numpy(x))
        assert np.max(np.abs(logits.cpu().numpy() - r["logits"])) < 1e-4
        assert np.max(np.abs(s.cpu().numpy() - r["s"])) < 1e-5
        from parity import candidate_sets, check_order
        for t in range(T):
            sets, ex = candidate_sets(r["logits"][t], shape.k)
            assert tuple(sorted(ids[t].tolist())) in sets
            assert check_order(r["logits"][t], ids[t].cpu().numpy())


@pytest.mark.parametrize("name,T", [("bf16", 1), ("bf16", 2), ("bf16", 3), ("bf16", 4), ("int4", 1), ("int4", 3),
                                    ("int2", 1), ("tiny", 4)])
def test_decode_after_shared_memory_poison(gpu_lib, name, T):
    """Every SM's shared memory is filled with NaN right before the call, so a read of a
    ring stage, of x or of h ahead of its data shows up in the results of this call."""
    shape = {"bf16": QWEN, "int4": QWEN_INT4, "int2": QWEN_INT2, "tiny": TINY}[name]
    if name == "tiny":
        L = {k: (v.cuda() if v is not None else None) for k, v in mi.make_layer(shape, 5, "cpu").items()}
        x = mi.make_x(shape, T, 5, "cpu").cuda()
    else:
        L = _dev_layer(shape, 5000 + T)
        x = mi.make_x(shape, T, 5000 + T, "cuda")
    lay = smg.Layer.from_shape(L, shape)
    ws = smg.new_workspace(lay, T)
    ot, wt = tolerances(shape)
    for call in range(2):
        out = torch.full((T, shape.H), float("nan"), device="cuda")
        ids = torch.full((T, shape.k), -1, dtype=torch.int32, device="cuda")
        w = torch.full((T, shape.k), float("nan"), device="cuda")
        smg.redmoe_fill_shared_memory()
        smg.redmoe_forward(lay, x, out, ids, w, ws)
        smg.redmoe_check_timeout(ws)
        assert bool(torch.isfinite(out).all()), f"{name} T={T} call {call}: non-finite outputs"
        assert_layer_parity(shape, L, x, out, ids, w, ot, wt, f"poisoned {name} T={T} call {call}")
