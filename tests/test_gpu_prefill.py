"""Batched (T > 4) path: tensor-core router GEMM, top-k, grouping, gather and the two
tensor-core grouped GEMMs, checked against the fp64 oracle through the C ABI."""

import numpy as np
import pytest
import torch

import moe_inputs as mi
import oracle
import sparse_moe_gemv_b200 as smg
from parity import assert_layer_parity, tolerances

pytestmark = pytest.mark.gpu

SMALL = mi.LayerShape(H=256, E=16, k=2, I=128, Is=128, sigma=0.05)
QWEN = mi.LayerShape(H=2048, E=512, k=10, I=512, Is=512)
QWEN_ZIPF = mi.LayerShape(H=2048, E=512, k=10, I=512, Is=512, zipf_s=1.1)


def _run(shape, L, x, dbg=False):
    T = x.shape[0]
    lay = smg.Layer.from_shape(L, shape)
    ws = smg.new_workspace(lay, T)
    out = torch.full((T, shape.H), float("nan"), device="cuda")
    ids = torch.full((T, shape.k), -1, dtype=torch.int32, device="cuda")
    w = torch.full((T, shape.k), float("nan"), device="cuda")
    d = None
    if dbg:
        d = (torch.full((shape.E,), -1, dtype=torch.int32, device="cuda"),
             torch.full((shape.E + 1,), -1, dtype=torch.int32, device="cuda"),
             torch.full((T * shape.k,), -1, dtype=torch.int32, device="cuda"))
    smg.redmoe_forward(lay, x, out, ids, w, ws, dbg=d)
    smg.redmoe_check_timeout(ws)
    return out, ids, w, d


@pytest.mark.parametrize("T", [5, 37, 130, 300])
def test_small_layer_batched(gpu_lib, T):
    shape = SMALL
    L = mi.make_layer(shape, 300 + T, "cuda")
    x = mi.make_x(shape, T, 300 + T, "cuda")
    out, ids, w, _ = _run(shape, L, x)
    ot, wt = tolerances(shape)
    assert_layer_parity(shape, L, x, out, ids, w, ot, wt, f"small batched T={T}")


@pytest.mark.parametrize("T", [5, 200])
def test_qwen_layer_batched(gpu_lib, T):
    shape = QWEN
    L = mi.make_layer(shape, 3100 + T, "cuda")
    x = mi.make_x(shape, T, 3100 + T, "cuda")
    out, ids, w, dbg = _run(shape, L, x, dbg=True)
    ot, wt = tolerances(shape)
    assert_layer_parity(shape, L, x, out, ids, w, ot, wt, f"qwen batched T={T}")
    _assert_grouping_of_gpu_ids(ids, dbg, shape.E)


def test_prefill_chunk_zipf_2048(gpu_lib):
    """The 2048-token prefill chunk with Zipf(1.1) router offsets: every token's ids,
    weights and output row (tolerance relative to the RMS of the whole [T, H] output),
    and the grouping, bit-exact against the oracle's stable grouping of the GPU's own ids
    (the reference for a near-tie token is then still unique)."""
    shape = QWEN_ZIPF
    T = 2048
    L = mi.make_layer(shape, 3000, "cuda")
    x = mi.make_x(shape, T, 3000, "cuda")
    out, ids, w, dbg = _run(shape, L, x, dbg=True)
    ot, wt = tolerances(shape)
    r = assert_layer_parity(shape, L, x, out, ids, w, ot, wt, "prefill zipf")
    _assert_grouping_of_gpu_ids(ids, dbg, shape.E)
    c_ref = oracle.route_build(r["ref"]["ids"], shape.E)[0]
    # the workload's shape: a few hot experts take hundreds of tokens, most take none
    assert int((c_ref >= 100).sum()) >= 5 and int((c_ref == 0).sum()) >= 200


def _assert_grouping_of_gpu_ids(ids, dbg, E):
    """counts, offsets and perm of the forward equal the oracle's grouping of the ids the
    GPU chose, bit for bit."""
    c_ref, o_ref, p_ref = oracle.route_build(ids.cpu().numpy(), E)
    np.testing.assert_array_equal(dbg[0].cpu().numpy(), c_ref)
    np.testing.assert_array_equal(dbg[1].cpu().numpy(), o_ref)
    np.testing.assert_array_equal(dbg[2].cpu().numpy(), p_ref)


MID = mi.LayerShape(H=512, E=40, k=3, I=256, Is=256, sigma=0.04)


@pytest.mark.parametrize("T", [6, 250])
def test_mid_layer_batched(gpu_lib, T):
    """Several n-tiles in both grouped GEMMs (I / 128 = 2, H / 256 = 2) and a router width
    that is not a multiple of the 64-expert GEMM tile."""
    shape = MID
    L = mi.make_layer(shape, 500 + T, "cuda")
    x = mi.make_x(shape, T, 500 + T, "cuda")
    out, ids, w, _ = _run(shape, L, x)
    ot, wt = tolerances(shape)
    assert_layer_parity(shape, L, x, out, ids, w, ot, wt, f"mid batched T={T}")


def test_top1_routing_batched(gpu_lib):
    shape = mi.LayerShape(H=256, E=16, k=1, I=128, Is=128, sigma=0.05)
    T = 64
    L = mi.make_layer(shape, 640, "cuda")
    x = mi.make_x(shape, T, 640, "cuda")
    out, ids, w, _ = _run(shape, L, x)
    assert torch.all(w == 1.0)  # renormalising a single selection gives weight 1
    ot, wt = tolerances(shape)
    assert_layer_parity(shape, L, x, out, ids, w, ot, wt, "top-1 batched")


def test_chunk_4096_all_experts(gpu_lib):
    """A 4096-token chunk with unbiased routing: every expert receives tokens and every CTA
    of the grouped GEMMs runs many tiles. Ids, weights and output rows of every token,
    and the grouping bit-exact against the oracle's grouping of the GPU's ids."""
    shape = QWEN
    T = 4096
    L = mi.make_layer(shape, 4096, "cuda")
    x = mi.make_x(shape, T, 4096, "cuda")
    out, ids, w, dbg = _run(shape, L, x, dbg=True)
    ot, wt = tolerances(shape)
    assert_layer_parity(shape, L, x, out, ids, w, ot, wt, "chunk 4096")
    _assert_grouping_of_gpu_ids(ids, dbg, shape.E)
    assert int((dbg[0] > 0).sum()) == shape.E


def test_batched_repeat_is_stable(gpu_lib):
    """Two calls on the same input: ids, weights and grouping are identical; the outputs
    differ at most by the order of the fp32 reductions of the combine."""
    shape = QWEN
    T = 300
    L = mi.make_layer(shape, 77, "cuda")
    x = mi.make_x(shape, T, 77, "cuda")
    o1, i1, w1, d1 = _run(shape, L, x, dbg=True)
    o2, i2, w2, d2 = _run(shape, L, x, dbg=True)
    assert torch.equal(i1, i2) and torch.equal(w1, w2)
    for a, b in zip(d1, d2):
        assert torch.equal(a, b)
    scale = float(o1.abs().max())
    assert float((o1 - o2).abs().max()) <= 1e-5 * scale
