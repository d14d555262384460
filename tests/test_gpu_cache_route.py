"""Opt-in cache-aware routing (redmoe_forward_cached) against the oracle's cache-aware
mode, through the C ABI, on every execution path: the one-row decode kernel (T = 1), the
few-row decode kernel (T = 2, 3) and the batched tensor-core path (T > 4)."""

import numpy as np
import pytest
import torch

import moe_inputs as mi
import sparse_moe_gemv_b200 as smg
from parity import assert_layer_parity, tolerances

pytestmark = pytest.mark.gpu

QWEN = mi.LayerShape(H=2048, E=512, k=10, I=512, Is=512)
QWEN_INT4 = mi.LayerShape(H=2048, E=512, k=10, I=512, Is=512, expert_dtype="int4g32")
SMALL = mi.LayerShape(H=256, E=16, k=2, I=128, Is=128, sigma=0.05)


def _cached_mask(E, frac, seed):
    rng = np.random.default_rng(seed)
    m = np.zeros(E, np.uint8)
    m[rng.choice(E, max(1, int(E * frac)), replace=False)] = 1
    return m


@pytest.mark.parametrize("shape,T,lam", [(QWEN, 1, 0.3), (QWEN, 1, 1.5), (QWEN_INT4, 1, 0.3), (QWEN, 2, 0.3),
                                         (QWEN, 3, 1.5), (SMALL, 37, 0.3), (QWEN, 200, 0.3), (QWEN, 1, 0.0)])
def test_cache_aware_routing_matches_oracle(gpu_lib, shape, T, lam):
    seed = 7000 + T + int(10 * lam)
    L = mi.make_layer(shape, seed, "cuda")
    x = mi.make_x(shape, T, seed, "cuda")
    cached = _cached_mask(shape.E, 0.25, seed)
    lay = smg.Layer.from_shape(L, shape)
    ws = smg.new_workspace(lay, T)
    out = torch.full((T, shape.H), float("nan"), device="cuda")
    ids = torch.full((T, shape.k), -1, dtype=torch.int32, device="cuda")
    w = torch.full((T, shape.k), float("nan"), device="cuda")
    smg.redmoe_forward_cached(lay, x, out, ids, w, torch.from_numpy(cached).cuda(), lam, ws)
    smg.redmoe_check_timeout(ws)
    ot, wt = tolerances(shape)
    assert_layer_parity(shape, L, x, out, ids, w, ot, wt, f"cached T={T} lam={lam}", cache=(cached, lam))
    if lam > 1.0 and int(cached.sum()) >= shape.k:
        assert bool(torch.from_numpy(cached).cuda()[ids.long()].bool().all())  # only cached experts run


def test_lambda_zero_equals_plain_forward(gpu_lib):
    shape, T = QWEN, 1
    L = mi.make_layer(shape, 7100, "cuda")
    x = mi.make_x(shape, T, 7100, "cuda")
    lay = smg.Layer.from_shape(L, shape)
    ws = smg.new_workspace(lay, T)
    outs = []
    for cached in (None, torch.ones(shape.E, dtype=torch.uint8, device="cuda")):
        out = torch.empty(T, shape.H, device="cuda")
        ids = torch.empty(T, shape.k, dtype=torch.int32, device="cuda")
        w = torch.empty(T, shape.k, device="cuda")
        if cached is None:
            smg.redmoe_forward(lay, x, out, ids, w, ws)
        else:
            smg.redmoe_forward_cached(lay, x, out, ids, w, cached, 0.0, ws)
        outs.append((out, ids, w))
    torch.cuda.synchronize()
    assert torch.equal(outs[0][1], outs[1][1])
    assert torch.equal(outs[0][0], outs[1][0])
