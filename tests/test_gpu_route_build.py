"""Token->expert grouping on the GPU, bit-exact against the oracle's stable counting sort."""

import numpy as np
import pytest
import torch

import moe_inputs as mi
import oracle
import sparse_moe_gemv_b200 as smg

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("T,k,E,zipf", [
    (1, 10, 512, None), (2, 10, 512, None), (3, 10, 512, None), (17, 2, 16, None), (33, 4, 64, 1.1),
    (2048, 10, 512, 1.1), (2048, 10, 512, None), (4096, 8, 1024, 1.1), (1000, 32, 1024, None),
    (5, 1, 1, None),
])
def test_route_build_bit_exact(gpu_lib, T, k, E, zipf):
    ids = mi.random_topk_ids(T, k, E, seed=T + 31 * k + E, zipf_s=zipf)
    c_ref, o_ref, p_ref = oracle.route_build(ids.numpy(), E)
    d_ids = ids.cuda()
    counts = torch.full((E,), -7, dtype=torch.int32, device="cuda")
    offsets = torch.full((E + 1,), -7, dtype=torch.int32, device="cuda")
    perm = torch.full((T * k,), -7, dtype=torch.int32, device="cuda")
    for _ in range(2):  # determinism: the second run must give the same bits
        smg.redmoe_route_build(d_ids, E, counts, offsets, perm)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(counts.cpu().numpy(), c_ref)
        np.testing.assert_array_equal(offsets.cpu().numpy(), o_ref)
        np.testing.assert_array_equal(perm.cpu().numpy(), p_ref)


def test_forward_debug_grouping_matches_oracle(gpu_lib):
    shape = mi.LayerShape(H=2048, E=512, k=10, I=512, Is=512)
    L = mi.make_layer(shape, 55, "cuda")
    x = mi.make_x(shape, 3, 55, "cuda")
    lay = smg.Layer.from_shape(L, shape)
    ws = smg.new_workspace(lay, 3)
    out = torch.empty(3, shape.H, device="cuda")
    ids = torch.empty(3, shape.k, dtype=torch.int32, device="cuda")
    w = torch.empty(3, shape.k, device="cuda")
    dbg = (torch.empty(shape.E, dtype=torch.int32, device="cuda"),
           torch.empty(shape.E + 1, dtype=torch.int32, device="cuda"),
           torch.empty(3 * shape.k, dtype=torch.int32, device="cuda"))
    smg.redmoe_forward(lay, x, out, ids, w, ws, dbg=dbg)
    torch.cuda.synchronize()
    # the oracle groups its own routing; this seed has no near-ties, so the ids must agree
    r = oracle.router(mi.layer_to_numpy(L, experts=[]), shape, mi.to_numpy(x))
    np.testing.assert_array_equal(ids.cpu().numpy(), r["ids"])
    c_ref, o_ref, p_ref = oracle.route_build(r["ids"], shape.E)
    np.testing.assert_array_equal(dbg[0].cpu().numpy(), c_ref)
    np.testing.assert_array_equal(dbg[1].cpu().numpy(), o_ref)
    np.testing.assert_array_equal(dbg[2].cpu().numpy(), p_ref)
