"""redmoe_forward_noalloc: the decode-size forward for callers that cannot allocate
device memory (strict stream capture, allocator-free hot loops, plug-ins without a
memory budget). Its scratch is a fixed array inside the library; the test checks,
through the C ABI, that two calls in a row give the result of redmoe_forward with a
caller workspace and of the fp64 oracle, and that the scratch's error word reads clean.
The file name makes pytest collect it last."""

import pytest
import torch

import moe_inputs as mi
import sparse_moe_gemv_b200 as smg
from parity import assert_layer_parity, tolerances

pytestmark = pytest.mark.gpu

QWEN = mi.LayerShape(H=2048, E=512, k=10, I=512, Is=512)


@pytest.mark.parametrize("T", [1, 3])
def test_noalloc_matches_workspace_forward_twice(gpu_lib, T):
    shape = QWEN
    L = mi.make_layer(shape, 9100 + T, "cuda")
    x = mi.make_x(shape, T, 9100 + T, "cuda")
    lay = smg.Layer.from_shape(L, shape)
    ws = smg.new_workspace(lay, T)
    ref = torch.empty(T, shape.H, device="cuda")
    ref_ids = torch.empty(T, shape.k, dtype=torch.int32, device="cuda")
    ref_w = torch.empty(T, shape.k, device="cuda")
    smg.redmoe_forward(lay, x, ref, ref_ids, ref_w, ws)
    torch.cuda.synchronize()
    out_tol, w_tol = tolerances(shape)
    rms = float(ref.double().pow(2).mean().sqrt())
    for call in range(2):
        out = torch.full((T, shape.H), float("nan"), device="cuda")
        ids = torch.full((T, shape.k), -1, dtype=torch.int32, device="cuda")
        w = torch.full((T, shape.k), float("nan"), device="cuda")
        smg.redmoe_forward_noalloc(lay, x, out, ids, w)
        smg.redmoe_check_timeout(None)
        assert torch.equal(ids, ref_ids), f"call {call}: ids differ"
        assert float((w - ref_w).abs().max()) <= w_tol, f"call {call}: weights differ"
        err = float((out.double() - ref.double()).abs().max())
        assert err <= out_tol * rms, f"call {call}: max err {err:.3e} > {out_tol} * RMS {rms:.3e}"
        assert_layer_parity(shape, L, x, out, ids, w, out_tol, w_tol, f"noalloc T={T} call {call}")
