"""redmoe_forward_host: x and the results in host memory. At decode sizes with pinned
outputs the kernel stores the results straight into host memory; larger T and pageable
outputs take the device staging and copies. Each case is checked against the fp64 oracle
and, where the path is deterministic, bit for bit against redmoe_forward on device buffers."""

import pytest
import torch

import moe_inputs as mi
import sparse_moe_gemv_b200 as smg
from parity import assert_layer_parity, tolerances

pytestmark = pytest.mark.gpu

QWEN = mi.LayerShape(H=2048, E=512, k=10, I=512, Is=512)
QWEN_INT4 = mi.LayerShape(H=2048, E=512, k=10, I=512, Is=512, expert_dtype="int4g32")
QWEN_INT2 = mi.LayerShape(H=2048, E=512, k=10, I=512, Is=512, expert_dtype="int2g32")
TINY = mi.WORKLOADS["tiny_f32"]["shape"]  # fp32 layer: the three- and four-row kernel at T = 1


def _host_call(shape, L, x_dev, pinned=True):
    T = x_dev.shape[0]
    lay = smg.Layer.from_shape(L, shape)
    ws = smg.new_workspace_host(lay, T)
    hx = x_dev.cpu()
    hout = torch.full((T, shape.H), float("nan"))
    hids = torch.full((T, shape.k), -1, dtype=torch.int32)
    hw = torch.full((T, shape.k), float("nan"))
    if pinned:
        hx, hout, hids, hw = hx.pin_memory(), hout.pin_memory(), hids.pin_memory(), hw.pin_memory()
    s = torch.cuda.Stream()
    smg.redmoe_forward_host(lay, hx, hout, hids, hw, ws, stream=s)
    s.synchronize()
    smg.redmoe_check_timeout(ws)
    return hout, hids, hw, lay


def _device_call(shape, lay, x_dev):
    T = x_dev.shape[0]
    ws = smg.new_workspace(lay, T)
    out = torch.empty(T, shape.H, device="cuda")
    ids = torch.empty(T, shape.k, dtype=torch.int32, device="cuda")
    w = torch.empty(T, shape.k, device="cuda")
    smg.redmoe_forward(lay, x_dev, out, ids, w, ws)
    torch.cuda.synchronize()
    return out.cpu(), ids.cpu(), w.cpu()


@pytest.mark.parametrize("shape,T,pinned", [
    (QWEN, 1, True), (QWEN, 1, False), (QWEN, 2, True), (QWEN, 3, True), (QWEN, 4, True), (QWEN_INT4, 1, True),
    (QWEN_INT2, 1, True), (TINY, 1, True), (TINY, 3, True), (QWEN_INT4, 2, True), (QWEN, 2, False),
])
def test_decode_sizes_match_device_buffers_and_oracle(gpu_lib, shape, T, pinned):
    L = mi.make_layer(shape, 7000 + T, "cuda")
    x = mi.make_x(shape, T, 7000 + T, "cuda")
    hout, hids, hw, lay = _host_call(shape, L, x, pinned)
    dout, dids, dw = _device_call(shape, lay, x)
    # the decode kernels are deterministic: the host results equal the device ones exactly
    assert torch.equal(hids, dids) and torch.equal(hw, dw) and torch.equal(hout, dout)
    ot, wt = tolerances(shape)
    assert_layer_parity(shape, L, x, hout.cuda(), hids.cuda(), hw.cuda(), ot, wt, f"host T={T} pinned={pinned}")


def test_batched_size_through_staging(gpu_lib):
    shape = QWEN
    T = 200
    L = mi.make_layer(shape, 7200, "cuda")
    x = mi.make_x(shape, T, 7200, "cuda")
    hout, hids, hw, lay = _host_call(shape, L, x, True)
    dout, dids, dw = _device_call(shape, lay, x)
    assert torch.equal(hids, dids) and torch.equal(hw, dw)
    # the batched combine's summation order is not fixed: equal up to fp32 rounding
    assert torch.allclose(hout, dout, rtol=0, atol=1e-5 * float(dout.abs().max()))
    ot, wt = tolerances(shape)
    assert_layer_parity(shape, L, x, hout.cuda(), hids.cuda(), hw.cuda(), ot, wt, "host T=200")


def test_back_to_back_calls_keep_their_results(gpu_lib):
    """Several calls queued on one stream into different pinned host buffers: each buffer
    holds its own call's results once the stream is synchronised."""
    shape = QWEN
    lay_t = [mi.make_layer(shape, 7300 + i, "cuda") for i in range(3)]
    lays = [smg.Layer.from_shape(t, shape) for t in lay_t]
    xs = [mi.make_x(shape, 1, 7300 + i, "cuda") for i in range(3)]
    ws = smg.new_workspace_host(lays[0], 1)
    outs = [torch.empty(1, shape.H).pin_memory() for _ in range(3)]
    idss = [torch.empty(1, shape.k, dtype=torch.int32).pin_memory() for _ in range(3)]
    wss = [torch.empty(1, shape.k).pin_memory() for _ in range(3)]
    hxs = [x.cpu().pin_memory() for x in xs]
    s = torch.cuda.Stream()
    for i in range(3):
        smg.redmoe_forward_host(lays[i], hxs[i], outs[i], idss[i], wss[i], ws, stream=s)
    s.synchronize()
    smg.redmoe_check_timeout(ws)
    for i in range(3):
        dout, dids, dw = _device_call(shape, lays[i], xs[i])
        assert torch.equal(outs[i], dout) and torch.equal(idss[i], dids) and torch.equal(wss[i], dw)


def test_rewritten_host_x_is_read_again(gpu_lib):
    """One pinned x buffer rewritten by the host between calls (the decode loop's usual
    pattern): each call reads the current contents, not a cached copy of the last ones."""
    shape = QWEN
    L = mi.make_layer(shape, 7400, "cuda")
    lay = smg.Layer.from_shape(L, shape)
    ws = smg.new_workspace_host(lay, 1)
    hx = torch.empty(1, shape.H, dtype=torch.bfloat16).pin_memory()
    hout = torch.empty(1, shape.H).pin_memory()
    hids = torch.empty(1, shape.k, dtype=torch.int32).pin_memory()
    hw = torch.empty(1, shape.k).pin_memory()
    s = torch.cuda.Stream()
    for seed in (7401, 7402, 7403):
        x = mi.make_x(shape, 1, seed, "cuda")
        hx.copy_(x.cpu())
        smg.redmoe_forward_host(lay, hx, hout, hids, hw, ws, stream=s)
        s.synchronize()
        dout, dids, dw = _device_call(shape, lay, x)
        assert torch.equal(hout, dout) and torch.equal(hids, dids) and torch.equal(hw, dw), seed
    smg.redmoe_check_timeout(ws)


@pytest.mark.parametrize("shape,T,pinned", [
    (QWEN, 1, True), (QWEN_INT4, 1, True), (QWEN_INT2, 1, True), (QWEN, 2, True), (QWEN_INT4, 2, True),
    (QWEN, 1, False), (QWEN, 3, True),
])
def test_stack_host_matches_device_stack(gpu_lib, shape, T, pinned):
    """A stack of distinct layers with every x and result in host memory: one launch that
    reads each layer's x over the link (T = 1, pinned), or layer-by-layer host calls;
    either way bit for bit the device-buffer stack's results."""
    n = 3
    tens = [mi.make_layer(shape, 7500 + l, "cuda") for l in range(n)]
    lays = [smg.Layer.from_shape(t, shape) for t in tens]
    xs = [mi.make_x(shape, T, 7600 + l, "cuda") for l in range(n)]
    dws = smg.new_workspace(lays[0], T)
    douts = [torch.empty(T, shape.H, device="cuda") for _ in range(n)]
    dids = [torch.empty(T, shape.k, dtype=torch.int32, device="cuda") for _ in range(n)]
    dw = [torch.empty(T, shape.k, device="cuda") for _ in range(n)]
    smg.redmoe_forward_stack(lays, xs, douts, dids, dw, dws)
    torch.cuda.synchronize()

    def host(t):
        return t.pin_memory() if pinned else t
    hxs = [host(x.cpu()) for x in xs]
    houts = [host(torch.full((T, shape.H), float("nan"))) for _ in range(n)]
    hids = [host(torch.full((T, shape.k), -1, dtype=torch.int32)) for _ in range(n)]
    hw = [host(torch.full((T, shape.k), float("nan"))) for _ in range(n)]
    ws = smg.new_workspace_host(lays[0], T)
    s = torch.cuda.Stream()
    smg.redmoe_forward_stack_host(lays, hxs, houts, hids, hw, ws, stream=s)
    s.synchronize()
    smg.redmoe_check_timeout(ws)
    for l in range(n):
        assert torch.equal(houts[l], douts[l].cpu()) and torch.equal(hids[l], dids[l].cpu()), l
        assert torch.equal(hw[l], dw[l].cpu()), l
    ot, wt = tolerances(shape)
    assert_layer_parity(shape, tens[1], xs[1], houts[1].cuda(), hids[1].cuda(), hw[1].cuda(), ot, wt, "stack host layer 1")
