"""The bounded in-kernel waits give up and report, instead of hanging.

redmoe_selftest_wait_limit runs a grid barrier of the kind every persistent kernel of
the library uses, with one block that never arrives and a 2 ms limit. The other blocks
give up, record the timeout and return; the host then sees REDMOE_ERR_TIMEOUT through
redmoe_check_timeout, and after redmoe_workspace_init the same workspace serves a
normal, oracle-matching forward. The same holds for the allocation-free scratch."""

import pytest
import torch

import moe_inputs as mi
import sparse_moe_gemv_b200 as smg
from parity import assert_layer_parity, tolerances

pytestmark = pytest.mark.gpu

TINY = mi.WORKLOADS["tiny_f32"]["shape"]
LIMIT_NS = 2_000_000


def _layer():
    L = mi.make_layer(TINY, 0, "cpu")
    L = {k: (v.cuda() if v is not None else None) for k, v in L.items()}
    x = mi.make_x(TINY, 2, 0, "cpu").cuda()
    return L, x, smg.Layer.from_shape(L, TINY)


def _expect_timeout(ws):
    with pytest.raises(smg.RedmoeError) as e:
        smg.redmoe_check_timeout(ws)
    assert e.value.status == 5  # REDMOE_ERR_TIMEOUT


def test_withheld_arrival_times_out_then_workspace_recovers(gpu_lib):
    L, x, lay = _layer()
    ws = smg.new_workspace(lay, 2)
    smg.redmoe_selftest_wait_limit(ws, -1, LIMIT_NS)  # everyone arrives: no timeout
    smg.redmoe_check_timeout(ws)
    smg.redmoe_selftest_wait_limit(ws, 3, LIMIT_NS)
    _expect_timeout(ws)
    _expect_timeout(ws)  # the error word stays set until the workspace is re-initialised
    smg.redmoe_workspace_init(ws)
    smg.redmoe_check_timeout(ws)
    out = torch.full((2, TINY.H), float("nan"), device="cuda")
    ids = torch.full((2, TINY.k), -1, dtype=torch.int32, device="cuda")
    w = torch.full((2, TINY.k), float("nan"), device="cuda")
    smg.redmoe_forward(lay, x, out, ids, w, ws)
    smg.redmoe_check_timeout(ws)
    ot, wt = tolerances(TINY)
    assert_layer_parity(TINY, L, x, out, ids, w, ot, wt, "after a timeout")


def test_noalloc_scratch_reports_a_timeout(gpu_lib):
    L, x, lay = _layer()
    smg.redmoe_workspace_init(None)
    smg.redmoe_selftest_wait_limit(None, 0, LIMIT_NS)
    _expect_timeout(None)
    out = torch.full((2, TINY.H), float("nan"), device="cuda")
    ids = torch.full((2, TINY.k), -1, dtype=torch.int32, device="cuda")
    w = torch.full((2, TINY.k), float("nan"), device="cuda")
    # a forward does not wipe the recorded timeout; only an explicit init does
    smg.redmoe_forward_noalloc(lay, x, out, ids, w)
    _expect_timeout(None)
    smg.redmoe_workspace_init(None)
    smg.redmoe_forward_noalloc(lay, x, out, ids, w)
    smg.redmoe_check_timeout(None)
    ot, wt = tolerances(TINY)
    assert_layer_parity(TINY, L, x, out, ids, w, ot, wt, "noalloc after a timeout")


def test_limits_out_of_range_are_rejected(gpu_lib):
    L, x, lay = _layer()
    ws = smg.new_workspace(lay, 2)
    for limit in (0, 2_000_000_000):
        with pytest.raises(smg.RedmoeError) as e:
            smg.redmoe_selftest_wait_limit(ws, 0, limit)
        assert e.value.status == 1
    with pytest.raises(smg.RedmoeError):
        smg.redmoe_selftest_wait_limit(ws, 100000, LIMIT_NS)
    smg.redmoe_check_timeout(ws)
