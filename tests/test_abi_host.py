"""Host-side checks of the C ABI (no GPU needed): the library loads, exports every entry
point that include/redmoe.h declares, and rejects bad arguments before touching CUDA."""

import ctypes as C
import os
import re

import pytest

import sparse_moe_gemv_b200 as smg

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "redmoe.h")

OK, INVALID, UNSUPPORTED, WORKSPACE = 0, 1, 2, 3


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(smg.LIB_PATH):
        from sparse_moe_gemv_b200 import build
        build.build()
    return smg.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(redmoe_[a-z_]+)\s*\(", text)))


def test_header_and_binding_agree():
    assert sorted(smg.SYMBOLS) == declared_functions()


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
        assert C.cast(getattr(lib, name), C.c_void_p).value


def test_version_and_status_strings(lib):
    assert smg.redmoe_abi_version() == smg.ABI_VERSION
    for s in range(6):
        assert smg.redmoe_status_string(s) and smg.redmoe_status_string(s) != "unknown status"
    assert smg.redmoe_status_string(99) == "unknown status"


FAKE = 0x7f0000000000  # a 256-byte aligned address that is never dereferenced by these calls


def _layer(**over):
    s = smg._Layer()
    s.hidden, s.n_experts, s.top_k, s.inter, s.shared_inter = 2048, 512, 10, 512, 512
    s.x_dtype = s.router_dtype = s.expert_dtype = 1
    for i, (name, _) in enumerate(smg._Layer._fields_[8:]):
        setattr(s, name, FAKE + 0x100000 * (i + 1))
    s.router_bias = None
    s.s_gate = s.s_up = s.s_down = s.sh_s_gate = s.sh_s_up = s.sh_s_down = None
    for k, v in over.items():
        setattr(s, k, v)
    return s


def _fwd(lib, L, T=1, x=FAKE, out=FAKE, ids=FAKE, w=FAKE, ws=FAKE, ws_bytes=1 << 30):
    return lib.redmoe_forward(C.byref(L), x, T, out, ids, w, ws, ws_bytes, None, 0)


def test_workspace_bytes(lib):
    L = _layer()
    n1 = lib.redmoe_workspace_bytes(C.byref(L), 1)
    n4 = lib.redmoe_workspace_bytes(C.byref(L), 4)
    assert n1 > 256 and n1 % 256 == 0 and n4 >= n1
    assert lib.redmoe_workspace_bytes(C.byref(L), -1) == 0
    assert lib.redmoe_workspace_bytes(None, 1) == 0
    assert lib.redmoe_workspace_bytes(C.byref(_layer(top_k=600)), 1) == 0


@pytest.mark.parametrize("field,value,expect", [
    ("hidden", 0, INVALID), ("hidden", 2050, INVALID), ("n_experts", 0, INVALID), ("n_experts", 2048, INVALID),
    ("top_k", 0, INVALID), ("top_k", 33, INVALID), ("inter", 500, INVALID), ("shared_inter", -1, INVALID),
    ("x_dtype", 7, INVALID), ("router_dtype", 2, INVALID), ("x_dtype", 0, UNSUPPORTED),
    ("router_w", None, INVALID), ("w_down", FAKE + 8, INVALID), ("sh_up", None, INVALID),
    ("router_bias", FAKE + 2, INVALID),
])
def test_forward_rejects_bad_layer(lib, field, value, expect):
    assert _fwd(lib, _layer(**{field: value})) == expect


def test_forward_rejects_bad_call_arguments(lib):
    L = _layer()
    assert _fwd(lib, L, T=-1) == INVALID
    assert _fwd(lib, L, x=None) == INVALID
    assert _fwd(lib, L, x=FAKE + 4) == INVALID
    assert _fwd(lib, L, out=FAKE + 8) == INVALID
    assert _fwd(lib, L, ids=None) == INVALID
    assert _fwd(lib, L, w=FAKE + 1) == INVALID
    assert _fwd(lib, L, ws=None) == WORKSPACE
    assert _fwd(lib, L, ws=FAKE + 128) == WORKSPACE
    assert _fwd(lib, L, ws_bytes=1024) == WORKSPACE
    # T == 0 is an empty call: accepted, nothing enqueued (no CUDA call is made)
    assert _fwd(lib, L, T=0) == OK


def test_forward_host_checks_before_touching_cuda(lib):
    """The host-buffer forward: its workspace holds the forward's plus the staging, and bad
    arguments are rejected before any copy is enqueued."""
    L = _layer()
    for T in (1, 4, 5, 2048):
        n, nh = lib.redmoe_workspace_bytes(C.byref(L), T), lib.redmoe_workspace_bytes_host(C.byref(L), T)
        # staging: x (bf16) + out (fp32) + ids + w, each 256-aligned
        assert nh % 256 == 0 and nh >= n + T * 2048 * 2 + T * 2048 * 4 + 2 * T * 10 * 4
    assert lib.redmoe_workspace_bytes_host(C.byref(L), -1) == 0
    assert lib.redmoe_workspace_bytes_host(None, 1) == 0
    need = lib.redmoe_workspace_bytes_host(C.byref(L), 1)

    def fh(T=1, x=FAKE, out=FAKE, ids=FAKE, w=FAKE, ws=FAKE, ws_bytes=need):
        return lib.redmoe_forward_host(C.byref(L), x, T, out, ids, w, ws, ws_bytes, 0)

    assert fh(T=-1) == INVALID
    assert fh(T=0) == OK
    assert fh(x=None) == INVALID
    assert fh(x=FAKE + 4) == INVALID
    assert fh(out=FAKE + 8) == INVALID
    assert fh(ids=FAKE + 2) == INVALID
    assert fh(w=None) == INVALID
    assert fh(ws=None) == WORKSPACE
    assert fh(ws=FAKE + 128) == WORKSPACE
    assert fh(ws_bytes=need - 256) == WORKSPACE
    assert lib.redmoe_forward_host(C.byref(_layer(hidden=0)), FAKE, 1, FAKE, FAKE, FAKE, FAKE, need, 0) == INVALID


def test_forward_stack_host_checks_before_touching_cuda(lib):
    L = _layer()
    need = lib.redmoe_workspace_bytes_host(C.byref(L), 1)
    arr = (smg._Layer * 2)(L, L)
    P2 = C.c_void_p * 2

    def fsh(n=2, T=1, x=FAKE, out=FAKE, ids=FAKE, w=FAKE, ws=FAKE, ws_bytes=need, layers=arr):
        return lib.redmoe_forward_stack_host(C.cast(layers, C.c_void_p), n, C.cast(P2(x, x), C.c_void_p), T,
                                             C.cast(P2(out, out), C.c_void_p), C.cast(P2(ids, ids), C.c_void_p),
                                             C.cast(P2(w, w), C.c_void_p), ws, ws_bytes, 0)

    assert fsh(n=0) == OK and fsh(T=0) == OK
    assert fsh(n=-1) == INVALID and fsh(T=-1) == INVALID
    assert fsh(x=FAKE + 4) == INVALID and fsh(out=FAKE + 8) == INVALID and fsh(ids=FAKE + 2) == INVALID
    assert fsh(ws=None) == WORKSPACE and fsh(ws_bytes=need - 256) == WORKSPACE
    assert fsh(layers=(smg._Layer * 2)(L, _layer(top_k=8))) == INVALID


def test_int4_layer_needs_scales(lib):
    L = _layer(expert_dtype=2)
    assert _fwd(lib, L) == INVALID
    sc = {n: FAKE + 0x10000000 + 0x100000 * i for i, n in
          enumerate(("s_gate", "s_up", "s_down", "sh_s_gate", "sh_s_up", "sh_s_down"))}
    L2 = _layer(expert_dtype=2, **{**sc, "s_down": FAKE + 1})
    assert _fwd(lib, L2) == INVALID


def test_route_build_rejects_bad_arguments(lib):
    f = lib.redmoe_route_build
    assert f(FAKE, 4, 0, 16, FAKE, FAKE, FAKE, None, 0, 0) == INVALID
    assert f(FAKE, 4, 17, 16, FAKE, FAKE, FAKE, None, 0, 0) == INVALID
    assert f(FAKE, -1, 2, 16, FAKE, FAKE, FAKE, None, 0, 0) == INVALID
    assert f(None, 4, 2, 16, FAKE, FAKE, FAKE, None, 0, 0) == INVALID
    assert f(FAKE, 4, 2, 16, FAKE + 2, FAKE, FAKE, None, 0, 0) == INVALID
    assert f(FAKE, 4, 2, 2000, FAKE, FAKE, FAKE, None, 0, 0) == INVALID


def test_router_and_stack_reject_bad_arguments(lib):
    L = _layer()
    assert lib.redmoe_router(C.byref(L), None, 2, FAKE, FAKE, FAKE, None, FAKE, 1 << 30, 0) == INVALID
    assert lib.redmoe_router(C.byref(L), FAKE, 2, FAKE, FAKE, None, None, FAKE, 1 << 30, 0) == INVALID
    assert lib.redmoe_router(C.byref(L), FAKE, 2, FAKE, FAKE, FAKE, None, FAKE, 64, 0) == WORKSPACE
    arr = (smg._Layer * 2)(L, _layer(inter=1024))
    P = C.c_void_p * 2
    ptrs = P(FAKE, FAKE)
    assert lib.redmoe_forward_stack(C.cast(arr, C.c_void_p), 2, C.cast(ptrs, C.c_void_p), 1,
                                    C.cast(ptrs, C.c_void_p), C.cast(ptrs, C.c_void_p),
                                    C.cast(ptrs, C.c_void_p), FAKE, 1 << 30, 0) == INVALID
    assert lib.redmoe_forward_stack(None, 2, None, 1, None, None, None, FAKE, 1 << 30, 0) == INVALID
    # a misaligned workspace is refused before any CUDA call
    assert lib.redmoe_workspace_init(C.c_void_p(FAKE + 16), 256, 0) == WORKSPACE
    assert lib.redmoe_workspace_init(FAKE, 255, 0) == WORKSPACE
    assert lib.redmoe_check_timeout(C.c_void_p(FAKE + 16), 0) == WORKSPACE


def test_null_workspace_means_the_noalloc_scratch(lib):
    """NULL selects the library's own scratch array; with no CUDA device the lookup of
    its address fails, which is a CUDA error, not a workspace error."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("needs a host without a CUDA device")
    CUDA = 4
    assert lib.redmoe_workspace_init(None, 0, 0) == CUDA
    assert lib.redmoe_check_timeout(None, 0) == CUDA


def test_selftest_rejects_bad_limits_before_touching_cuda(lib):
    f = lib.redmoe_selftest_wait_limit
    assert f(FAKE, 256, 0, 0, 0) == INVALID
    assert f(FAKE, 256, 0, 2_000_000_000, 0) == INVALID
    assert f(C.c_void_p(FAKE + 16), 256, 0, 1000, 0) == WORKSPACE
    assert f(FAKE, 128, 0, 1000, 0) == WORKSPACE


def test_noalloc_rejects_before_touching_cuda(lib):
    L = _layer()
    f = lib.redmoe_forward_noalloc
    assert f(C.byref(L), FAKE, -1, FAKE, FAKE, FAKE, 0) == INVALID
    assert f(C.byref(L), None, 1, FAKE, FAKE, FAKE, 0) == INVALID
    assert f(C.byref(L), FAKE, 5, FAKE, FAKE, FAKE, 0) == UNSUPPORTED
    assert f(C.byref(L), FAKE, 0, FAKE, FAKE, FAKE, 0) == OK
    # a layer whose decode scratch exceeds the fixed 1 MiB array is refused
    big = _layer(top_k=32, inter=2048, n_experts=64)
    assert f(C.byref(big), FAKE, 4, FAKE, FAKE, FAKE, 0) == WORKSPACE


def test_batched_path_shape_rules(lib):
    """T > 4 runs the batched path, which takes bf16 layers with shared_inter == inter,
    hidden % 256 == 0 and inter % 128 == 0; the others are refused on the host before any
    CUDA call."""
    sc = {n: FAKE + 0x10000000 + 0x100000 * i for i, n in
          enumerate(("s_gate", "s_up", "s_down", "sh_s_gate", "sh_s_up", "sh_s_down"))}
    assert _fwd(lib, _layer(expert_dtype=2, **sc), T=8) == UNSUPPORTED          # int4 experts
    assert _fwd(lib, _layer(shared_inter=256), T=8) == UNSUPPORTED              # shared_inter != inter
    assert _fwd(lib, _layer(inter=96, shared_inter=96), T=8) == UNSUPPORTED     # inter % 128 != 0
    assert _fwd(lib, _layer(hidden=2080), T=8) == UNSUPPORTED                   # hidden % 256 != 0
    assert _fwd(lib, _layer(x_dtype=0, router_dtype=0, expert_dtype=0), T=8) == UNSUPPORTED  # fp32 layer


def test_batched_workspace_holds_the_grouped_buffers(lib):
    L = _layer()
    T, k, H, I, E = 2048, 10, 2048, 512, 512
    need = lib.redmoe_workspace_bytes(C.byref(L), T)
    # logits, the gathered x rows and the SwiGLU rows at least
    assert need >= 4 * T * E + 2 * T * k * H + 2 * (T * k + T) * I
    assert need % 256 == 0


def test_missing_library_fails_loudly(monkeypatch):
    """No fallback: without the built library the binding raises, it never computes."""
    monkeypatch.setattr(smg, "_lib", None)
    monkeypatch.setattr(smg, "LIB_PATH", os.path.join(os.path.dirname(smg.LIB_PATH), "absent", "libredmoe.so"))
    with pytest.raises(RuntimeError, match="is missing"):
        smg.load()
    with pytest.raises(RuntimeError, match="is missing"):
        smg.redmoe_status_string(0)
