"""Python binding of libredmoe.so (C ABI: include/redmoe.h).

Argument marshalling only: every step of the layer runs in the library's CUDA kernels.
torch provides device memory and streams. The binding never computes a result itself
and has no fallback: if the library is missing it raises.

Names match the C entry points (redmoe_forward, redmoe_router, redmoe_route_build,
redmoe_forward_stack, redmoe_forward_noalloc, redmoe_workspace_bytes,
redmoe_workspace_init, redmoe_check_timeout, redmoe_selftest_wait_limit,
redmoe_fill_shared_memory, redmoe_forward_cached, redmoe_expert_cache_slot_bytes,
redmoe_expert_cache_init, redmoe_forward_host_experts, redmoe_expert_cache_prefetch,
redmoe_status_string, redmoe_abi_version).
"""

from __future__ import annotations

import ctypes as C
import os
import threading
from typing import Dict, Optional, Sequence

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libredmoe.so")
ABI_VERSION = 1
DTYPES = {"f32": 0, "bf16": 1, "int4g32": 2, "int2g32": 3}
STATUS = {0: "REDMOE_OK", 1: "REDMOE_ERR_INVALID_ARG", 2: "REDMOE_ERR_UNSUPPORTED", 3: "REDMOE_ERR_WORKSPACE",
          4: "REDMOE_ERR_CUDA", 5: "REDMOE_ERR_TIMEOUT"}
# entry points declared in include/redmoe.h
SYMBOLS = ("redmoe_abi_version", "redmoe_status_string", "redmoe_workspace_bytes", "redmoe_workspace_init",
           "redmoe_forward", "redmoe_router", "redmoe_route_build", "redmoe_forward_stack",
           "redmoe_check_timeout", "redmoe_forward_noalloc", "redmoe_selftest_wait_limit",
           "redmoe_fill_shared_memory", "redmoe_forward_cached", "redmoe_expert_cache_slot_bytes",
           "redmoe_expert_cache_init", "redmoe_forward_host_experts", "redmoe_expert_cache_prefetch",
           "redmoe_workspace_bytes_host", "redmoe_forward_host", "redmoe_forward_stack_host")

_lock = threading.Lock()
_lib = None


class RedmoeError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = int(status)
        super().__init__(f"{where}: {STATUS.get(self.status, self.status)} ({redmoe_status_string(self.status)})")


class _Layer(C.Structure):
    _fields_ = [
        ("hidden", C.c_int32), ("n_experts", C.c_int32), ("top_k", C.c_int32), ("inter", C.c_int32),
        ("shared_inter", C.c_int32), ("x_dtype", C.c_int32), ("router_dtype", C.c_int32),
        ("expert_dtype", C.c_int32),
        ("router_w", C.c_void_p), ("router_bias", C.c_void_p), ("shared_gate_w", C.c_void_p),
        ("w_gate", C.c_void_p), ("w_up", C.c_void_p), ("w_down", C.c_void_p),
        ("s_gate", C.c_void_p), ("s_up", C.c_void_p), ("s_down", C.c_void_p),
        ("sh_gate", C.c_void_p), ("sh_up", C.c_void_p), ("sh_down", C.c_void_p),
        ("sh_s_gate", C.c_void_p), ("sh_s_up", C.c_void_p), ("sh_s_down", C.c_void_p),
    ]


class _ExpertCache(C.Structure):
    _fields_ = [("n_slots", C.c_int32), ("slot_gate", C.c_void_p), ("slot_up", C.c_void_p), ("slot_down", C.c_void_p),
                ("slot_s_gate", C.c_void_p), ("slot_s_up", C.c_void_p), ("slot_s_down", C.c_void_p),
                ("slot_of", C.c_void_p), ("expert_in", C.c_void_p), ("hot", C.c_void_p), ("stats", C.c_void_p),
                ("fill", C.c_void_p)]


class _RouteDebug(C.Structure):
    _fields_ = [("counts", C.c_void_p), ("offsets", C.c_void_p), ("perm", C.c_void_p)]


def load():
    """Load libredmoe.so (built in-tree). Raises if it has not been built."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m sparse_moe_gemv_b200.build`")
        lib = C.CDLL(LIB_PATH)
        P, i32, sz = C.c_void_p, C.c_int32, C.c_size_t
        lib.redmoe_abi_version.restype = i32
        lib.redmoe_abi_version.argtypes = []
        lib.redmoe_status_string.restype = C.c_char_p
        lib.redmoe_status_string.argtypes = [i32]
        lib.redmoe_workspace_bytes.restype = sz
        lib.redmoe_workspace_bytes.argtypes = [P, i32]
        lib.redmoe_workspace_init.restype = i32
        lib.redmoe_workspace_init.argtypes = [P, sz, P]
        lib.redmoe_forward.restype = i32
        lib.redmoe_forward.argtypes = [P, P, i32, P, P, P, P, sz, P, P]
        lib.redmoe_router.restype = i32
        lib.redmoe_router.argtypes = [P, P, i32, P, P, P, P, P, sz, P]
        lib.redmoe_route_build.restype = i32
        lib.redmoe_route_build.argtypes = [P, i32, i32, i32, P, P, P, P, sz, P]
        lib.redmoe_forward_stack.restype = i32
        lib.redmoe_forward_stack.argtypes = [P, i32, P, i32, P, P, P, P, sz, P]
        lib.redmoe_check_timeout.restype = i32
        lib.redmoe_check_timeout.argtypes = [P, P]
        lib.redmoe_forward_noalloc.restype = i32
        lib.redmoe_forward_noalloc.argtypes = [P, P, i32, P, P, P, P]
        lib.redmoe_selftest_wait_limit.restype = i32
        lib.redmoe_selftest_wait_limit.argtypes = [P, sz, i32, C.c_uint64, P]
        lib.redmoe_forward_cached.restype = i32
        lib.redmoe_forward_cached.argtypes = [P, P, i32, P, P, P, P, C.c_float, P, sz, P]
        lib.redmoe_expert_cache_slot_bytes.restype = sz
        lib.redmoe_expert_cache_slot_bytes.argtypes = [P]
        lib.redmoe_expert_cache_init.restype = i32
        lib.redmoe_expert_cache_init.argtypes = [P, P, P]
        lib.redmoe_forward_host_experts.restype = i32
        lib.redmoe_forward_host_experts.argtypes = [P, P, i32, P, P, P, P, P, sz, P]
        lib.redmoe_expert_cache_prefetch.restype = i32
        lib.redmoe_expert_cache_prefetch.argtypes = [P, P, P, i32, P, sz, P]
        lib.redmoe_fill_shared_memory.restype = i32
        lib.redmoe_fill_shared_memory.argtypes = [C.c_uint32, P]
        lib.redmoe_workspace_bytes_host.restype = sz
        lib.redmoe_workspace_bytes_host.argtypes = [P, i32]
        lib.redmoe_forward_host.restype = i32
        lib.redmoe_forward_host.argtypes = [P, P, i32, P, P, P, P, sz, P]
        lib.redmoe_forward_stack_host.restype = i32
        lib.redmoe_forward_stack_host.argtypes = [P, i32, P, i32, P, P, P, P, sz, P]
        if lib.redmoe_abi_version() != ABI_VERSION:
            raise RuntimeError("libredmoe.so ABI version mismatch")
        _lib = lib
        return lib


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _check(status: int, where: str):
    if status != 0:
        raise RedmoeError(status, where)


class Layer:
    """A layer's device tensors plus its C descriptor.

    `tensors` uses the names of the C struct (router_w, router_bias, shared_gate_w,
    w_gate, w_up, w_down, s_gate, s_up, s_down, sh_gate, sh_up, sh_down, sh_s_gate,
    sh_s_up, sh_s_down); the tensors are kept alive by this object.
    """

    def __init__(self, tensors: Dict[str, Optional[torch.Tensor]], hidden: int, n_experts: int, top_k: int,
                 inter: int, shared_inter: int, x_dtype: str = "bf16", router_dtype: str = "bf16",
                 expert_dtype: str = "bf16"):
        self.tensors = dict(tensors)
        s = _Layer()
        s.hidden, s.n_experts, s.top_k, s.inter, s.shared_inter = hidden, n_experts, top_k, inter, shared_inter
        s.x_dtype, s.router_dtype, s.expert_dtype = DTYPES[x_dtype], DTYPES[router_dtype], DTYPES[expert_dtype]
        for name, _ in _Layer._fields_[8:]:
            setattr(s, name, _ptr(self.tensors.get(name)))
        self.struct = s
        self.hidden, self.n_experts, self.top_k = hidden, n_experts, top_k
        self.inter, self.shared_inter = inter, shared_inter
        self.x_dtype, self.router_dtype, self.expert_dtype = x_dtype, router_dtype, expert_dtype

    @classmethod
    def from_shape(cls, tensors, shape):
        """`shape` has attributes H, E, k, I, Is, x_dtype, router_dtype, expert_dtype."""
        return cls(tensors, shape.H, shape.E, shape.k, shape.I, shape.Is, shape.x_dtype, shape.router_dtype,
                   shape.expert_dtype)

    @property
    def ref(self):
        return C.byref(self.struct)


def redmoe_abi_version() -> int:
    return int(load().redmoe_abi_version())


def redmoe_status_string(status: int) -> str:
    return load().redmoe_status_string(int(status)).decode()


def redmoe_workspace_bytes(layer: Layer, T: int) -> int:
    return int(load().redmoe_workspace_bytes(layer.ref, int(T)))


def redmoe_workspace_init(workspace: Optional[torch.Tensor], stream=None) -> None:
    """Zero a workspace's control block; None: the allocation-free scratch of this device."""
    nbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(load().redmoe_workspace_init(_ptr(workspace), nbytes, _stream(stream)), "redmoe_workspace_init")


def new_workspace(layer: Layer, T: int, device=None) -> torch.Tensor:
    """A zeroed workspace tensor of redmoe_workspace_bytes(layer, T) bytes."""
    n = redmoe_workspace_bytes(layer, T)
    if n == 0:
        raise ValueError("invalid layer or token count")
    return torch.zeros(n, dtype=torch.uint8, device=device or "cuda")


def redmoe_forward(layer: Layer, x: torch.Tensor, out: torch.Tensor, topk_ids: torch.Tensor, topk_w: torch.Tensor,
                   workspace: torch.Tensor, dbg: Optional[Sequence[torch.Tensor]] = None, stream=None,
                   T: Optional[int] = None) -> None:
    """out[T,H] fp32, topk_ids[T,k] int32, topk_w[T,k] fp32 <- layer(x[T,H])."""
    lib = load()
    dbg_s = None
    if dbg is not None:
        dbg_s = _RouteDebug(_ptr(dbg[0]), _ptr(dbg[1]), _ptr(dbg[2]))
    T = x.shape[0] if T is None else T
    st = lib.redmoe_forward(layer.ref, _ptr(x), int(T), _ptr(out), _ptr(topk_ids), _ptr(topk_w),
                            _ptr(workspace), workspace.numel() * workspace.element_size(),
                            None if dbg_s is None else C.byref(dbg_s), _stream(stream))
    _check(st, "redmoe_forward")


def redmoe_workspace_bytes_host(layer: Layer, T: int) -> int:
    return int(load().redmoe_workspace_bytes_host(layer.ref, int(T)))


def new_workspace_host(layer: Layer, T: int, device=None) -> torch.Tensor:
    """A zeroed workspace tensor of redmoe_workspace_bytes_host(layer, T) bytes."""
    n = redmoe_workspace_bytes_host(layer, T)
    if n == 0:
        raise ValueError("invalid layer or token count")
    return torch.zeros(n, dtype=torch.uint8, device=device or "cuda")


def redmoe_forward_host(layer: Layer, x_host: torch.Tensor, out_host: torch.Tensor, ids_host: torch.Tensor,
                        w_host: torch.Tensor, workspace: torch.Tensor, stream=None) -> None:
    """redmoe_forward with x and the results in host memory (pinned for asynchronous
    copies, and for results stored straight from the kernel at T <= 4). The results are
    valid once `stream` has been synchronised."""
    T = x_host.shape[0]
    st = load().redmoe_forward_host(layer.ref, _ptr(x_host), int(T), _ptr(out_host), _ptr(ids_host), _ptr(w_host),
                                    _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "redmoe_forward_host")


def redmoe_forward_cached(layer: Layer, x: torch.Tensor, out: torch.Tensor, topk_ids: torch.Tensor,
                          topk_w: torch.Tensor, cached: torch.Tensor, lam: float, workspace: torch.Tensor,
                          stream=None) -> None:
    """redmoe_forward with the opt-in cache-aware routing bias: cached [E] uint8 device mask
    of experts resident in the caller's cache, lam >= 0 (0: plain routing)."""
    T = x.shape[0]
    st = load().redmoe_forward_cached(layer.ref, _ptr(x), int(T), _ptr(out), _ptr(topk_ids), _ptr(topk_w),
                                      _ptr(cached), float(lam), _ptr(workspace),
                                      workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "redmoe_forward_cached")


def redmoe_router(layer: Layer, x: torch.Tensor, topk_ids: torch.Tensor, topk_w: torch.Tensor,
                  shared_gate: torch.Tensor, workspace: torch.Tensor, logits: Optional[torch.Tensor] = None,
                  stream=None) -> None:
    st = load().redmoe_router(layer.ref, _ptr(x), int(x.shape[0]), _ptr(topk_ids), _ptr(topk_w), _ptr(shared_gate),
                              _ptr(logits), _ptr(workspace), workspace.numel() * workspace.element_size(),
                              _stream(stream))
    _check(st, "redmoe_router")


def redmoe_route_build(topk_ids: torch.Tensor, n_experts: int, counts: torch.Tensor, offsets: torch.Tensor,
                       perm: torch.Tensor, stream=None) -> None:
    T, k = topk_ids.shape
    st = load().redmoe_route_build(_ptr(topk_ids), int(T), int(k), int(n_experts), _ptr(counts), _ptr(offsets),
                                   _ptr(perm), None, 0, _stream(stream))
    _check(st, "redmoe_route_build")


def redmoe_forward_stack(layers: Sequence[Layer], xs: Sequence[torch.Tensor], outs: Sequence[torch.Tensor],
                         ids: Sequence[torch.Tensor], ws: Sequence[torch.Tensor], workspace: torch.Tensor,
                         stream=None) -> None:
    n = len(layers)
    arr = (_Layer * n)(*[l.struct for l in layers])
    P = C.c_void_p * n
    T = xs[0].shape[0] if n else 0
    st = load().redmoe_forward_stack(C.cast(arr, C.c_void_p), n, C.cast(P(*[_ptr(t) for t in xs]), C.c_void_p),
                                     int(T), C.cast(P(*[_ptr(t) for t in outs]), C.c_void_p),
                                     C.cast(P(*[_ptr(t) for t in ids]), C.c_void_p),
                                     C.cast(P(*[_ptr(t) for t in ws]), C.c_void_p), _ptr(workspace),
                                     workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "redmoe_forward_stack")


def redmoe_forward_stack_host(layers: Sequence[Layer], xs: Sequence[torch.Tensor], outs: Sequence[torch.Tensor],
                              ids: Sequence[torch.Tensor], ws: Sequence[torch.Tensor], workspace: torch.Tensor,
                              stream=None) -> None:
    """redmoe_forward_stack with every x and result in host memory (pinned for the
    copy-free one-launch path); valid once `stream` has been synchronised."""
    n = len(layers)
    arr = (_Layer * n)(*[l.struct for l in layers])
    P = C.c_void_p * n
    T = xs[0].shape[0] if n else 0
    st = load().redmoe_forward_stack_host(C.cast(arr, C.c_void_p), n, C.cast(P(*[_ptr(t) for t in xs]), C.c_void_p),
                                          int(T), C.cast(P(*[_ptr(t) for t in outs]), C.c_void_p),
                                          C.cast(P(*[_ptr(t) for t in ids]), C.c_void_p),
                                          C.cast(P(*[_ptr(t) for t in ws]), C.c_void_p), _ptr(workspace),
                                          workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "redmoe_forward_stack_host")


def redmoe_check_timeout(workspace: Optional[torch.Tensor], stream=None) -> None:
    """Raise REDMOE_ERR_TIMEOUT if a bounded in-kernel wait gave up; None: the
    allocation-free scratch of this device."""
    _check(load().redmoe_check_timeout(_ptr(workspace), _stream(stream)), "redmoe_check_timeout")


def redmoe_forward_noalloc(layer: Layer, x: torch.Tensor, out: torch.Tensor, topk_ids: torch.Tensor,
                           topk_w: torch.Tensor, stream=None) -> None:
    """redmoe_forward for 1..4 token rows without a workspace argument.

    For callers that cannot allocate device memory (a strict stream capture, a loop that
    must not touch the allocator, a plug-in without a memory budget of its own): the
    scratch is a fixed 1 MiB array inside the library, shared by every call on the
    device. Calls must not overlap on the GPU; the first call on a device must not be
    made inside a stream capture (it looks up the array's address). A bounded wait that
    gave up is reported by redmoe_check_timeout(None) and cleared by
    redmoe_workspace_init(None).
    """
    st = load().redmoe_forward_noalloc(layer.ref, _ptr(x), int(x.shape[0]), _ptr(out), _ptr(topk_ids),
                                       _ptr(topk_w), _stream(stream))
    _check(st, "redmoe_forward_noalloc")


def redmoe_selftest_wait_limit(workspace: Optional[torch.Tensor], withhold: int, limit_ns: int, stream=None) -> None:
    """Run the bounded-wait self-test: block `withhold` skips a grid barrier, the others
    give up after limit_ns and record a timeout (read it with redmoe_check_timeout)."""
    nbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(load().redmoe_selftest_wait_limit(_ptr(workspace), nbytes, int(withhold), int(limit_ns), _stream(stream)),
           "redmoe_selftest_wait_limit")


NAN_PATTERN = 0x7FC00000


def redmoe_fill_shared_memory(pattern: int = NAN_PATTERN, stream=None) -> None:
    """Fill every SM's shared memory with a 32-bit pattern before the next launch."""
    _check(load().redmoe_fill_shared_memory(int(pattern) & 0xFFFFFFFF, _stream(stream)), "redmoe_fill_shared_memory")


class ExpertCache:
    """A bounded device cache of routed experts (redmoe_expert_cache): n_slots slots in the
    layer's expert dtype plus the directory; device tensors owned by this object."""

    def __init__(self, layer: "Layer", n_slots: int, device=None):
        dev = device or "cuda"
        H, I, E = layer.hidden, layer.inter, layer.n_experts
        dt = layer.expert_dtype
        per = {"bf16": 2.0, "f32": 4.0, "int4g32": 0.5, "int2g32": 0.25}[dt]

        def stack(n, k):
            return torch.empty(n_slots, int(n * k * per), dtype=torch.uint8, device=dev)

        t = {"slot_gate": stack(I, H), "slot_up": stack(I, H), "slot_down": stack(H, I)}
        if dt in ("int4g32", "int2g32"):
            t.update(slot_s_gate=torch.empty(n_slots, I * H // 32, dtype=torch.bfloat16, device=dev),
                     slot_s_up=torch.empty(n_slots, I * H // 32, dtype=torch.bfloat16, device=dev),
                     slot_s_down=torch.empty(n_slots, H * I // 32, dtype=torch.bfloat16, device=dev))
        t.update(slot_of=torch.empty(E, dtype=torch.int32, device=dev),
                 expert_in=torch.empty(n_slots, dtype=torch.int32, device=dev),
                 hot=torch.empty(E, dtype=torch.float32, device=dev),
                 stats=torch.empty(4, dtype=torch.int32, device=dev),
                 fill=torch.empty(257, dtype=torch.int32, device=dev))
        self.tensors = t
        st = _ExpertCache()
        st.n_slots = n_slots
        for name, _ in _ExpertCache._fields_[1:]:
            setattr(st, name, _ptr(t.get(name)))
        self.struct = st
        self.n_slots = n_slots

    @property
    def ref(self):
        return C.byref(self.struct)


def redmoe_expert_cache_slot_bytes(layer: Layer) -> int:
    return int(load().redmoe_expert_cache_slot_bytes(layer.ref))


def redmoe_expert_cache_init(layer: Layer, cache: ExpertCache, stream=None) -> None:
    _check(load().redmoe_expert_cache_init(layer.ref, cache.ref, _stream(stream)), "redmoe_expert_cache_init")


def redmoe_forward_host_experts(layer: Layer, x: torch.Tensor, out: torch.Tensor, topk_ids: torch.Tensor,
                                topk_w: torch.Tensor, cache: ExpertCache, workspace: torch.Tensor, stream=None) -> None:
    """One token through a layer whose routed experts may be in pinned host memory."""
    st = load().redmoe_forward_host_experts(layer.ref, _ptr(x), int(x.shape[0]), _ptr(out), _ptr(topk_ids),
                                            _ptr(topk_w), cache.ref, _ptr(workspace),
                                            workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "redmoe_forward_host_experts")


def redmoe_expert_cache_prefetch(layer: Layer, cache: ExpertCache, ids: torch.Tensor, workspace: torch.Tensor,
                                 stream=None) -> None:
    st = load().redmoe_expert_cache_prefetch(layer.ref, cache.ref, _ptr(ids), int(ids.numel()), _ptr(workspace),
                                             workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "redmoe_expert_cache_prefetch")
