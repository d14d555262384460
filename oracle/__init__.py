"""Python marshalling for the fp64 CPU oracle in ``moe_oracle.c``.

TEST INFRASTRUCTURE ONLY: imported by the tests, by ``__graft_entry__.smoke()`` and by
the benchmark's CPU-baseline leg, never by the product package. It only moves numpy
arrays into the C oracle and back; all arithmetic of the layer is in ``moe_oracle.c``.

A layer is a dict of host numpy arrays (bf16 as uint16 bit patterns) with the names
and layouts of ``moe_inputs``. Routed expert tensors may be full stacks [E, N, K] or
``{expert_id: [N, K] array}`` dicts holding only some experts; the oracle reports
``OracleError('missing expert')`` if the routing needs one that is absent.
"""

from __future__ import annotations

import ctypes as C
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_DT = {"f32": 0, "bf16": 1, "int4g32": 2, "int2g32": 3}
_lock = threading.Lock()
_handle = None


class OracleError(RuntimeError):
    pass


def build(force: bool = False) -> str:
    """Compile moe_oracle.c into oracle/liboracle.so with gcc (OpenMP over tokens)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-Wall", "-fopenmp", "-fPIC", "-shared",
                               _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


class _Layer(C.Structure):
    _fields_ = [
        ("H", C.c_int32), ("E", C.c_int32), ("k", C.c_int32), ("I", C.c_int32), ("Is", C.c_int32),
        ("x_dtype", C.c_int32), ("router_dtype", C.c_int32), ("expert_dtype", C.c_int32),
        ("router_w", C.c_void_p), ("router_bias", C.c_void_p), ("shared_gate_w", C.c_void_p),
        ("gate", C.c_void_p), ("up", C.c_void_p), ("down", C.c_void_p),
        ("gate_scale", C.c_void_p), ("up_scale", C.c_void_p), ("down_scale", C.c_void_p),
        ("sh_gate", C.c_void_p), ("sh_up", C.c_void_p), ("sh_down", C.c_void_p),
        ("sh_gate_scale", C.c_void_p), ("sh_up_scale", C.c_void_p), ("sh_down_scale", C.c_void_p),
    ]


def _lib():
    global _handle
    with _lock:
        if _handle is None:
            # ORACLE_LIB names another build of moe_oracle.c (the mutation tests use it)
            lib = C.CDLL(os.environ.get("ORACLE_LIB") or build())
            P = C.c_void_p
            i32 = C.c_int32
            lib.orc_router.argtypes = [P, i32, P, P, P, P, P, P]
            lib.orc_experts.argtypes = [P, i32, P, P, P, P, P]
            lib.orc_forward.argtypes = [P, i32, P, P, P, P, P, P]
            lib.orc_brute.argtypes = [P, i32, P, P, P, P]
            lib.orc_expert_ffn.argtypes = [P, i32, P, P]
            lib.orc_route_build.argtypes = [i32, i32, i32, P, P, P, P]
            lib.orc_dequant_int4.argtypes = [i32, i32, P, P, P]
            lib.orc_dequant_int2.argtypes = [i32, i32, P, P, P]
            lib.orc_renorm.argtypes = [i32, i32, P, P, P]
            lib.orc_cache_route.argtypes = [i32, i32, i32, P, P, C.c_double, P, P, P]
            lib.orc_num_threads.argtypes = []
            lib.orc_set_num_threads.argtypes = [i32]
            lib.orc_set_num_threads.restype = None
            _handle = lib
    return _handle


def _ptr(a):
    return None if a is None else a.ctypes.data


def _check(rc):
    if rc == 0:
        return
    raise OracleError({-1: "bad argument", -2: "missing expert", -3: "out of memory"}.get(rc, str(rc)))


class _Marshalled:
    """Keeps the arrays and pointer tables of one ctypes layer struct alive."""

    def __init__(self, layer: dict, shape):
        self.keep = []
        E = shape.E
        s = _Layer()
        s.H, s.E, s.k, s.I, s.Is = shape.H, shape.E, shape.k, shape.I, shape.Is
        s.x_dtype = _DT[shape.x_dtype]
        s.router_dtype = _DT[shape.router_dtype]
        s.expert_dtype = _DT[shape.expert_dtype]
        s.router_w = _ptr(self._arr(layer["router_w"]))
        s.router_bias = _ptr(self._arr(layer.get("router_bias"), np.float32))
        s.shared_gate_w = _ptr(self._arr(layer["shared_gate_w"]))
        s.gate = self._table(layer.get("w_gate"), E)
        s.up = self._table(layer.get("w_up"), E)
        s.down = self._table(layer.get("w_down"), E)
        s.gate_scale = self._table(layer.get("s_gate"), E)
        s.up_scale = self._table(layer.get("s_up"), E)
        s.down_scale = self._table(layer.get("s_down"), E)
        for name in ("sh_gate", "sh_up", "sh_down"):
            setattr(s, name, _ptr(self._arr(layer.get(name))))
        for name, key in (("sh_gate_scale", "sh_s_gate"), ("sh_up_scale", "sh_s_up"),
                          ("sh_down_scale", "sh_s_down")):
            setattr(s, name, _ptr(self._arr(layer.get(key))))
        self.struct = s

    def _arr(self, a, dtype=None):
        if a is None:
            return None
        a = np.ascontiguousarray(a if dtype is None else a.astype(dtype, copy=False))
        self.keep.append(a)
        return a

    def _table(self, w, E):
        if w is None:
            return None
        tab = (C.c_void_p * E)()
        if isinstance(w, dict):
            for e, a in w.items():
                tab[int(e)] = _ptr(self._arr(a))
        else:
            w = self._arr(w)
            stride = w.strides[0]
            for e in range(E):
                tab[e] = w.ctypes.data + e * stride
        self.keep.append(tab)
        return C.cast(tab, C.c_void_p).value

    @property
    def ref(self):
        return C.byref(self.struct)


def _x(x):
    x = np.ascontiguousarray(x)
    return x


def router(layer, shape, x):
    """Router stage: dict(logits [T,E], probs [T,E], ids [T,k], w [T,k], s [T]) in fp64."""
    x = _x(x)
    T = x.shape[0]
    m = _Marshalled(layer, shape)
    logits = np.zeros((T, shape.E), np.float64)
    probs = np.zeros((T, shape.E), np.float64)
    ids = np.zeros((T, shape.k), np.int32)
    w = np.zeros((T, shape.k), np.float64)
    s = np.zeros((T,), np.float64)
    _check(_lib().orc_router(m.ref, T, _ptr(x), _ptr(logits), _ptr(probs), _ptr(ids), _ptr(w), _ptr(s)))
    return dict(logits=logits, probs=probs, ids=ids, w=w, s=s)


def experts(layer, shape, x, ids, w, s):
    """out [T,H] = sum_j w y_ids + s y_shared, for the routing given (fp64)."""
    x = _x(x)
    T = x.shape[0]
    m = _Marshalled(layer, shape)
    ids = np.ascontiguousarray(ids, np.int32)
    w = np.ascontiguousarray(w, np.float64)
    s = np.ascontiguousarray(s, np.float64)
    out = np.zeros((T, shape.H), np.float64)
    _check(_lib().orc_experts(m.ref, T, _ptr(x), _ptr(ids), _ptr(w), _ptr(s), _ptr(out)))
    return out


def forward(layer, shape, x):
    """Whole layer: dict(out, ids, w, s, logits)."""
    x = _x(x)
    T = x.shape[0]
    m = _Marshalled(layer, shape)
    out = np.zeros((T, shape.H), np.float64)
    ids = np.zeros((T, shape.k), np.int32)
    w = np.zeros((T, shape.k), np.float64)
    s = np.zeros((T,), np.float64)
    logits = np.zeros((T, shape.E), np.float64)
    _check(_lib().orc_forward(m.ref, T, _ptr(x), _ptr(out), _ptr(ids), _ptr(w), _ptr(s), _ptr(logits)))
    return dict(out=out, ids=ids, w=w, s=s, logits=logits)


def brute(layer, shape, x):
    """Dense all-experts reference (tiny shapes): dict(out, ids, w)."""
    x = _x(x)
    T = x.shape[0]
    m = _Marshalled(layer, shape)
    out = np.zeros((T, shape.H), np.float64)
    ids = np.zeros((T, shape.k), np.int32)
    w = np.zeros((T, shape.k), np.float64)
    _check(_lib().orc_brute(m.ref, T, _ptr(x), _ptr(out), _ptr(ids), _ptr(w)))
    return dict(out=out, ids=ids, w=w)


def expert_ffn(layer, shape, e, xd):
    """One expert (e = -1: shared) on one token given as fp64 [H]."""
    m = _Marshalled(layer, shape)
    xd = np.ascontiguousarray(xd, np.float64)
    y = np.zeros((shape.H,), np.float64)
    _check(_lib().orc_expert_ffn(m.ref, int(e), _ptr(xd), _ptr(y)))
    return y


def renorm(logits_row, ids):
    """Renormalised softmax weights of the expert subset `ids` of one token."""
    logits_row = np.ascontiguousarray(logits_row, np.float64)
    ids = np.ascontiguousarray(ids, np.int32)
    w = np.zeros(ids.shape, np.float64)
    _check(_lib().orc_renorm(logits_row.shape[0], ids.shape[0], _ptr(logits_row), _ptr(ids), _ptr(w)))
    return w


def cache_route(logits, cached, lam, k):
    """Opt-in cache-aware routing of logits [T, E]: selection by z + lam * (max z - min z)
    * cached, weights from the unbiased softmax renormalised over the selection.
    Returns dict(ids [T,k] int32, w [T,k], biased [T,E])."""
    logits = np.ascontiguousarray(logits, np.float64)
    T, E = logits.shape
    cached = np.ascontiguousarray(cached, np.uint8)
    ids = np.zeros((T, k), np.int32)
    w = np.zeros((T, k), np.float64)
    biased = np.zeros((T, E), np.float64)
    _check(_lib().orc_cache_route(T, E, k, _ptr(logits), _ptr(cached), float(lam), _ptr(ids), _ptr(w),
                                  _ptr(biased)))
    return dict(ids=ids, w=w, biased=biased)


def route_build(ids, E):
    """Stable token->expert grouping: (counts [E], offsets [E+1], perm [T*k]) int32."""
    ids = np.ascontiguousarray(ids, np.int32)
    T, k = ids.shape
    counts = np.zeros((E,), np.int32)
    offsets = np.zeros((E + 1,), np.int32)
    perm = np.zeros((T * k,), np.int32)
    _check(_lib().orc_route_build(T, k, E, _ptr(ids), _ptr(counts), _ptr(offsets), _ptr(perm)))
    return counts, offsets, perm


def dequant_int4(packed, scales):
    """Dequantise an int4 group-32 matrix (packed u8 [N, K/2], scales bf16 bits [N, K/32])."""
    packed = np.ascontiguousarray(packed, np.uint8)
    scales = np.ascontiguousarray(scales, np.uint16)
    N, K = packed.shape[0], packed.shape[1] * 2
    out = np.zeros((N, K), np.float64)
    _check(_lib().orc_dequant_int4(N, K, _ptr(packed), _ptr(scales), _ptr(out)))
    return out


def dequant_int2(packed, scales):
    """Dequantise an int2 group-32 matrix (packed u8 [N, K/4], scales bf16 bits [N, K/32])."""
    packed = np.ascontiguousarray(packed, np.uint8)
    scales = np.ascontiguousarray(scales, np.uint16)
    N, K = packed.shape[0], packed.shape[1] * 4
    out = np.zeros((N, K), np.float64)
    _check(_lib().orc_dequant_int2(N, K, _ptr(packed), _ptr(scales), _ptr(out)))
    return out


def num_threads():
    return int(_lib().orc_num_threads())


def set_num_threads(n):
    """OpenMP threads of later oracle calls (timing only; results do not depend on it)."""
    _lib().orc_set_num_threads(int(n))
