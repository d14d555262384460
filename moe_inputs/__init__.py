"""Seeded synthetic inputs for one sparse mixture-of-experts FFN layer.

This module only draws random numbers and lays them out in memory. It holds none
of the layer's arithmetic (no router, no softmax, no top-k, no SwiGLU, no combine,
no dequantisation), so both the CUDA path and the fp64 oracle can take their inputs
from it without sharing any of the method.

Shapes follow the Qwen3-Next-80B-A3B MoE block as given on the "Architecture" page
("Qwen3-Next shape": hidden 2048, 512 routed experts, top-10 per token, one shared
expert, expert intermediate 512). The merged expert tensors keep the expert as the
outer dimension, as the "Red Lite v0.3 streaming development" page describes for
``blk.N.ffn_{gate,up,down}_exps.weight`` ("Implemented in dev1").

Layout of one layer (every tensor contiguous, row-major):

=================  ===============  ==========================================
name               shape            dtype
=================  ===============  ==========================================
router_w           [E, H]           f32 | bf16
router_bias        [E]              f32, or None (prefill Zipf workload only)
shared_gate_w      [H]              same dtype as router_w
w_gate, w_up       [E, I, H]        f32 | bf16 | u8 packed int4 [E, I, H/2] | int2 [E, I, H/4]
w_down             [E, H, I]        f32 | bf16 | u8 packed int4 [E, H, I/2] | int2 [E, H, I/4]
s_gate, s_up       [E, I, H/32]     bf16 scales (int4 / int2 only)
s_down             [E, H, I/32]     bf16 scales (int4 / int2 only)
sh_gate, sh_up     [Is, H]          expert dtype (packed like the routed experts)
sh_down            [H, Is]          expert dtype
sh_s_*             [..., K/32]      bf16 scales (int4 / int2 only)
=================  ===============  ==========================================

int4 group-32 storage format (defined here; the pages ship GGUF IQ formats only):
per row and per group of 32 consecutive K elements, scale ``s = bf16(amax / 7)``
(round to nearest even), codes ``q = clamp(round_half_even(w / float(s)), -7, 7)``
(``q = 0`` when ``s == 0``) computed in fp32, stored as the nibble ``q + 8``.
Byte ``b`` of a row holds element ``2b`` in its low nibble and ``2b + 1`` in its
high nibble. A reader recovers ``float(s) * (nibble - 8)``. Quantisation is input
generation: the kernels and the oracle read the same packed bytes.

int2 group-32 storage format (also defined here; the lower-bit counterpart of int4 g32,
after the 2-bit expert files the pages ship): per row and per group of 32 consecutive K
elements, scale ``s = bf16(amax / 1)``, codes ``q = clamp(round_half_even(w / float(s)),
-1, 1)`` (``q = 0`` when ``s == 0``) computed in fp32, stored as the 2-bit code ``q + 2``.
Byte ``b`` of a row holds elements ``4b, 4b+1, 4b+2, 4b+3`` in bits 0-1, 2-3, 4-5 and 6-7.
A reader recovers ``float(s) * (code - 2)`` (code 0, which the quantiser never writes,
reads as -2).
"""

from __future__ import annotations

import dataclasses
import math
from typing import Dict, Optional

import numpy as np
import torch

DTYPES = ("f32", "bf16", "int4g32", "int2g32")


@dataclasses.dataclass(frozen=True)
class LayerShape:
    H: int          # hidden
    E: int          # routed experts
    k: int          # experts per token
    I: int          # routed expert intermediate
    Is: int         # shared expert intermediate
    x_dtype: str = "bf16"
    router_dtype: str = "bf16"
    expert_dtype: str = "bf16"
    sigma: float = 0.02      # std of every weight before rounding
    rms_norm_x: bool = True  # x = z / rms(z), z ~ N(0, 1)
    zipf_s: Optional[float] = None  # per-expert Zipf(s) router-logit offset


# The five workloads. Each entry: layer shape, tokens per call, layers in the stack.
WORKLOADS: Dict[str, dict] = {
    # Tiny fp32 layer for exact-tolerance parity (x ~ N(0,1), not RMS-normalised).
    "tiny_f32": dict(shape=LayerShape(H=256, E=16, k=2, I=64, Is=64, x_dtype="f32",
                                      router_dtype="f32", expert_dtype="f32",
                                      sigma=0.05, rms_norm_x=False),
                     T=4, layers=1, seed_base=0),
    # Qwen3-Next-shaped layer, bf16 weights, one decode token.
    "decode_t1_bf16": dict(shape=LayerShape(H=2048, E=512, k=10, I=512, Is=512),
                           T=1, layers=1, seed_base=1000),
    # Few-row decode (parallel-2 and 2/3-row verify): 12 distinct layers back to back.
    "fewrow_bf16": dict(shape=LayerShape(H=2048, E=512, k=10, I=512, Is=512),
                        T=2, layers=12, seed_base=2000),
    # 2048-token prefill chunk with a Zipf(1.1) per-expert router-logit offset.
    "prefill_zipf_bf16": dict(shape=LayerShape(H=2048, E=512, k=10, I=512, Is=512,
                                               zipf_s=1.1),
                              T=2048, layers=1, seed_base=3000),
    # 48 distinct int4 group-32 layers, one decode token, router in bf16.
    "int4_decode_48": dict(shape=LayerShape(H=2048, E=512, k=10, I=512, Is=512,
                                            expert_dtype="int4g32"),
                           T=1, layers=48, seed_base=4000),
}


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=torch.device(device))
    g.manual_seed(int(seed))
    return g


def _normal(shape, sigma: float, g: torch.Generator, device) -> torch.Tensor:
    return torch.randn(*shape, generator=g, device=device, dtype=torch.float32) * sigma


def _store(w: torch.Tensor, dtype: str) -> torch.Tensor:
    if dtype == "f32":
        return w.contiguous()
    if dtype == "bf16":
        return w.to(torch.bfloat16).contiguous()
    raise ValueError(dtype)


def quantize_int4g32(w: torch.Tensor):
    """Pack an fp32 matrix [..., N, K] into the int4 group-32 format described above.

    Returns (packed u8 [..., N, K/2], scales bf16 [..., N, K/32]).
    """
    K = w.shape[-1]
    if K % 32:
        raise ValueError("K must be a multiple of 32 for int4 group-32")
    grp = w.reshape(*w.shape[:-1], K // 32, 32)
    amax = grp.abs().amax(dim=-1)
    s = (amax / 7.0).to(torch.bfloat16)
    sf = s.to(torch.float32).unsqueeze(-1)
    safe = torch.where(sf == 0, torch.ones_like(sf), sf)
    q = torch.round(grp / safe).clamp_(-7, 7)
    q = torch.where(sf == 0, torch.zeros_like(q), q)
    u = (q + 8).to(torch.uint8).reshape(*w.shape[:-1], K)
    packed = (u[..., 0::2] | (u[..., 1::2] << 4)).contiguous()
    return packed, s.contiguous()


def quantize_int2g32(w: torch.Tensor):
    """Pack an fp32 matrix [..., N, K] into the int2 group-32 format described above.

    Returns (packed u8 [..., N, K/4], scales bf16 [..., N, K/32]).
    """
    K = w.shape[-1]
    if K % 32:
        raise ValueError("K must be a multiple of 32 for int2 group-32")
    grp = w.reshape(*w.shape[:-1], K // 32, 32)
    amax = grp.abs().amax(dim=-1)
    s = amax.to(torch.bfloat16)
    sf = s.to(torch.float32).unsqueeze(-1)
    safe = torch.where(sf == 0, torch.ones_like(sf), sf)
    q = torch.round(grp / safe).clamp_(-1, 1)
    q = torch.where(sf == 0, torch.zeros_like(q), q)
    u = (q + 2).to(torch.uint8).reshape(*w.shape[:-1], K)
    packed = (u[..., 0::4] | (u[..., 1::4] << 2) | (u[..., 2::4] << 4) | (u[..., 3::4] << 6)).contiguous()
    return packed, s.contiguous()


QUANTIZERS = {"int4g32": (quantize_int4g32, 2), "int2g32": (quantize_int2g32, 4)}  # (packer, elements per byte)


def _expert_tensor(shape, sigma, dtype, g, device, chunk=64):
    """Draw [E, N, K] weights expert-chunk by expert-chunk (bounded fp32 temporaries)."""
    E, N, K = shape
    if dtype not in QUANTIZERS:
        tdt = torch.float32 if dtype == "f32" else torch.bfloat16
        out = torch.empty(E, N, K, dtype=tdt, device=device)
        for e0 in range(0, E, chunk):
            e1 = min(E, e0 + chunk)
            out[e0:e1] = _store(_normal((e1 - e0, N, K), sigma, g, device), dtype)
        return out, None
    quant, per_byte = QUANTIZERS[dtype]
    packed = torch.empty(E, N, K // per_byte, dtype=torch.uint8, device=device)
    scales = torch.empty(E, N, K // 32, dtype=torch.bfloat16, device=device)
    for e0 in range(0, E, chunk):
        e1 = min(E, e0 + chunk)
        p, s = quant(_normal((e1 - e0, N, K), sigma, g, device))
        packed[e0:e1] = p
        scales[e0:e1] = s
    return packed, scales


def _shared_tensor(shape, sigma, dtype, g, device):
    w, s = _expert_tensor((1,) + tuple(shape), sigma, dtype, g, device)
    return w[0], (None if s is None else s[0])


def zipf_log_offsets(E: int, s: float, g: torch.Generator, device) -> torch.Tensor:
    """Per-expert router-logit offset b[pi(r)] = ln(r^-s / sum_r' r'^-s), r = 1..E.

    pi is a seeded permutation of the expert ids, so the hot experts are spread
    over the id range. Computed in fp64, stored fp32.
    """
    r = np.arange(1, E + 1, dtype=np.float64)
    pr = r ** (-s)
    logp = np.log(pr / pr.sum())
    perm = torch.randperm(E, generator=g, device=device).cpu().numpy()
    b = np.empty(E, dtype=np.float64)
    b[perm] = logp
    return torch.from_numpy(b.astype(np.float32)).to(device)


def make_layer(shape: LayerShape, seed: int, device="cpu") -> Dict[str, Optional[torch.Tensor]]:
    """All weights of one layer, drawn from one generator in a fixed order."""
    g = _gen(seed, device)
    H, E, I, Is = shape.H, shape.E, shape.I, shape.Is
    sig = shape.sigma
    L: Dict[str, Optional[torch.Tensor]] = {}
    L["router_w"] = _store(_normal((E, H), sig, g, device), shape.router_dtype)
    L["shared_gate_w"] = _store(_normal((H,), sig, g, device), shape.router_dtype)
    L["w_gate"], L["s_gate"] = _expert_tensor((E, I, H), sig, shape.expert_dtype, g, device)
    L["w_up"], L["s_up"] = _expert_tensor((E, I, H), sig, shape.expert_dtype, g, device)
    L["w_down"], L["s_down"] = _expert_tensor((E, H, I), sig, shape.expert_dtype, g, device)
    L["sh_gate"], L["sh_s_gate"] = _shared_tensor((Is, H), sig, shape.expert_dtype, g, device)
    L["sh_up"], L["sh_s_up"] = _shared_tensor((Is, H), sig, shape.expert_dtype, g, device)
    L["sh_down"], L["sh_s_down"] = _shared_tensor((H, Is), sig, shape.expert_dtype, g, device)
    L["router_bias"] = None
    if shape.zipf_s is not None:
        L["router_bias"] = zipf_log_offsets(E, shape.zipf_s, _gen(seed + 777_777, device), device)
    return L


def make_x(shape: LayerShape, T: int, seed: int, device="cpu") -> torch.Tensor:
    """Token activations [T, H]: z ~ N(0,1) fp32, optionally z / sqrt(mean_h z^2), then stored."""
    g = _gen(seed + 500_000, device)
    z = torch.randn(T, shape.H, generator=g, device=device, dtype=torch.float32)
    if shape.rms_norm_x and T > 0:
        z = z / torch.sqrt((z * z).mean(dim=1, keepdim=True))
    return _store(z, shape.x_dtype)


def random_topk_ids(T: int, k: int, E: int, seed: int, device="cpu", zipf_s: Optional[float] = None):
    """Valid top-k id rows (k distinct experts per token) for grouping tests.

    With zipf_s the experts are drawn without replacement with Zipf(s) weights, so
    a few experts collect most rows and many collect none.
    """
    g = _gen(seed, device="cpu")
    if zipf_s is None:
        w = torch.ones(E, dtype=torch.float64)
    else:
        w = torch.arange(1, E + 1, dtype=torch.float64) ** (-zipf_s)
        w = w[torch.randperm(E, generator=g)]
    ids = torch.multinomial(w.expand(max(T, 1), E), k, replacement=False, generator=g)[:T]
    return ids.to(torch.int32).to(device).contiguous()


# ---------------------------------------------------------------- host views
def to_numpy(t: Optional[torch.Tensor]):
    """Host numpy view of a tensor: bf16 becomes its uint16 bit pattern."""
    if t is None:
        return None
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.uint16).numpy()
    return t.numpy()


def layer_to_numpy(L: Dict[str, Optional[torch.Tensor]], experts=None) -> Dict[str, object]:
    """Copy a layer to host numpy arrays.

    experts=None copies every routed expert. Otherwise only the listed expert ids are
    copied and the routed weights become {expert_id: array} dicts, so that a 3 GB
    layer never has to be copied whole.
    """
    out: Dict[str, object] = {}
    for name in ("router_w", "router_bias", "shared_gate_w", "sh_gate", "sh_up", "sh_down",
                 "sh_s_gate", "sh_s_up", "sh_s_down"):
        out[name] = to_numpy(L.get(name))
    for name in ("w_gate", "w_up", "w_down", "s_gate", "s_up", "s_down"):
        t = L.get(name)
        if t is None:
            out[name] = None
        elif experts is None:
            out[name] = to_numpy(t)
        else:
            out[name] = {int(e): to_numpy(t[int(e)]) for e in sorted(set(int(v) for v in experts))}
    return out
