"""MoE-layer benchmark on B200 (one process per GPU).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl redmoe|reference]

Workloads (synthetic seeded layers of the Qwen3-Next-80B-A3B MoE shape: hidden 2048,
512 experts, top-10, expert and shared intermediate 512):

  decode_t1   (default) one token through one bf16 layer per step; the steps rotate over
              12 distinct layers (38.7 GB), so no step finds its weights in L2
  fewrow_t2 / fewrow_t3   a 12-layer bf16 stack of independent layers, 2 or 3 tokens
  int4_48     a 48-layer int4 group-32 stack, one token
  int2_48     a 48-layer int2 group-32 stack (this library's lower-bit format), one token
  prefill     a 2048-token chunk through one bf16 layer with Zipf(1.1) router offsets

One JSON line on rank 0: the device-timed throughput (CUDA events on the launching
stream, the timed steps replayed from CUDA graphs, barrier + synchronize around the
timed region, max over ranks), the roofline of the dominant kernel, the end-to-end
figure through the C ABI with pinned host buffers, the fp64 oracle on the host cores,
and the SM clocks seen during the timed region. A step of a stack workload is one token
(T rows) through the whole stack, so its tokens/s are model-depth tokens. The default
run (decode_t1) adds one object per other workload (fewrow_t2, fewrow_t3, int4_48,
int2_48, prefill, prefill_uniform), each with its own roofline, end-to-end figure and clocks.
The path does not shard (one layer fits one GPU): with N > 1 every rank runs its own
replica ("replicas only"), the value is the sum over ranks.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import moe_inputs as mi  # noqa: E402

METRIC = "MoE-layer tokens/s at 1 B200; decode HBM GB/s (% of peak); prefill TFLOP/s"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
QWEN = mi.LayerShape(H=2048, E=512, k=10, I=512, Is=512)
QWEN_INT4 = mi.LayerShape(H=2048, E=512, k=10, I=512, Is=512, expert_dtype="int4g32")
QWEN_INT2 = mi.LayerShape(H=2048, E=512, k=10, I=512, Is=512, expert_dtype="int2g32")
QWEN_ZIPF = mi.LayerShape(H=2048, E=512, k=10, I=512, Is=512, zipf_s=1.1)

WORKLOADS = {
    "decode_t1": dict(shape=QWEN, T=1, layers=12, stack=False, seed=1000, kernel="decode1_kernel",
                      desc="Qwen3-Next-shaped MoE layer, bf16 weights / fp32 accumulate, decode T=1"),
    "fewrow_t2": dict(shape=QWEN, T=2, layers=12, stack=True, seed=2000, kernel="decodefr_kernel",
                      desc="12 distinct Qwen3-Next-shaped bf16 layers back to back, T=2"),
    "fewrow_t3": dict(shape=QWEN, T=3, layers=12, stack=True, seed=2000, kernel="decodefr_kernel + decode1_kernel",
                      desc="12 distinct Qwen3-Next-shaped bf16 layers back to back, T=3"),
    "int4_48": dict(shape=QWEN_INT4, T=1, layers=48, stack=True, seed=4000, kernel="decode1_kernel",
                    desc="48 distinct Qwen3-Next-shaped layers, int4 group-32 experts, decode T=1"),
    "int2_48": dict(shape=QWEN_INT2, T=1, layers=48, stack=True, seed=5000, kernel="decode1_kernel",
                    desc="48 distinct Qwen3-Next-shaped layers, int2 group-32 experts, decode T=1"),
    "prefill": dict(shape=QWEN_ZIPF, T=2048, layers=1, stack=False, seed=3000, kernel="layer (4 kernels)",
                    desc="Qwen3-Next-shaped MoE layer, bf16, 2048-token prefill chunk, Zipf(1.1) router offsets"),
    # one token per step through one bf16 layer whose routed experts stay in pinned host
    # memory behind a 64-slot device cache (Zipf(1.1) router offsets make some experts hot)
    "hostexp": dict(shape=QWEN_ZIPF, T=1, layers=1, stack=False, seed=6000, kernel="host experts (4 kernels)",
                    desc="Qwen3-Next-shaped MoE layer, bf16, decode T=1, routed experts in pinned host memory "
                         "behind a 64-slot device cache, Zipf(1.1) router offsets", slots=64, tokens=100),
    # the same chunk with unbiased routing: every expert is touched, so the step streams all
    # 512 experts' weights and the HBM floor moves above the tensor-core one
    "prefill_uniform": dict(shape=QWEN, T=2048, layers=1, stack=False, seed=3000, kernel="layer (4 kernels)",
                            desc="Qwen3-Next-shaped MoE layer, bf16, 2048-token prefill chunk, unbiased router"),
}


def layer_flops(shape, T):
    """Algorithmic FLOPs of one layer call: router 2*T*E*H, routed experts 2*T*k*3*H*I,
    shared expert 2*T*3*H*Is (multiply-adds counted as two)."""
    return 2.0 * T * (shape.E * shape.H + shape.k * 3 * shape.H * shape.I + 3 * shape.H * shape.Is)


# ------------------------------------------------------------------ helpers
def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", 0)), "measured"
    return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, 1400.0, "fallback"


def _matrix_bytes(dtype, H, I):
    """Bytes of one expert's three H x I matrices (packed types: codes + bf16 group scales)."""
    if dtype == "int4g32":
        return 3 * (H * I // 2 + H * I // 32 * 2)
    if dtype == "int2g32":
        return 3 * (H * I // 4 + H * I // 32 * 2)
    return 3 * H * I * (4 if dtype == "f32" else 2)


def expert_bytes(shape):
    """Bytes of one routed expert's three matrices."""
    return _matrix_bytes(shape.expert_dtype, shape.H, shape.I)


def shared_bytes(shape):
    return _matrix_bytes(shape.expert_dtype, shape.H, shape.Is)


def layer_call_bytes(shape, T, distinct):
    """Algorithmic HBM bytes of one layer call: every weight the math needs read once
    (router, shared gate, the distinct routed experts, the shared expert), x read once,
    out / ids / weights written once."""
    rb = 4 if shape.router_dtype == "f32" else 2
    xb = 4 if shape.x_dtype == "f32" else 2
    return (shape.E * shape.H * rb + shape.H * rb + distinct * expert_bytes(shape) + shared_bytes(shape)
            + T * shape.H * xb + T * shape.H * 4 + T * shape.k * 8)


# kernel sources behind each path: a committed DRAM-traffic figure stays valid while these
# files are unchanged
DECODE_SOURCES = ["common.cuh", "decode.cu", "decode1.cu", "decode_fr.cu", "gemv.cuh", "internal.h", "rowdot.cuh",
                  "topk.cuh"]
PREFILL_SOURCES = ["common.cuh", "ggemm.cu", "ggemm_params.h", "internal.h", "prefill.cu", "route.cu", "tc.cuh", "topk.cuh"]


def source_digest(files):
    h = hashlib.sha256()
    for f in sorted(files):
        h.update(f.encode())
        h.update(open(os.path.join(ROOT, "sparse_moe_gemv_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


def profile_traffic(workload, layers_per_launch=1):
    """DRAM bytes per launch (per step for the batched layer) from the committed ncu summary,
    if it was taken on the current kernel sources. A layer stack's figure is stored per layer
    (captured on a shorter stack of the same layers) and scaled by the layers of one launch."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p)).get(workload)
    files = PREFILL_SOURCES if workload.startswith("prefill") else DECODE_SOURCES
    if not d or d.get("source_digest") != source_digest(files):
        return None
    if "dram_bytes_per_layer" in d:
        return d["dram_bytes_per_layer"] * layers_per_launch
    return d.get("dram_bytes_per_launch")


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while the timed region runs."""

    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4, "hw_slowdown": 0x8,
        "sync_boost": 0x10, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
        "hw_power_brake_slowdown": 0x80, "display_clock_setting": 0x100,
    }

    def __init__(self, device_index):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:  # NVML missing: report no clocks rather than fail the run
            self.nv = None

    def _run(self):
        while not self._stop.is_set():
            self._sample()
            time.sleep(0.005)

    def _sample(self):
        try:
            self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
            r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
            for name, bit in self.REASONS.items():
                if r & bit and name != "gpu_idle":
                    self.reasons.add(name)
        except Exception:
            pass

    def __enter__(self):
        if self.nv is not None:
            self._sample()
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *a):
        if self._thread is not None:
            self._stop.set()
            self._thread.join()
            self._sample()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ---------------------------------------------------------------- distributed
def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(local)
    return world, rank, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def _reduce(v, world, op):
    if world == 1:
        return v
    # NCCL reduces device tensors; gloo (the CPU tests of this logic) host tensors
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=op)
    return float(t.item())


def max_over_ranks(v, world):
    return _reduce(v, world, torch.distributed.ReduceOp.MAX)


def sum_over_ranks(v, world):
    return _reduce(v, world, torch.distributed.ReduceOp.SUM)


def job_throughput(units, seconds, world):
    """Whole-job rate: the units every rank processed over the slowest rank's time."""
    return sum_over_ranks(units, world) / max_over_ranks(seconds, world)


# ------------------------------------------------------------- CPU baseline
def _used_experts(lay, shape, x):
    """Experts the oracle's own routing of x selects (so that only those are fetched)."""
    import oracle
    r = oracle.router(lay, shape, x)
    return sorted(set(r["ids"].reshape(-1).tolist()))


def _host_layer(L, shape, x):
    import oracle  # noqa: F401
    lay = mi.layer_to_numpy(L, experts=[])
    return mi.layer_to_numpy(L, experts=_used_experts(lay, shape, x))


def _time_oracle(fn, threads):
    import oracle
    oracle.set_num_threads(threads)
    fn()  # warm-up call (page-in, thread start)
    t0 = time.perf_counter()
    fn()
    return time.perf_counter() - t0


def cpu_oracle_sample(wl, seconds=10.0):
    """The fp64 oracle on the host cores over a bounded sample of the workload: decode
    tokens through layer 0 of the workload (one oracle call, OpenMP over tokens)."""
    import oracle
    shape = wl["shape"]
    cores = oracle.num_threads()
    L = mi.make_layer(shape, wl["seed"], "cuda")
    x1 = mi.to_numpy(mi.make_x(shape, 1, wl["seed"] + 99, "cpu"))
    lay = mi.layer_to_numpy(L)
    del L
    t1 = _time_oracle(lambda: oracle.forward(lay, shape, x1), cores)
    n = int(max(cores, min(4096, seconds * cores / max(t1, 1e-3))))
    n = max(cores, (n // cores) * cores)
    x = mi.to_numpy(mi.make_x(shape, n, wl["seed"] + 123, "cpu"))
    t0 = time.perf_counter()
    oracle.forward(lay, shape, x)
    el = time.perf_counter() - t0
    # one thread on one decode token (the single-thread time of a T = 1 layer call)
    t_single = _time_oracle(lambda: oracle.forward(lay, shape, x1), 1)
    oracle.set_num_threads(cores)
    return {"value": n / el, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "omp_num_threads": cores, "omp_env": os.environ.get("OMP_NUM_THREADS"), "nproc": os.cpu_count(),
            "sample": f"{n} decode tokens through one {wl['desc']} layer, one oracle call "
                      f"(fp64, OpenMP over tokens), {el:.1f} s wall",
            "single_thread": {"value": 1.0 / t_single, "unit": "tokens/s", "seconds_per_call": t_single,
                              "sample": "one T=1 call of the same layer on one thread"}}


def cpu_oracle_stack(wl, B, T=2):
    """The oracle over the 12-layer few-row stack at T tokens (one step = T tokens through
    all layers), every thread of the host; experts fetched as the oracle routes them."""
    import oracle
    shape = wl["shape"]
    cores = oracle.num_threads()
    hl = []
    for l in range(len(B["tens"])):
        x = mi.to_numpy(B["xs"][l][:T])
        hl.append((_host_layer(B["tens"][l], shape, x), x))
    el = _time_oracle(lambda: [oracle.forward(lay, shape, x) for lay, x in hl], cores)
    return {"value": T / el, "unit": "tokens/s", "cores": min(cores, T), "threads": cores,
            "seconds_per_step": el,
            "sample": f"one step: T={T} tokens through {len(hl)} distinct layers, fp64 oracle "
                      f"(threads beyond T idle: OpenMP over a call's tokens)"}


def cpu_oracle_prefill(wl, B, n=256):
    """The oracle on the first n tokens of the prefill chunk (a bounded sample)."""
    import oracle
    shape = wl["shape"]
    cores = oracle.num_threads()
    x = mi.to_numpy(B["xs"][0][:n])
    lay = _host_layer(B["tens"][0], shape, x)
    el = _time_oracle(lambda: oracle.forward(lay, shape, x), cores)
    return {"value": n / el, "unit": "tokens/s", "cores": cores, "seconds": el,
            "sample": f"the first {n} of the {wl['T']} tokens of the chunk, one oracle call "
                      f"({len(lay['w_gate'])} experts fetched), fp64, OpenMP over tokens"}


def workload_config(wl, world):
    """The `config` object both arms report for a workload."""
    return {"workload": wl["desc"], "tokens_per_step": wl["T"], "layers": wl["layers"],
            "layers_per_step": wl["layers"] if wl["stack"] else 1,
            "l2": "inputs larger than L2: each step reads a different layer's weights "
                  f"({wl['layers']} distinct layers)" if not wl["stack"] else
                  f"inputs larger than L2: {wl['layers']} distinct layers per step",
            "parallelism": "replicas" if world > 1 else "single GPU"}


def reference_arm(args, wl, world, rank):
    """The fp64 oracle as the reference implementation, timed on the host cores."""
    import oracle
    if rank != 0:
        return None
    shape = wl["shape"]
    T = wl["T"]
    threads = oracle.num_threads()
    cores = min(threads, T)  # the oracle splits a call over its tokens: threads beyond T idle
    nl = min(wl["layers"], 2)
    layers = []
    for l in range(nl):
        L = mi.make_layer(shape, wl["seed"] + l, "cuda")
        layers.append(mi.layer_to_numpy(L))
        del L
    torch.cuda.empty_cache()
    xs = [mi.to_numpy(mi.make_x(shape, T, wl["seed"] + 7 * s, "cpu")) for s in range(4)]
    tokens_per_step = T  # a stack step is T tokens through every layer

    def step(s):
        for l in range(wl["layers"] if wl["stack"] else 1):
            oracle.forward(layers[(s + l) % nl], shape, xs[s % 4])

    tw = time.perf_counter()
    for s in range(args.warmup):  # warm-up, bounded in time like the timed loop
        step(s)
        if time.perf_counter() - tw > 30.0:
            break
    budget = 120.0
    t0 = time.perf_counter()
    done = 0
    for s in range(args.steps):
        step(s)
        done += 1
        if time.perf_counter() - t0 > budget:
            break
    el = time.perf_counter() - t0
    value = done * tokens_per_step / el
    unit = "tokens/s"
    sample = (f"{done} of {args.steps} steps (time-bounded at {budget:.0f} s), each "
              f"{'a ' + str(wl['layers']) + '-layer stack' if wl['stack'] else 'one layer'} at T={T}, "
              f"fp64 oracle, {cores} of {threads} threads busy (OpenMP over the call's tokens)")
    return {"metric": METRIC, "value": value, "unit": unit, "n_gpus": 1, "steps": done, "warmup": args.warmup,
            "ms_per_step": 1e3 * el / max(done, 1), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {**workload_config(wl, world),
                       "timing": "host wall clock around the timed steps (rank 0 alone runs this arm)"},
            "impl": "reference",
            "cpu_baseline": {"value": value, "unit": unit, "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


# ------------------------------------------------------------------ GPU arm
def build_workload(wl, smg, tens=None):
    """Device layers (or the given ones), inputs, outputs and a workspace for the workload."""
    shape, T, nl = wl["shape"], wl["T"], wl["layers"]
    if tens is None:
        tens = [mi.make_layer(shape, wl["seed"] + l, "cuda") for l in range(nl)]
    lays = [smg.Layer.from_shape(t, shape) for t in tens]
    xs = [mi.make_x(shape, T, wl["seed"] + l, "cuda") for l in range(nl)]
    outs = [torch.empty(T, shape.H, device="cuda") for _ in range(nl)]
    ids = [torch.empty(T, shape.k, dtype=torch.int32, device="cuda") for _ in range(nl)]
    ws_ = [torch.empty(T, shape.k, device="cuda") for _ in range(nl)]
    work = smg.new_workspace(lays[0], T)
    return dict(tens=tens, lays=lays, xs=xs, outs=outs, ids=ids, ws=ws_, work=work)


def make_step(wl, smg, B, stream):
    """step(i): the i-th step's launches on `stream`."""
    nl = wl["layers"]
    shape = wl["shape"]
    # three and four rows run as rows 0-1 on the few-row kernel plus the rest: two launches
    split = 2 if wl["T"] in (3, 4) and shape.x_dtype == "bf16" and shape.expert_dtype in ("bf16", "int4g32") else 1
    if wl["stack"]:
        def step(i):
            smg.redmoe_forward_stack(B["lays"], B["xs"], B["outs"], B["ids"], B["ws"], B["work"], stream=stream)
        return step, split * (1 if nl <= 64 else math.ceil(nl / 64))

    def step(i):
        l = i % nl
        smg.redmoe_forward(B["lays"][l], B["xs"][l], B["outs"][l], B["ids"][l], B["ws"][l], B["work"], stream=stream)
    return step, split


def capture(step, n, stream):
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(n):
            step(i)
    return g


class GraphRunner:
    """Replays n consecutive steps (step 0 .. n-1) as whole CUDA graphs of up to CHUNK steps
    each, so that no eager host call sits between timed launches and a timed region of up
    to CHUNK steps is a single graph launch."""

    CHUNK = 4096

    def __init__(self, step, stream):
        self.step, self.stream = step, stream
        self.graphs = {}

    def _capture(self, start, n):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=self.stream):
            for i in range(start, start + n):
                self.step(i)
        return g

    def prepare(self, n):
        if n not in self.graphs:
            self.graphs[n] = [self._capture(s, min(self.CHUNK, n - s)) for s in range(0, n, self.CHUNK)]

    def run(self, n):
        for g in self.graphs[n]:
            g.replay()


def distinct_experts(B):
    """Distinct routed experts of each layer's last call, from the ids it returned."""
    return [len(set(ids.view(-1).tolist())) for ids in B["ids"]]


def gpu_arm(args, wl, world, rank, local, B=None, name=None):
    import sparse_moe_gemv_b200 as smg
    smg.load()
    shape, T = wl["shape"], wl["T"]
    if B is None:
        B = build_workload(wl, smg)
    stream = torch.cuda.Stream()
    step, launches_per_step = make_step(wl, smg, B, stream)
    with torch.cuda.stream(stream):
        step(0)  # one eager call: per-device set-up (attributes, driver entry points) outside capture
    torch.cuda.synchronize()
    K, W = args.steps, args.warmup
    runner = GraphRunner(step, stream)
    runner.prepare(W)
    runner.prepare(K)
    torch.cuda.synchronize()

    with torch.cuda.stream(stream):
        runner.run(W)   # the W warm-up steps
        runner.run(K)   # one untimed replay of the timed graphs (their first launch uploads them)
    torch.cuda.synchronize()
    smg.redmoe_check_timeout(B["work"], stream=stream)

    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        with torch.cuda.stream(stream):
            ev0.record(stream)
            runner.run(K)
            ev1.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    smg.redmoe_check_timeout(B["work"], stream=stream)
    el_ms = ev0.elapsed_time(ev1)
    tokens_per_step = T  # one layer call, or T tokens through the whole stack
    value = job_throughput(K * tokens_per_step, el_ms / 1e3, world)  # this rank's time in
    el_ms = max_over_ranks(el_ms, world)

    distinct = distinct_experts(B)
    # algorithmic bytes of one step: the whole stack, or one layer call (averaged over the
    # rotation's layers)
    if wl["stack"]:
        bytes_per_step = sum(layer_call_bytes(shape, T, d) for d in distinct)
    else:
        bytes_per_step = sum(layer_call_bytes(shape, T, d) for d in distinct) / len(distinct)
    launches = K * launches_per_step
    step_s = el_ms / 1e3 / K
    hbm, bf16, bf16_sus, src = peaks()
    achieved = bytes_per_step / step_s / 1e9
    key = name or args.workload
    if T > 4:
        # batched path: four kernels per step. Its roofline is the binding one of two: the
        # step's algorithmic bytes (every touched expert's weights once, x, out) at the HBM
        # peak, and its FLOPs at the bf16 tensor peak. With a few tokens per expert the
        # weights dominate and the HBM time is the larger.
        flops = layer_flops(shape, T)
        tfl = flops / step_s / 1e12
        gbs = bytes_per_step / step_s / 1e9
        t_hbm, t_tc = bytes_per_step / (hbm * 1e9), flops / (bf16 * 1e12)
        both = {"traffic": profile_traffic(key), "kernel": wl["kernel"], "flops_per_step": flops,
                "bytes_per_step": bytes_per_step, "hbm_floor_us": t_hbm * 1e6, "tensor_floor_us": t_tc * 1e6,
                "tensor_tflops": tfl, "tensor_frac": tfl / bf16, "hbm_gbs": gbs, "hbm_frac": gbs / hbm}
        if t_hbm >= t_tc:
            roof = {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm, **both,
                    "peak_source": f"{src} (MEASURED_PEAKS.json hbm_gbs)" if src == "measured" else "fallback"}
        else:
            roof = {"bound": "tensor", "achieved": tfl, "peak": bf16, "unit": "TFLOP/s", "frac": tfl / bf16, **both,
                    "peak_source": f"{src} (MEASURED_PEAKS.json bf16_tflops, burst)"}
        launches = K * 4
    else:
        roof = {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
                "traffic": profile_traffic(key, wl["layers"] if wl["stack"] else 1), "kernel": wl["kernel"],
                "bytes_per_step": bytes_per_step, "step_us": step_s * 1e6,
                "launches_per_step": launches_per_step, "distinct_experts_per_layer": statistics.mean(distinct),
                "peak_source": f"{src} (MEASURED_PEAKS.json hbm_gbs)" if src == "measured" else "fallback"}

    # end to end through the C ABI with pinned host buffers: per step H2D x, forward, D2H out/ids/w
    e2e = e2e_arm(args, wl, smg, B, stream, world)
    result = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K, "warmup": W,
        "ms_per_step": el_ms / K, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": shape.expert_dtype,
        "data": "synthetic",
        "config": {**workload_config(wl, world),
                   "timing": "CUDA graph replay of exactly the timed steps (one graph up to 4096 steps); "
                             "untimed before it: the warm-up steps and one replay of the timed graph"},
        "roofline": roof,
        "e2e": e2e,
        "gpu_launches": launches,
        "clocks": clk.summary(),
    }
    return result, B


def e2e_arm(args, wl, smg, B, stream, world):
    shape, T = wl["shape"], wl["T"]
    nl = wl["layers"]
    K = args.steps
    xb = 4 if shape.x_dtype == "f32" else 2
    hx = [B["xs"][l].cpu().pin_memory() for l in range(nl)]
    hout = torch.empty(T, shape.H, dtype=torch.float32).pin_memory()
    hids = torch.empty(T, shape.k, dtype=torch.int32).pin_memory()
    hw = torch.empty(T, shape.k, dtype=torch.float32).pin_memory()
    # the host-buffer entry points: x comes in over the link (read by the kernel at T = 1,
    # one copy otherwise) and the results land in the pinned host buffers
    wsh = smg.new_workspace_host(B["lays"][0], T)
    if wl["stack"]:
        houts = [torch.empty(T, shape.H, dtype=torch.float32).pin_memory() for _ in range(nl)]
        hidss = [torch.empty(T, shape.k, dtype=torch.int32).pin_memory() for _ in range(nl)]
        hws = [torch.empty(T, shape.k, dtype=torch.float32).pin_memory() for _ in range(nl)]

    def step(i):
        if wl["stack"]:
            smg.redmoe_forward_stack_host(B["lays"], hx, houts, hidss, hws, wsh, stream=stream)
        else:
            l = i % nl
            smg.redmoe_forward_host(B["lays"][l], hx[l], hout, hids, hw, wsh, stream=stream)

    n_e2e = K
    with torch.cuda.stream(stream):
        for i in range(min(args.warmup, 50)):
            step(i)
    torch.cuda.synchronize()
    barrier(world)
    t0 = time.perf_counter()
    with torch.cuda.stream(stream):
        for i in range(n_e2e):
            step(i)
    stream.synchronize()
    el = time.perf_counter() - t0
    per = (nl if wl["stack"] else 1)
    rate = job_throughput(n_e2e * T, el, world)  # this rank's wall time in; T tokens per step
    h2d = T * shape.H * xb * per
    d2h = (T * shape.H * 4 + T * shape.k * 8) * per
    return {"value": rate, "unit": "tokens/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "steps": n_e2e,
            "how": ("redmoe_forward_stack_host" if wl["stack"] else "redmoe_forward_host") +
                   " through the C ABI per step, every x and result in pinned host memory: x read over the link "
                   "by the kernel at T = 1 (copied in otherwise), results stored straight into the host buffers "
                   "at T <= 4 (copied back otherwise); host wall clock around the K steps"}


def host_link_gbs(nbytes=512 * 2**20, reps=5):
    """Host-to-device copy rate from pinned memory (the link the host-expert fills use)."""
    h = torch.empty(nbytes, dtype=torch.uint8).pin_memory()
    d = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    d.copy_(h, non_blocking=True)
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record()
    for _ in range(reps):
        d.copy_(h, non_blocking=True)
    ev1.record()
    torch.cuda.synchronize()
    return reps * nbytes / (ev0.elapsed_time(ev1) / 1e3) / 1e9


def hostexp_arm(args, wl, world, rank, local):
    """Decode tokens through a layer whose routed experts live in pinned host memory, served
    by redmoe_forward_host_experts through a bounded device cache. Reports tokens/s, the
    cache hit rate and the fill traffic against the measured host-to-device copy rate."""
    import sparse_moe_gemv_b200 as smg
    smg.load()
    shape, n = wl["shape"], wl["tokens"]
    L = mi.make_layer(shape, wl["seed"], "cuda")
    Lh = dict(L)
    for name in ("w_gate", "w_up", "w_down", "s_gate", "s_up", "s_down"):
        if L.get(name) is not None:
            Lh[name] = L[name].cpu().pin_memory()
            L[name] = None
    torch.cuda.empty_cache()
    lay = smg.Layer.from_shape(Lh, shape)
    cache = smg.ExpertCache(lay, wl["slots"])
    ws = smg.new_workspace(lay, 1)
    xs = [mi.make_x(shape, 1, wl["seed"] + 1 + i, "cuda") for i in range(n)]
    out = torch.empty(1, shape.H, device="cuda")
    ids = torch.empty(1, shape.k, dtype=torch.int32, device="cuda")
    w = torch.empty(1, shape.k, device="cuda")
    stream = torch.cuda.Stream()

    def step(i):
        smg.redmoe_forward_host_experts(lay, xs[i % n], out, ids, w, cache, ws, stream=stream)

    K, W = args.steps, args.warmup
    smg.redmoe_expert_cache_init(lay, cache, stream=stream)
    with torch.cuda.stream(stream):
        step(0)
    torch.cuda.synchronize()
    runner = GraphRunner(step, stream)
    try:
        runner.prepare(K)
        timing = "CUDA graph replay of the timed steps"
    except RuntimeError:  # capture refused: time eager launches instead
        torch.cuda.synchronize()
        runner = None
        timing = "eager launches (graph capture refused)"
    # warm-up: the first W tokens of the stream, then the cache starts empty again
    with torch.cuda.stream(stream):
        for i in range(W):
            step(i)
    torch.cuda.synchronize()
    smg.redmoe_expert_cache_init(lay, cache, stream=stream)
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        with torch.cuda.stream(stream):
            ev0.record(stream)
            if runner is not None:
                runner.run(K)
            else:
                for i in range(K):
                    step(i)
            ev1.record(stream)
        torch.cuda.synchronize()
    smg.redmoe_check_timeout(ws, stream=stream)
    el = ev0.elapsed_time(ev1) / 1e3
    st = cache.tensors["stats"].cpu().tolist()
    tokens, hits, misses = st[0], st[1], st[2]
    eb = expert_bytes(shape)
    link = host_link_gbs()
    fill_gbs = misses * eb / el / 1e9
    return {"workload": wl["desc"], "value": K / el, "unit": "tokens/s", "ms_per_step": el * 1e3 / K, "steps": K,
            "warmup": W, "dtype": shape.expert_dtype,
            "cache": {"slots": wl["slots"], "slot_bytes": smg.redmoe_expert_cache_slot_bytes(lay),
                      "tokens": tokens, "hits": hits, "misses": misses,
                      "hit_rate": hits / max(1, hits + misses), "starts": "empty"},
            "timing": timing,
            "roofline": {"bound": "host link", "achieved": fill_gbs, "peak": link, "unit": "GB/s",
                         "frac": fill_gbs / link, "traffic": None, "kernel": wl["kernel"],
                         "bytes_per_step": misses * eb / K,
                         "peak_source": "pinned host-to-device copy measured in this run"},
            "gpu_launches": 4 * K, "clocks": clk.summary()}


MIDBATCH_T = (1, 2, 3, 4, 5, 8, 16, 32, 64, 128, 256)


def midbatch_sweep(args, world, rank, local):
    """Per-call time of one bf16 layer at T = 1 .. 256 on a rotation of 12 distinct layers
    (inputs larger than L2): the decode kernels serve T <= 4, the batched tensor-core path
    T > 4. Reports, per T, the device time per call (CUDA events around a CUDA graph of the
    timed calls), the distinct experts touched, the algorithmic bytes and their rate."""
    import sparse_moe_gemv_b200 as smg
    smg.load()
    wl = dict(WORKLOADS["decode_t1"])
    shape, nl = wl["shape"], wl["layers"]
    tens = [mi.make_layer(shape, wl["seed"] + l, "cuda") for l in range(nl)]
    hbm, bf16, _, src = peaks()
    rows = []
    for T in MIDBATCH_T:
        twl = dict(wl, T=T)
        B = build_workload(twl, smg, tens=tens)
        stream = torch.cuda.Stream()
        step, _ = make_step(twl, smg, B, stream)
        with torch.cuda.stream(stream):
            step(0)
        torch.cuda.synchronize()
        reps = max(2, min(args.steps, 240) // nl)
        runner = GraphRunner(step, stream)
        runner.prepare(nl * reps)
        with torch.cuda.stream(stream):
            runner.run(nl * reps)  # warm-up, and the graph's upload
        torch.cuda.synchronize()
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            ev0.record(stream)
            runner.run(nl * reps)
            ev1.record(stream)
        torch.cuda.synchronize()
        smg.redmoe_check_timeout(B["work"], stream=stream)
        us = ev0.elapsed_time(ev1) * 1e3 / (nl * reps)
        distinct = distinct_experts(B)
        nbytes = statistics.mean(layer_call_bytes(shape, T, d) for d in distinct)
        rows.append({"T": T, "path": "decode" if T <= 4 else "batched", "us_per_call": us,
                     "tokens_per_s": T / us * 1e6, "distinct_experts": statistics.mean(distinct),
                     "bytes_per_call": nbytes, "gbs": nbytes / us / 1e3, "hbm_frac": nbytes / us / 1e3 / hbm,
                     "tflops": layer_flops(shape, T) / us / 1e6})
        B.clear()
        torch.cuda.synchronize()
    return {"metric": METRIC, "workload": "midbatch", "unit": "us per layer call",
            "config": {"workload": wl["desc"].replace("decode T=1", "T = 1..256"), "layers_in_rotation": nl,
                       "peak_source": src},
            "rows": rows}


SUB_WORKLOADS = ("fewrow_t2", "fewrow_t3", "int4_48", "int2_48", "prefill", "prefill_uniform", "hostexp")
SUB_STEPS = {"fewrow_t2": 200, "fewrow_t3": 200, "int4_48": 100, "int2_48": 100, "prefill": 50, "prefill_uniform": 30,
             "hostexp": 100}


def sub_result(res):
    if "cache" in res:  # hostexp reports its own object
        return res
    keep = ("value", "unit", "ms_per_step", "steps", "warmup", "dtype", "roofline", "e2e", "gpu_launches", "clocks")
    d = {k: res[k] for k in keep}
    d["workload"] = res["config"]["workload"]
    d["tokens_per_step"] = res["config"]["tokens_per_step"]
    return d


def free(B):
    if B is not None:
        B.clear()
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


def run_sub_workload(args, name):
    """One extra workload of the default line, in a child process with a CUDA context of its
    own, so that the workloads share no device state; returns (object, cpu-baseline extras)."""
    import subprocess
    steps = SUB_STEPS[name] if name == "hostexp" else min(args.steps, SUB_STEPS[name])  # hostexp: its whole stream
    cmd = [sys.executable, os.path.abspath(__file__), "--workload", name, "--steps", str(steps), "--warmup", "3", "--sub"]
    if not args.no_cpu_baseline:
        cmd.append("--sub-cpu")
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=900)
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    if r.returncode != 0 or not lines:
        tail = (r.stderr or r.stdout).strip().splitlines()[-1:] or ["no output"]
        return {"workload": WORKLOADS[name]["desc"], "error": f"exit {r.returncode}: {tail[0][:300]}"}, {}
    d = json.loads(lines[-1])
    return sub_result(d), d.get("cpu_extra", {})


def sub_cpu_extra(name, B):
    """The oracle timings that belong to a workload (rank 0, N = 1)."""
    if name == "fewrow_t2":
        return {"fewrow_t2_stack": cpu_oracle_stack(WORKLOADS[name], B, T=2)}
    if name == "prefill":
        return {"prefill_chunk": cpu_oracle_prefill(WORKLOADS[name], B)}
    return {}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=240)
    ap.add_argument("--workload", default="decode_t1", choices=sorted(WORKLOADS) + ["midbatch"])
    ap.add_argument("--impl", default="redmoe", choices=["redmoe", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="default run: skip the objects of the other workloads")
    ap.add_argument("--layers", type=int, default=None,
                    help="override the number of distinct layers (small cases for profiler captures)")
    ap.add_argument("--sub", action="store_true", help=argparse.SUPPRESS)      # child of the default line
    ap.add_argument("--sub-cpu", action="store_true", help=argparse.SUPPRESS)  # child also times its oracle leg
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    world, rank, local = dist_setup()
    if args.workload == "midbatch":
        res = midbatch_sweep(args, world, rank, local)
        if rank == 0:
            print(json.dumps(res), flush=True)
        if world > 1:
            torch.distributed.destroy_process_group()
        return
    wl = dict(WORKLOADS[args.workload])
    if args.layers:
        wl["layers"] = args.layers
    if args.impl == "reference":
        res = reference_arm(args, wl, world, rank)
        if rank == 0:
            print(json.dumps(res), flush=True)
        if world > 1:
            torch.distributed.destroy_process_group()
        return
    if args.workload == "hostexp":
        res = hostexp_arm(args, wl, world, rank, local)
        if rank == 0:
            print(json.dumps(res), flush=True)
        return
    if args.sub:
        res, B = gpu_arm(args, wl, world, rank, local, name=args.workload)
        if args.sub_cpu:
            res["cpu_extra"] = sub_cpu_extra(args.workload, B)
        print(json.dumps(res), flush=True)
        return
    cpu = world == 1 and rank == 0 and not args.no_cpu_baseline
    res, B = gpu_arm(args, wl, world, rank, local)
    free(B)
    extra_cpu = {}
    if args.workload == "decode_t1" and not args.no_extra and world == 1:
        # the other workloads, each in a process of its own (one GPU: at N > 1 the line
        # carries the headline workload only)
        for name in SUB_WORKLOADS:
            obj, cpu_extra = run_sub_workload(args, name)
            res[name] = obj
            extra_cpu.update(cpu_extra)
    if rank == 0:
        if cpu:
            res["cpu_baseline"] = cpu_oracle_sample(wl)
            res["cpu_baseline"].update(extra_cpu)
        print(json.dumps(res), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
