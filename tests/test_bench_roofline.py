"""The roofline numerators bench.py reports, checked on CPU against figures derived by hand
from the layer shape (hidden 2048, 512 experts, top-10, expert and shared intermediate
512): algorithmic bytes per decode layer call, int4 group-32 expert bytes, and the FLOPs
of a 2048-token chunk. Also the workload table's invariants and the rule that a stored
DRAM-traffic figure is used only while the kernel sources it was taken on are unchanged."""

import importlib.util
import json
import os

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench", os.path.join(ROOT, "bench.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def test_bf16_expert_and_decode_layer_bytes(bench):
    # one expert: gate, up [512, 2048] and down [2048, 512] in bf16
    assert bench.expert_bytes(bench.QWEN) == 3 * 512 * 2048 * 2 == 6_291_456
    weights = 512 * 2048 * 2 + 2048 * 2 + (10 + 1) * 6_291_456  # router, shared gate, 10 routed + shared
    assert weights == 71_307_264
    io = 2048 * 2 + 2048 * 4 + 10 * (4 + 4)  # x in, out fp32, ids int32 + weights fp32
    assert bench.layer_call_bytes(bench.QWEN, 1, 10) == weights + io == 71_319_632


def test_int4_expert_and_layer_bytes(bench):
    codes = 3 * 512 * 2048 // 2  # two 4-bit codes per byte
    scales = 3 * 512 * 2048 // 32 * 2  # one bf16 scale per 32 elements
    assert (codes, scales) == (1_572_864, 196_608)
    assert bench.expert_bytes(bench.QWEN_INT4) == codes + scales == 1_769_472
    weights = 512 * 2048 * 2 + 2048 * 2 + 11 * 1_769_472  # router and shared gate stay bf16
    assert weights == 21_565_440
    assert bench.layer_call_bytes(bench.QWEN_INT4, 1, 10) == weights + 2048 * 2 + 2048 * 4 + 80


def test_few_row_bytes_grow_with_distinct_experts_only(bench):
    b10 = bench.layer_call_bytes(bench.QWEN, 2, 10)
    b19 = bench.layer_call_bytes(bench.QWEN, 2, 19)
    assert b19 - b10 == 9 * 6_291_456


def test_prefill_chunk_flops(bench):
    T = 2048
    router = 2 * T * 512 * 2048
    routed = 2 * T * 10 * 3 * 2048 * 512
    shared = 2 * T * 3 * 2048 * 512
    assert (router, routed, shared) == (4_294_967_296, 128_849_018_880, 12_884_901_888)
    assert bench.layer_flops(bench.QWEN_ZIPF, T) == router + routed + shared
    assert abs(bench.layer_flops(bench.QWEN_ZIPF, T) / 1e9 - 146.03) < 0.01


def test_workload_table(bench):
    for name, wl in bench.WORKLOADS.items():
        s = wl["shape"]
        assert (s.H, s.E, s.k, s.I, s.Is) == (2048, 512, 10, 512, 512), name
        assert wl["T"] >= 1 and wl["layers"] >= 1, name
        # T > 4 takes the batched (tensor-core) path; its bench reports the tensor roofline
        assert (wl["T"] > 4) == name.startswith("prefill"), name
    assert bench.WORKLOADS["prefill"]["shape"].zipf_s == 1.1
    assert bench.WORKLOADS["prefill_uniform"]["shape"].zipf_s is None
    assert bench.WORKLOADS["int4_48"]["shape"].expert_dtype == "int4g32"
    assert bench.WORKLOADS["int4_48"]["layers"] == 48 and bench.WORKLOADS["int4_48"]["stack"]


def test_traffic_figure_needs_matching_sources(bench, tmp_path, monkeypatch):
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        committed = json.load(f)
    # a committed figure is reported exactly when it names the current sources
    for wl, d in committed.items():
        files = bench.PREFILL_SOURCES if wl.startswith("prefill") else bench.DECODE_SOURCES
        current = d["source_digest"] == bench.source_digest(files)
        if "dram_bytes_per_layer" in d:
            # a stack's figure is per layer, scaled by the layers of one launch
            want = d["dram_bytes_per_layer"] * bench.WORKLOADS[wl]["layers"]
            got = bench.profile_traffic(wl, bench.WORKLOADS[wl]["layers"])
        else:
            want, got = d["dram_bytes_per_launch"], bench.profile_traffic(wl)
        assert got == (want if current else None), wl
    # a workload without a capture reports none
    assert bench.profile_traffic("prefill_uniform") is None
    # a figure taken on other sources is not reported
    stale = {k: dict(v, source_digest="0" * 16) for k, v in committed.items()}
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(stale))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "source_digest", lambda files: "f" * 16)
    for wl in committed:
        assert bench.profile_traffic(wl) is None, wl
