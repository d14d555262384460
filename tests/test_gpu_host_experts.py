"""Routed experts in pinned host memory, served through the bounded device cache
(redmoe_forward_host_experts): every call matches the fp64 oracle, and the cache's
directory follows its policy exactly (checked against a plain Python model of it, fed
with the routing the GPU chose): hotness +1 per routed token, halved every 16 tokens,
misses in expert order, victims free-first then by (hotness, slot) among experts the call
does not use. Prefetch fills without counting a use."""

from collections import Counter

import numpy as np
import pytest
import torch

import moe_inputs as mi
import sparse_moe_gemv_b200 as smg
from parity import assert_layer_parity, tolerances

pytestmark = pytest.mark.gpu

ZIPF = mi.LayerShape(H=2048, E=512, k=10, I=512, Is=512, zipf_s=1.1)
ZIPF_INT4 = mi.LayerShape(H=2048, E=512, k=10, I=512, Is=512, zipf_s=1.1, expert_dtype="int4g32")
ROUTED = ("w_gate", "w_up", "w_down", "s_gate", "s_up", "s_down")


class CacheModel:
    def __init__(self, E, S):
        self.E, self.S = E, S
        self.slot_of = [-1] * E
        self.expert_in = [-1] * S
        self.hot = np.zeros(E, np.float32)
        self.tokens = self.hits = self.misses = self.prefetched = 0

    def call(self, ids, count_use=True, T=1):
        uses = Counter(int(e) for e in ids)
        if count_use:
            halve = self.tokens // 16 != (self.tokens + T) // 16
            for e in range(self.E):
                h = np.float32(self.hot[e] + np.float32(uses.get(e, 0)))
                self.hot[e] = np.float32(h * np.float32(0.5)) if halve else h
        miss = sorted(e for e in uses if self.slot_of[e] < 0)
        hits = sum(1 for e in uses if self.slot_of[e] >= 0)
        for e in miss:
            best = None
            for s in range(self.S):
                r = self.expert_in[s]
                if r < 0:
                    key = (0, 0.0, s)
                elif uses.get(r, 0) > 0:
                    continue
                else:
                    key = (1, float(self.hot[r]), s)
                best = key if best is None or key < best else best
            s = best[2]
            if self.expert_in[s] >= 0:
                self.slot_of[self.expert_in[s]] = -1
            self.expert_in[s] = e
            self.slot_of[e] = s
            uses[e] = max(uses.get(e, 0), 1)
        if count_use:
            self.tokens += T
            self.hits += hits
            self.misses += len(miss)
        else:
            self.prefetched += len(miss)


def _host_layer(shape, seed):
    L = mi.make_layer(shape, seed, "cuda")
    Lh = dict(L)
    for name in ROUTED:
        if L.get(name) is not None:
            Lh[name] = L[name].cpu().pin_memory()
    return L, Lh


def _check_directory(cache, model, label):
    t = cache.tensors
    assert t["slot_of"].cpu().tolist() == model.slot_of, f"{label}: slot_of"
    assert t["expert_in"].cpu().tolist() == model.expert_in, f"{label}: expert_in"
    np.testing.assert_array_equal(t["hot"].cpu().numpy(), model.hot, err_msg=f"{label}: hotness")
    assert t["stats"].cpu().tolist() == [model.tokens, model.hits, model.misses, model.prefetched], label


@pytest.mark.parametrize("shape,n_slots,calls", [(ZIPF_INT4, 24, 40), (ZIPF, 16, 12)])
def test_host_experts_match_oracle_and_follow_the_policy(gpu_lib, shape, n_slots, calls):
    L, Lh = _host_layer(shape, 8100)
    lay_h = smg.Layer.from_shape(Lh, shape)
    cache = smg.ExpertCache(lay_h, n_slots)
    smg.redmoe_expert_cache_init(lay_h, cache)
    ws = smg.new_workspace(lay_h, 1)
    model = CacheModel(shape.E, n_slots)
    ot, wt = tolerances(shape)
    for c in range(calls):
        x = mi.make_x(shape, 1, 8200 + c, "cuda")
        out = torch.full((1, shape.H), float("nan"), device="cuda")
        ids = torch.full((1, shape.k), -1, dtype=torch.int32, device="cuda")
        w = torch.full((1, shape.k), float("nan"), device="cuda")
        smg.redmoe_forward_host_experts(lay_h, x, out, ids, w, cache, ws)
        smg.redmoe_check_timeout(ws)
        model.call(ids.view(-1).cpu().tolist())
        _check_directory(cache, model, f"call {c}")
        if c % 4 == 0 or c == calls - 1:
            assert_layer_parity(shape, L, x, out, ids, w, ot, wt, f"host experts call {c}")
    # the Zipf offsets make a few experts hot: later calls find some of them resident
    assert model.hits > 0 and model.misses > 0


def test_prefetch_fills_without_a_use_and_the_next_call_hits(gpu_lib):
    shape = ZIPF_INT4
    L, Lh = _host_layer(shape, 8300)
    lay_h = smg.Layer.from_shape(Lh, shape)
    lay_d = smg.Layer.from_shape(L, shape)
    cache = smg.ExpertCache(lay_h, 16)
    smg.redmoe_expert_cache_init(lay_h, cache)
    ws = smg.new_workspace(lay_h, 1)
    x = mi.make_x(shape, 1, 8301, "cuda")
    # the router of the layer picks the experts to prefetch (router-driven prefetch)
    pid = torch.empty(1, shape.k, dtype=torch.int32, device="cuda")
    pw = torch.empty(1, shape.k, device="cuda")
    sg = torch.empty(1, device="cuda")
    smg.redmoe_router(lay_d, x, pid, pw, sg, smg.new_workspace(lay_d, 1))
    smg.redmoe_expert_cache_prefetch(lay_h, cache, pid.view(-1), ws)
    model = CacheModel(shape.E, 16)
    model.call(pid.view(-1).cpu().tolist(), count_use=False)
    _check_directory(cache, model, "after prefetch")
    out = torch.empty(1, shape.H, device="cuda")
    ids = torch.empty(1, shape.k, dtype=torch.int32, device="cuda")
    w = torch.empty(1, shape.k, device="cuda")
    smg.redmoe_forward_host_experts(lay_h, x, out, ids, w, cache, ws)
    smg.redmoe_check_timeout(ws)
    model.call(ids.view(-1).cpu().tolist())
    _check_directory(cache, model, "after the call")
    assert model.misses == 0 and model.hits == shape.k
    ot, wt = tolerances(shape)
    assert_layer_parity(shape, L, x, out, ids, w, ot, wt, "after prefetch")


def test_unreadable_home_memory_and_small_caches_are_refused(gpu_lib):
    shape = mi.LayerShape(H=2048, E=512, k=10, I=512, Is=512, expert_dtype="int2g32")
    L = mi.make_layer(shape, 8400, "cuda")
    Lp = dict(L)
    Lp["w_gate"] = L["w_gate"].cpu()  # pageable host memory: the GPU cannot read it
    lay = smg.Layer.from_shape(Lp, shape)
    cache = smg.ExpertCache(lay, 16)
    smg.redmoe_expert_cache_init(lay, cache)
    ws = smg.new_workspace(lay, 1)
    x = mi.make_x(shape, 1, 8401, "cuda")
    out = torch.empty(1, shape.H, device="cuda")
    ids = torch.empty(1, shape.k, dtype=torch.int32, device="cuda")
    w = torch.empty(1, shape.k, device="cuda")
    with pytest.raises(smg.RedmoeError) as e:
        smg.redmoe_forward_host_experts(lay, x, out, ids, w, cache, ws)
    assert e.value.status == 1
    small = smg.ExpertCache(smg.Layer.from_shape(L, shape), 4)  # fewer slots than top-k
    with pytest.raises(smg.RedmoeError) as e:
        smg.redmoe_forward_host_experts(smg.Layer.from_shape(L, shape), x, out, ids, w, small, ws)
    assert e.value.status == 1
