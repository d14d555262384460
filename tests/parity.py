"""Comparison of the CUDA path's results with the fp64 oracle (test helper).

Rules (per token row):

* top-k ids: compared exactly. A token whose oracle gap between the k-th and (k+1)-th
  largest logit is below GAP (1e-5) is exempt from the exact id comparison: its valid id
  sets are the experts surely above the boundary plus any choice from the near-tie band
  around it. The oracle enumerates those sets itself, each with its own renormalised
  weights and output; the GPU result must equal one of them (the matching set is picked by
  equality of id sets, so no GPU value ever enters the oracle).
* order within the top-k: by logit descending; adjacent positions whose oracle logits
  differ by less than GAP are compared as a set.
* weights: |w_gpu - w_oracle| <= w_tol for the same expert.
* outputs: max |out_gpu - out_oracle| <= out_tol * RMS(out_oracle), RMS over the layer's
  whole [T, H] output (1e-5 for fp32, 2e-2 for bf16 / int4).
"""

from __future__ import annotations

import itertools

import numpy as np
import torch

import moe_inputs as mi
import oracle

GAP = 1e-5


def host_routing_layer(L):
    """Router/shared tensors of a device layer as numpy (experts are fetched on demand)."""
    return mi.layer_to_numpy(L, experts=[])


def candidate_sets(logits_row, k):
    """All id sets a correct top-k may return given GAP (list of sorted tuples)."""
    order = np.lexsort((np.arange(logits_row.shape[0]), -logits_row))
    lk = logits_row[order[k - 1]]
    if k < logits_row.shape[0] and lk - logits_row[order[k]] >= GAP:
        return [tuple(sorted(order[:k].tolist()))], False
    sure = [int(e) for e in order if logits_row[e] > lk + GAP]
    band = [int(e) for e in order if abs(logits_row[e] - lk) <= GAP]
    need = k - len(sure)
    sets = [tuple(sorted(sure + list(c))) for c in itertools.combinations(band, need)]
    return sets, True


def check_order(logits_row, ids):
    """GPU order must be by logit descending, up to swaps inside GAP."""
    l = logits_row[np.asarray(ids)]
    return bool(np.all(np.diff(l) <= GAP))


def reference(shape, L, x_dev, gpu_ids=None, rows=None, cache=None):
    """Oracle routing + outputs for the device layer L and input x_dev.

    With gpu_ids given, exempt tokens take the oracle-enumerated set equal to the GPU's
    (if any); returns dict with ids/w (oracle order for that set), s, out, logits (the
    logits the selection ranks), exempt. cache = (cached mask [E], lambda) selects the
    opt-in cache-aware routing; its near-tie rule applies to the biased logits, and the
    weights of a matched set are renormalised from the unbiased ones.
    """
    x = mi.to_numpy(x_dev)
    lay = host_routing_layer(L)
    r = oracle.router(lay, shape, x)
    T = x.shape[0]
    ids = r["ids"].copy()
    w = r["w"].copy()
    sel_logits = r["logits"]
    if cache is not None:
        c = oracle.cache_route(r["logits"], np.asarray(cache[0], np.uint8), float(cache[1]), shape.k)
        ids, w, sel_logits = c["ids"].copy(), c["w"].copy(), c["biased"]
    exempt = np.zeros(T, bool)
    bad = []
    for t in range(T):
        sets, ex = candidate_sets(sel_logits[t], shape.k)
        exempt[t] = ex
        if not ex or gpu_ids is None:
            continue
        g = tuple(sorted(int(v) for v in gpu_ids[t]))
        if g not in sets:
            bad.append(t)
            continue
        # oracle order for the matched set: logit desc, id asc
        chosen = sorted(g, key=lambda e: (-sel_logits[t][e], e))
        ids[t] = chosen
        w[t] = oracle.renorm(r["logits"][t], np.array(chosen, np.int32))
    rows = np.arange(T) if rows is None else np.asarray(rows)
    used = sorted(set(ids[rows].reshape(-1).tolist()))
    lay_e = mi.layer_to_numpy(L, experts=used)
    out = oracle.experts(lay_e, shape, x[rows], ids[rows], w[rows], r["s"][rows])
    return dict(ids=ids, w=w, s=r["s"], out=out, logits=sel_logits, exempt=exempt, bad=bad, rows=rows)


def assert_layer_parity(shape, L, x_dev, out_gpu, ids_gpu, w_gpu, out_tol, w_tol, label="", rows=None, cache=None):
    """rows: token rows whose outputs are checked (all by default); ids and weights are
    always checked for every token."""
    ids_g = ids_gpu.detach().cpu().numpy()
    w_g = w_gpu.detach().cpu().numpy().astype(np.float64)
    ref = reference(shape, L, x_dev, gpu_ids=ids_g, rows=rows, cache=cache)
    out_g = out_gpu.detach().cpu().numpy().astype(np.float64)[ref["rows"]]
    assert not ref["bad"], f"{label}: GPU top-k outside the valid near-tie sets for tokens {ref['bad']}"
    T = ids_g.shape[0]
    for t in range(T):
        assert set(ids_g[t].tolist()) == set(ref["ids"][t].tolist()), \
            f"{label}: token {t} ids {sorted(ids_g[t].tolist())} != oracle {sorted(ref['ids'][t].tolist())}"
        assert check_order(ref["logits"][t], ids_g[t]), f"{label}: token {t} ids not in logit order"
        wmap = dict(zip(ref["ids"][t].tolist(), ref["w"][t].tolist()))
        for e, wv in zip(ids_g[t].tolist(), w_g[t].tolist()):
            assert abs(wv - wmap[e]) <= w_tol, f"{label}: token {t} expert {e} weight {wv} vs {wmap[e]}"
    rms = float(np.sqrt(np.mean(ref["out"] ** 2)))
    err = float(np.max(np.abs(out_g - ref["out"]))) if out_g.size else 0.0
    assert err <= out_tol * rms, f"{label}: max|out err| {err:.3e} > {out_tol} * RMS {rms:.3e}"
    return dict(err=err, rms=rms, exempt=int(ref["exempt"].sum()), ref=ref)


def tolerances(shape):
    """(out_tol relative to RMS, absolute weight tolerance)."""
    if shape.expert_dtype == "f32" and shape.x_dtype == "f32":
        return 1e-5, 1e-5
    return 2e-2, 2e-4
