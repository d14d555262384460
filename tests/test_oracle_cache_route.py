"""Pins of the oracle's opt-in cache-aware routing (selection by z + lambda * Delta *
cached, Delta the token's logit range; weights from the unbiased softmax renormalised over
the selection) against hand-derived values, the plain router, and brute force."""

import itertools
from fractions import Fraction

import numpy as np
import pytest

import moe_inputs as mi
import oracle

Z = np.log(np.array([[1.0, 2.0, 3.0, 4.0]]))  # softmax p = (1, 2, 3, 4) / 10, Delta = ln 4


@pytest.mark.parametrize("cached,lam,ids,w", [
    # z' = (ln4, ln2, ln3, ln4): experts 0 and 3 tie at ln 4, the lower id first; the weights
    # mix the unbiased p_0 = 1/10 and p_3 = 4/10
    ((1, 0, 0, 0), 1.0, (0, 3), (Fraction(1, 5), Fraction(4, 5))),
    # z' = (ln2, ln2, ln3, ln4): the bias is too small to change the selection
    ((1, 0, 0, 0), 0.5, (3, 2), (Fraction(4, 7), Fraction(3, 7))),
    # z' = (ln4, ln8, ln3, ln4): expert 1 first, then the tie at ln 4 goes to expert 0
    ((1, 1, 0, 0), 1.0, (1, 0), (Fraction(2, 3), Fraction(1, 3))),
    # lambda = 0 is plain routing whatever is cached
    ((1, 1, 0, 0), 0.0, (3, 2), (Fraction(4, 7), Fraction(3, 7))),
    # everything cached: a common shift of every logit changes nothing
    ((1, 1, 1, 1), 3.0, (3, 2), (Fraction(4, 7), Fraction(3, 7))),
])
def test_hand_derived_cases(cached, lam, ids, w):
    r = oracle.cache_route(Z, np.array(cached, np.uint8), lam, 2)
    np.testing.assert_array_equal(r["ids"][0], ids)
    np.testing.assert_allclose(r["w"][0], [float(f) for f in w], rtol=0, atol=1e-15)


SHAPES = {
    "bf16_E16_k4": mi.LayerShape(H=64, E=16, k=4, I=32, Is=32, sigma=0.3),
    "bf16_E12_k3_bias": mi.LayerShape(H=32, E=12, k=3, I=32, Is=32, sigma=0.3, zipf_s=1.1),
}


def _router(name, T=6, seed=21):
    shape = SHAPES[name]
    L = mi.make_layer(shape, seed, "cpu")
    x = mi.to_numpy(mi.make_x(shape, T, seed, "cpu"))
    return shape, oracle.router(mi.layer_to_numpy(L), shape, x)


@pytest.mark.parametrize("name", list(SHAPES))
def test_lambda_zero_is_the_plain_router(name):
    shape, r = _router(name)
    cached = np.random.default_rng(0).integers(0, 2, shape.E).astype(np.uint8)
    c = oracle.cache_route(r["logits"], cached, 0.0, shape.k)
    np.testing.assert_array_equal(c["ids"], r["ids"])
    np.testing.assert_allclose(c["w"], r["w"], rtol=0, atol=1e-15)


@pytest.mark.parametrize("name", list(SHAPES))
@pytest.mark.parametrize("lam", [0.05, 0.3, 1.0, 1.5])
def test_selection_equals_a_brute_force_sort_and_weights_the_unbiased_softmax(name, lam):
    shape, r = _router(name)
    rng = np.random.default_rng(int(lam * 100))
    cached = rng.integers(0, 2, shape.E).astype(np.uint8)
    c = oracle.cache_route(r["logits"], cached, lam, shape.k)
    for t in range(r["logits"].shape[0]):
        z = r["logits"][t]
        delta = z.max() - z.min()
        zb = [z[e] + lam * delta * cached[e] for e in range(shape.E)]
        order = sorted(range(shape.E), key=lambda e: (-zb[e], e))
        np.testing.assert_array_equal(c["ids"][t], order[:shape.k])
        sel = z[order[:shape.k]]
        ex = np.exp(sel - sel.max())
        np.testing.assert_allclose(c["w"][t], ex / ex.sum(), rtol=0, atol=1e-14)
        np.testing.assert_allclose(c["biased"][t], zb, rtol=0, atol=0)


def test_strong_bias_picks_only_cached_experts_when_enough_are_cached():
    shape, r = _router("bf16_E16_k4", T=8)
    for seed in range(5):
        cached = np.zeros(shape.E, np.uint8)
        cached[np.random.default_rng(seed).choice(shape.E, shape.k + 2, replace=False)] = 1
        c = oracle.cache_route(r["logits"], cached, 1.5, shape.k)
        for t in range(8):
            assert all(cached[e] for e in c["ids"][t])
            # and they are the k best cached experts by the unbiased logits
            cand = [e for e in range(shape.E) if cached[e]]
            best = sorted(cand, key=lambda e: (-r["logits"][t][e], e))[:shape.k]
            assert sorted(c["ids"][t].tolist()) == sorted(best)


def test_few_cached_are_all_taken_then_the_best_uncached():
    shape, r = _router("bf16_E16_k4", T=5)
    cached = np.zeros(shape.E, np.uint8)
    cached[[2, 9]] = 1
    c = oracle.cache_route(r["logits"], cached, 2.0, shape.k)
    for t in range(5):
        ids = c["ids"][t].tolist()
        assert ids[:2] == sorted([2, 9], key=lambda e: (-r["logits"][t][e], e))
        rest = sorted((e for e in range(shape.E) if e not in (2, 9)), key=lambda e: (-r["logits"][t][e], e))
        assert ids[2:] == rest[:2]


def test_subsets_by_enumeration_on_a_tiny_row():
    # every k-subset is scored by its smallest biased logit; the selection must be a subset
    # whose smallest member beats every expert outside it (ties by id)
    z = np.array([[0.3, -1.2, 0.9, 0.1, -0.4]])
    cached = np.array([0, 1, 0, 1, 1], np.uint8)
    for lam in (0.1, 0.4, 0.8):
        c = oracle.cache_route(z, cached, lam, 3)
        zb = z[0] + lam * (z.max() - z.min()) * cached
        good = []
        for sub in itertools.combinations(range(5), 3):
            out = [e for e in range(5) if e not in sub]
            if all((zb[a], -a) > (zb[b], -b) for a in sub for b in out):
                good.append(sorted(sub))
        assert good == [sorted(c["ids"][0].tolist())]
