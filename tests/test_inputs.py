"""The seeded input recipe both sides consume (moe_inputs), checked on CPU against its
stated definition: Zipf(s) router-logit offsets, RMS-normalised activation rows, weight
spread, bf16 storage, and determinism by seed."""

import math

import numpy as np
import pytest
import torch

import moe_inputs as mi


@pytest.mark.parametrize("E,s", [(512, 1.1), (16, 1.1), (40, 2.0)])
def test_zipf_offsets_are_a_permuted_log_zipf_law(E, s):
    g = torch.Generator().manual_seed(7)
    b = mi.zipf_log_offsets(E, s, g, "cpu").double().numpy()
    # exp(b) is a probability distribution over the experts
    assert abs(np.exp(b).sum() - 1.0) < 1e-5
    # ranked, consecutive offsets follow the power law: b(r) - b(1) = -s ln r
    ranked = np.sort(b)[::-1]
    r = np.arange(1, E + 1)
    assert np.max(np.abs((ranked - ranked[0]) - (-s * np.log(r)))) < 1e-4
    # each rank's offset is used by exactly one expert
    assert len(np.unique(b)) == E


def test_zipf_permutation_depends_on_the_seed_only():
    a = mi.zipf_log_offsets(512, 1.1, torch.Generator().manual_seed(1), "cpu")
    b = mi.zipf_log_offsets(512, 1.1, torch.Generator().manual_seed(1), "cpu")
    c = mi.zipf_log_offsets(512, 1.1, torch.Generator().manual_seed(2), "cpu")
    assert torch.equal(a, b)
    assert not torch.equal(a, c)
    assert torch.equal(torch.sort(a).values, torch.sort(c).values)


def test_activation_rows_are_rms_normalised_then_rounded_to_bf16():
    shape = mi.LayerShape(H=2048, E=512, k=10, I=512, Is=512)
    x = mi.make_x(shape, 8, 123, "cpu")
    assert x.dtype == torch.bfloat16 and x.shape == (8, 2048)
    rms = torch.sqrt((x.double() ** 2).mean(dim=1))
    # rounding to bf16 (8-bit significand, round to nearest) moves each element by at most
    # 2^-8 relative, so the row RMS stays within 2^-8 of 1
    assert torch.all((rms - 1.0).abs() <= 2.0 ** -8)


def test_tiny_fp32_activations_are_plain_normal_draws():
    shape = mi.WORKLOADS["tiny_f32"]["shape"]
    assert shape.x_dtype == "f32" and not shape.rms_norm_x
    x = mi.make_x(shape, 64, 5, "cpu")
    assert x.dtype == torch.float32
    rms = torch.sqrt((x.double() ** 2).mean(dim=1))
    # N(0, 1) rows of 256 draws: RMS near 1 but not normalised to it
    assert torch.all((rms - 1.0).abs() < 0.25)
    assert (rms - 1.0).abs().max() > 1e-3


def test_weights_have_the_stated_spread_and_storage():
    shape = mi.LayerShape(H=256, E=16, k=2, I=64, Is=64)  # bf16, sigma 0.02
    L = mi.make_layer(shape, 11, "cpu")
    for name in ("router_w", "w_gate", "w_up", "w_down", "sh_gate", "sh_up", "sh_down"):
        w = L[name]
        assert w.dtype == torch.bfloat16, name
        sd = float(w.double().std())
        assert abs(sd - shape.sigma) < 0.05 * shape.sigma, (name, sd)
        assert abs(float(w.double().mean())) < 3 * shape.sigma / math.sqrt(w.numel()) + 1e-4, name
    assert L["router_bias"] is None and L["s_gate"] is None


def test_layers_and_activations_are_deterministic_by_seed():
    shape = mi.LayerShape(H=256, E=16, k=2, I=64, Is=64, zipf_s=1.1)
    a, b, c = (mi.make_layer(shape, s, "cpu") for s in (3, 3, 4))
    for name, v in a.items():
        if v is None:
            assert b[name] is None
            continue
        assert torch.equal(v, b[name]), name
        assert not torch.equal(v, c[name]), name
    assert torch.equal(mi.make_x(shape, 5, 9, "cpu"), mi.make_x(shape, 5, 9, "cpu"))
