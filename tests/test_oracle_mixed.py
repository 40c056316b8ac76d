"""Pins of the oracle's branch combination ``mixed_output`` (a O_intra +
c O_inter; "LinVideo: A Post-Training Framework towards O(n) Attention in
Efficient Video Generation" §2(b); "SALAD: Achieve High-Sparsity Attention via
Efficient Linear Attention Tuning for Video Diffusion Transformer" §2)."""

import math

import numpy as np
import pytest
import torch

from oracle import hybrid_layer as O


def _layer(seed=0, T=6, d=8):
    rng = np.random.default_rng(seed)
    q, k, v = (rng.standard_normal((1, T, 2, d)) for _ in range(3))
    phi = [np.eye(d)[None].repeat(2, 0) + 0.05 * rng.standard_normal((2, d, d)) for _ in range(3)]
    g, bl = rng.standard_normal((1, 2, T)), rng.standard_normal((1, 2, T))
    S = rng.standard_normal((1, 2, d, d))
    return q, k, v, phi, g, bl, S


def pin_unit_weights_give_the_layer_output():
    q, k, v, phi, g, bl, S = _layer(1)
    out, oi, oe, _ = O.layer_pass(q, k, v, *phi, g, bl, S, False)
    np.testing.assert_allclose(O.mixed_output(oi[0, :, 1], oe[0, :, 1], 1.0, 1.0), out[0, :, 1], rtol=0, atol=1e-12)


def pin_full_softmax_weight_is_library_sdpa():
    # r = 1 keeps only the softmax branch: torch's float64 SDPA of the frame
    q, k, v, phi, g, bl, S = _layer(2)
    _, oi, oe, _ = O.layer_pass(q, k, v, *phi, g, bl, S, False)
    got = O.mixed_output(oi[0, :, 0], oe[0, :, 0], 1.0, 0.0)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q[0, :, 0])[None], torch.from_numpy(k[0, :, 0])[None], torch.from_numpy(v[0, :, 0])[None],
        scale=1 / math.sqrt(8))[0].numpy()
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


def pin_full_linear_weight_with_zero_state_is_zero():
    q, k, v, phi, g, bl, _ = _layer(3)
    _, oi, oe, _ = O.layer_pass(q, k, v, *phi, g, bl, np.zeros((1, 2, 8, 8)), False)
    assert np.all(O.mixed_output(oi[0, :, 0], oe[0, :, 0], 0.0, 1.0) == 0.0)


def pin_bilinear_in_the_weights():
    rng = np.random.default_rng(4)
    a1, a2 = rng.standard_normal((2, 5, 3))
    x = O.mixed_output(a1, a2, 0.3, -1.7)
    y = O.mixed_output(a1, a2, 0.5, 2.0)
    np.testing.assert_allclose(O.mixed_output(a1, a2, 0.8, 0.3), x + y, rtol=1e-12, atol=1e-12)


PINS = [pin_unit_weights_give_the_layer_output, pin_full_softmax_weight_is_library_sdpa,
        pin_full_linear_weight_with_zero_state_is_zero, pin_bilinear_in_the_weights]


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin()


_orig = O.mixed_output


def _swapped(o_intra, o_inter, a, c):
    return _orig(o_intra, o_inter, c, a)


def _intra_only(o_intra, o_inter, a, c):
    return _orig(o_intra, o_inter, a, 0.0)


@pytest.mark.parametrize("mutant", [_swapped, _intra_only], ids=lambda f: f.__name__)
def test_planted_mistakes_are_caught(mutant, monkeypatch):
    monkeypatch.setattr(O, "mixed_output", mutant)
    caught = 0
    for pin in PINS:
        try:
            pin()
        except AssertionError:
            caught += 1
    assert caught >= 1, f"no pin caught {mutant.__name__}"
