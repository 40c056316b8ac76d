"""Pins of the oracle's key/value-cache softmax baseline (``kvcache_attention``,
the layer the hybrid one replaces; "Technical summary: Attend Locally, Remember
Linearly (ARL2)", §1 problem statement and §4 efficiency comparison), each
checked against something other than the oracle's own formula, and planted
mistakes that the pins must catch."""

import math

import numpy as np
import pytest
import torch

from oracle import hybrid_layer as O


def _frames(seed, n_frames, T, d, scale=1.0):
    rng = np.random.default_rng(seed)
    q = [rng.standard_normal((T, d)) * scale for _ in range(n_frames)]
    k = [rng.standard_normal((T, d)) * scale for _ in range(n_frames)]
    v = [rng.standard_normal((T, d)) for _ in range(n_frames)]
    return q, k, v


def pin_matches_library_sdpa():
    # textbook attention over the stacked frames, by torch's float64 SDPA
    q, k, v = _frames(1, 3, 9, 8)
    s = 1 / math.sqrt(8)
    got = O.kvcache_attention(q[2], k, v, s)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q[2])[None], torch.from_numpy(np.concatenate(k))[None],
        torch.from_numpy(np.concatenate(v))[None], scale=s)[0].numpy()
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


def pin_identical_keys_average_every_value():
    # one key repeated everywhere: every query takes the mean of all cached values
    q, _, v = _frames(2, 3, 5, 4)
    key = np.random.default_rng(3).standard_normal(4)
    k = [np.tile(key, (5, 1)) for _ in range(3)]
    got = O.kvcache_attention(q[2], k, v, 0.7)
    ref = np.tile(np.concatenate(v).mean(axis=0), (5, 1))
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


def pin_brute_force_scalar_loop():
    # explicit per-query, per-key loop with math.exp on tiny inputs
    q, k, v = _frames(4, 2, 3, 4)
    s = 0.5
    got = O.kvcache_attention(q[1], k, v, s)
    keys = [row for f in k for row in f]
    vals = [row for f in v for row in f]
    for i, qi in enumerate(q[1]):
        logits = [s * sum(float(a) * float(b) for a, b in zip(qi, kj)) for kj in keys]
        mx = max(logits)
        w = [math.exp(x - mx) for x in logits]
        z = sum(w)
        ref = [sum(w[j] * float(vals[j][c]) for j in range(len(keys))) / z for c in range(4)]
        np.testing.assert_allclose(got[i], ref, rtol=1e-12, atol=1e-12)


def pin_order_of_earlier_frames_is_irrelevant():
    # attention is a set operation over the cached keys (no positional term here)
    q, k, v = _frames(5, 4, 6, 8)
    a = O.kvcache_attention(q[3], k, v, 0.3)
    perm = [2, 0, 1, 3]
    b = O.kvcache_attention(q[3], [k[i] for i in perm], [v[i] for i in perm], 0.3)
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-12)


def pin_dominant_key_selects_its_value():
    # one key far more aligned with the query than all others: its value comes back
    q, k, v = _frames(6, 2, 4, 8)
    k = [f.copy() for f in k]
    k[0][2] = q[1][1] * 50.0
    got = O.kvcache_attention(q[1], k, v, 1.0)
    np.testing.assert_allclose(got[1], v[0][2], rtol=0, atol=1e-9)


PINS = [pin_matches_library_sdpa, pin_identical_keys_average_every_value, pin_brute_force_scalar_loop,
        pin_order_of_earlier_frames_is_irrelevant, pin_dominant_key_selects_its_value]


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin()


def _drop_current_frame(q, k_frames, v_frames, sm_scale):
    return _orig(q, k_frames[:-1] or k_frames, v_frames[:-1] or v_frames, sm_scale)


def _unit_scale(q, k_frames, v_frames, sm_scale):
    return _orig(q, k_frames, v_frames, 1.0)


def _normalise_over_queries(q, k_frames, v_frames, sm_scale):
    k = np.concatenate(k_frames)
    v = np.concatenate(v_frames)
    s = (np.asarray(q) @ k.T) * sm_scale
    w = np.exp(s - s.max(axis=0, keepdims=True))
    return (w / w.sum(axis=0, keepdims=True)) @ v


_orig = O.kvcache_attention


@pytest.mark.parametrize("mutant", [_drop_current_frame, _unit_scale, _normalise_over_queries],
                         ids=lambda f: f.__name__)
def test_planted_mistakes_are_caught(mutant, monkeypatch):
    monkeypatch.setattr(O, "kvcache_attention", mutant)
    caught = 0
    for pin in PINS:
        try:
            pin()
        except AssertionError:
            caught += 1
    assert caught >= 1, f"no pin caught {mutant.__name__}"
