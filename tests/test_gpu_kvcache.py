"""GPU parity of the key/value-cache softmax baseline (hyb_kvcache_attn_forward)
against the float64 oracle, frame by frame over a growing cache."""

import math

import numpy as np
import pytest
import torch

import gated_delta_linear_b200 as G
import oracle
import workloads as W
from tests import tolerances as tol

pytestmark = pytest.mark.gpu


def _run(w, heads=None, check_frames=None):
    """Feeds w.frames frames through one KVCacheAttention and checks the chosen
    frames and (b, h) pairs; returns the worst scaled errors seen."""
    layer = G.KVCacheAttention(w.B, w.H, w.T, w.d, w.frames)
    heads = heads or [(b, h) for b in range(w.B) for h in range(w.H)]
    s = 1.0 / math.sqrt(w.d)
    ks, vs = [], []
    worst = (0.0, 0.0)
    for n in range(w.frames):
        x = W.pass_inputs(w, n, 0)
        q, k, v = (t.cuda() for t in (x.q, x.k, x.v))
        out = layer.forward(q, k, v)
        torch.cuda.synchronize()
        assert layer.device_status() == G.HYB_OK
        assert layer.cached == (n + 1) * w.T
        ks.append(x.k.double().numpy())
        vs.append(x.v.double().numpy())
        if check_frames is not None and n not in check_frames:
            continue
        got = out.double().cpu().numpy()
        q64 = x.q.double().numpy()
        for b, h in heads:
            ref = oracle.kvcache_attention(q64[b, :, h], [f[b, :, h] for f in ks], [f[b, :, h] for f in vs], s)
            e = tol.scaled_errors(got[b, :, h], ref)
            assert e[0] <= tol.OUT_BF16[0] and e[1] <= tol.OUT_BF16[1], (n, b, h, e)
            worst = (max(worst[0], e[0]), max(worst[1], e[1]))
    return worst


def test_kvcache_small_every_frame():
    w = W.small_workload(W.WORKLOADS[1], wid=60, H=2, T=200, frames=4)
    print("worst", _run(w))


@pytest.mark.parametrize("T", [1, 129])
def test_kvcache_ragged_frames(T):
    w = W.small_workload(W.WORKLOADS[1], wid=61, B=2, H=3, T=T, frames=3)
    print("worst", _run(w))


def test_kvcache_480p_sampled_heads():
    w = W.small_workload(W.WORKLOADS[1], wid=62, frames=3)
    print("worst", _run(w, heads=[(0, 0), (0, 7), (0, 11)], check_frames={0, 2}))


def test_kvcache_first_frame_equals_intra_branch():
    # with nothing cached the baseline is the hybrid layer's intra-frame branch
    w = W.small_workload(W.WORKLOADS[1], wid=63, H=4, T=300, frames=1)
    x = W.pass_inputs(w, 0, 0)
    q, k, v = (t.cuda() for t in (x.q, x.k, x.v))
    base = G.KVCacheAttention(w.B, w.H, w.T, w.d, 1).forward(q, k, v)
    phi = [p.cuda() for p in W.feature_maps(w)]
    hyb = G.HybridAttention(w.B, w.H, w.T, w.d, torch.bfloat16, *phi)
    _, oi, _ = hyb.forward_branches(q, k, v, x.gate_logits.cuda(), x.beta_logits.cuda(), 0)
    torch.cuda.synchronize()
    d = (base.double() - oi.double()).abs()
    assert d.max().item() <= 2e-2 * max(1.0, oi.abs().max().item())


def test_kvcache_deterministic():
    w = W.small_workload(W.WORKLOADS[1], wid=64, H=2, T=256, frames=2)
    outs = []
    for _ in range(2):
        layer = G.KVCacheAttention(w.B, w.H, w.T, w.d, w.frames)
        for n in range(w.frames):
            x = W.pass_inputs(w, n, 0)
            o = layer.forward(x.q.cuda(), x.k.cuda(), x.v.cuda())
        outs.append(o.clone())
    torch.cuda.synchronize()
    assert torch.equal(outs[0], outs[1])
