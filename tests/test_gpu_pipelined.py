"""Frames issued back to back, as the benchmark issues them, checked against the
float64 oracle.

Every other parity test reads each pass's output back before the next pass,
which serialises the kernels of consecutive frames.  Here all frames of a
stream are enqueued on one CUDA stream without any host synchronisation, each
frame's output into its own buffer, so the kernels of frame N+1 may overlap
those of frame N exactly as in the timed loop.  Only then are the outputs and
the final state read and compared with the oracle.  Frame-level access (ARL2
summary, "Technical summary: Attend Locally, Remember Linearly (ARL2)" §2.2):
every token of frame N reads S_{N-1}, and the state is written after those
reads -- an ordering fault between a frame's reads and its update, or between
one frame's update and the next frame's reads, shows up as an output or state
mismatch.
"""

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from tests import tolerances as tol

pytestmark = pytest.mark.gpu


def _stream_parity(w):
    import gated_delta_linear_b200 as G
    phi = W.feature_maps(w)
    phi64 = [p.to(torch.float64).numpy() for p in phi]
    layer = G.HybridAttention(w.B, w.H, w.T, w.d, w.torch_dtype, *phi)
    host = [W.pass_inputs(w, n, 0) for n in range(w.frames)]
    dev = [[t.cuda() for t in (x.q, x.k, x.v, x.gate_logits, x.beta_logits)] for x in host]
    outs = [torch.empty_like(f[0]) for f in dev]
    torch.cuda.synchronize()
    for f, o in zip(dev, outs):          # no host synchronisation between frames
        layer.forward(*f, 1, out=o)
    torch.cuda.synchronize()
    assert layer.device_status() == G.HYB_OK

    S = W.zero_state(w)
    for n, x in enumerate(host):
        q, k, v, g, bl = x.as_f64()
        ref, _, _, S = oracle.layer_pass(q, k, v, *phi64, g, bl, S, True)
        got = outs[n].to("cpu", torch.float64).numpy()
        for b in range(w.B):
            for h in range(w.H):
                tol.check(tol.scaled_errors(got[b, :, h], ref[b, :, h]), tol.OUT_BF16,
                          f"{w.name} frame {n} b {b} h {h}")
    got_S = layer.state.to("cpu", torch.float64).numpy()
    worst = max(tol.rel_frobenius(got_S[b, h], S[b, h]) for b in range(w.B) for h in range(w.H))
    assert worst <= tol.STATE_BF16, worst
    return worst


def test_480p_stream_back_to_back_matches_oracle():
    """The benchmark's workload: B1 H12, 21 frames of 1560 tokens."""
    print("state rel", _stream_parity(W.WORKLOADS[1]))


def test_small_grid_stream_back_to_back_matches_oracle():
    """A small grid (2 heads, 200 tokens): every CTA of a kernel is resident at
    once, so nothing but the launch ordering separates the kernels."""
    w = W.small_workload(W.WORKLOADS[1], H=2, T=200, frames=21)
    print("state rel", _stream_parity(w))
