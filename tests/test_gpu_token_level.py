"""Parity of the token-level access variant (hyb_attn_forward_token_level,
"Technical summary: Attend Locally, Remember Linearly (ARL2)" §4 ablation)
with the float64 oracle's token loop (oracle.token_level_head_pass), through
the C ABI, on the same seeded inputs.  Bounds: tests/tolerances.py (the same
output and state bounds as the frame-level layer)."""

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from tests import tolerances as tol

pytestmark = pytest.mark.gpu


def _oracle_pass(x, phi64, S, clean, T):
    q, k, v, g, bl = x.as_f64()
    B, _, H, d = q.shape
    out = np.empty_like(q)
    S_new = S.copy()
    for b in range(B):
        for h in range(H):
            o, _, _, s = oracle.token_level_head_pass(q[b, :, h], k[b, :, h], v[b, :, h], phi64[0][h], phi64[1][h],
                                                      phi64[2][h], g[b, h] if clean else None,
                                                      bl[b, h] if clean else None, S[b, h], clean)
            out[b, :, h] = o
            S_new[b, h] = s
    return out, S_new


def _run(w, frames=None):
    import gated_delta_linear_b200 as G
    phi = W.feature_maps(w)
    phi64 = [p.to(torch.float64).numpy() for p in phi]
    layer = G.TokenLevelAttention(w.B, w.H, w.T, w.d, w.torch_dtype, *phi)
    S = W.zero_state(w)
    bf16 = w.dtype == "bf16"
    worst = [0.0, 0.0, 0.0]
    for n in range(frames or w.frames):
        for p, clean in enumerate(w.passes):
            x = W.pass_inputs(w, n, p)
            dev = [t.cuda() for t in (x.q, x.k, x.v, x.gate_logits, x.beta_logits)]
            got = layer.forward(*dev, int(clean))
            torch.cuda.synchronize()
            ref, S = _oracle_pass(x, phi64, S, clean, w.T)
            gotn = got.to("cpu", torch.float64).numpy()
            for b in range(w.B):
                for h in range(w.H):
                    e = tol.scaled_errors(gotn[b, :, h], ref[b, :, h])
                    worst[0], worst[1] = max(worst[0], e[0]), max(worst[1], e[1])
                    tol.check(e, tol.OUT_BF16 if bf16 else tol.OUT_FP32, f"frame {n} pass {p} b {b} h {h}")
            Sg = layer.state.to("cpu", torch.float64).numpy()
            r = max(tol.rel_frobenius(Sg[b, h], S[b, h]) for b in range(w.B) for h in range(w.H))
            worst[2] = max(worst[2], r)
            assert r <= (tol.STATE_BF16 if bf16 else tol.STATE_FP32), (n, p, r)
    assert layer.device_status() == G.HYB_OK
    return worst


def test_token_level_480p_size():
    """B1 H12, 1560 tokens (25 chunks, a ragged last one), three frames."""
    print("worst", _run(W.WORKLOADS[1], frames=3))


@pytest.mark.parametrize("T", [1, 17, 63, 64, 65, 129])
def test_token_level_ragged_lengths(T):
    w = W.small_workload(W.WORKLOADS[1], H=3, T=T, frames=3, passes=(False, True))
    print(T, "worst", _run(w))


def test_token_level_strong_forgetting():
    """Gate logits ~ N(-3, 2): forget gates down to ~1e-4 within a chunk."""
    w = W.small_workload(W.WORKLOADS[1], H=2, T=300, frames=3, gate_mu=-3.0, gate_sd=2.0)
    print("worst", _run(w))


def test_token_level_fp32_workload():
    """d = 32, fp32: 2 query-only passes and a clean pass per frame."""
    print("worst", _run(W.WORKLOADS[0]))


def test_token_level_query_only_pass_equals_frame_level():
    import gated_delta_linear_b200 as G
    w = W.small_workload(W.WORKLOADS[1], H=2, T=200, frames=1)
    phi = W.feature_maps(w)
    a = G.TokenLevelAttention(w.B, w.H, w.T, w.d, w.torch_dtype, *phi)
    f = G.HybridAttention(w.B, w.H, w.T, w.d, w.torch_dtype, *phi)
    S0 = torch.randn_like(a.state)
    a.state.copy_(S0)
    f.state.copy_(S0)
    x = W.pass_inputs(w, 0, 0)
    dev = [t.cuda() for t in (x.q, x.k, x.v, x.gate_logits, x.beta_logits)]
    oa = a.forward(*dev, 0)
    of = f.forward(*dev, 0)
    torch.cuda.synchronize()
    assert torch.equal(oa, of) and torch.equal(a.state, S0)
