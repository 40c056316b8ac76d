"""GPU parity of the branch-weighted pass (hyb_attn_forward_mixed): out =
a O_intra + c O_inter per (batch, head), against the float64 oracle; the
state update is the one of the plain pass."""

import numpy as np
import pytest
import torch

import gated_delta_linear_b200 as G
import oracle
import workloads as W
from tests import tolerances as tol
from tests.harness import f64

pytestmark = pytest.mark.gpu


def _mix(w, seed):
    rng = np.random.default_rng(seed)
    r = rng.uniform(0.0, 1.0, (w.B, w.H))
    s = 1.0 / (1.0 + np.exp(-rng.standard_normal((w.B, w.H))))
    mix = np.empty((w.B, w.H, 2), dtype=np.float32)
    mix[..., 0] = np.where(np.arange(w.H)[None] % 2 == 0, r, 1.0)   # even heads: (r, 1 - r)
    mix[..., 1] = np.where(np.arange(w.H)[None] % 2 == 0, 1.0 - r, s)  # odd heads: (1, sigmoid(z))
    return mix


@pytest.mark.parametrize("wid", [0, 1])
def test_mixed_pass_matches_oracle_and_keeps_the_update(wid):
    base = W.WORKLOADS[wid]
    w = W.small_workload(base, wid=70 + wid, H=4 if wid == 1 else base.H, T=300 if wid == 1 else base.T,
                         frames=2)
    ph = W.feature_maps(w)
    phi64 = [f64(p) for p in ph]
    mixed = G.HybridAttention(w.B, w.H, w.T, w.d, w.torch_dtype, *ph)
    plain = G.HybridAttention(w.B, w.H, w.T, w.d, w.torch_dtype, *ph)
    mix = _mix(w, 7 + wid)
    mix_dev = torch.from_numpy(mix).cuda()
    S_ref = f64(plain.state)
    bf16 = w.dtype == "bf16"
    for n in range(w.frames):
        x = W.pass_inputs(w, n, 0)
        q, k, v, g, bl = (t.cuda() for t in (x.q, x.k, x.v, x.gate_logits, x.beta_logits))
        out = mixed.forward_mixed(q, k, v, g, bl, 1, mix_dev)
        plain.forward(q, k, v, g, bl, 1)
        torch.cuda.synchronize()
        assert mixed.device_status() == G.HYB_OK
        _, ref_oi, ref_oe, S_ref = oracle.layer_pass(*x.as_f64()[:3], *phi64, *x.as_f64()[3:], S_ref, True)
        got = f64(out)
        for b in range(w.B):
            for h in range(w.H):
                ref = oracle.mixed_output(ref_oi[b, :, h], ref_oe[b, :, h], float(mix[b, h, 0]), float(mix[b, h, 1]))
                e = tol.scaled_errors(got[b, :, h], ref)
                tol.check(e, tol.OUT_BF16 if bf16 else tol.OUT_FP32, f"mixed out frame {n} b {b} h {h}")
        # the weights change only the output: the state update is bit-identical
        assert torch.equal(mixed.state, plain.state)


def test_unit_weights_equal_the_plain_pass():
    w = W.small_workload(W.WORKLOADS[1], wid=72, H=3, T=257, frames=2)
    ph = W.feature_maps(w)
    a = G.HybridAttention(w.B, w.H, w.T, w.d, torch.bfloat16, *ph)
    b = G.HybridAttention(w.B, w.H, w.T, w.d, torch.bfloat16, *ph)
    ones = torch.ones(w.B, w.H, 2, device="cuda")
    for n in range(w.frames):
        x = W.pass_inputs(w, n, 0)
        q, k, v, g, bl = (t.cuda() for t in (x.q, x.k, x.v, x.gate_logits, x.beta_logits))
        oa = a.forward_mixed(q, k, v, g, bl, 1, ones)
        ob = b.forward(q, k, v, g, bl, 1)
        torch.cuda.synchronize()
        assert torch.equal(oa, ob)
