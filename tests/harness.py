"""Drives the CUDA library and the CPU oracle over the same seeded workload.

The GPU side goes through the C ABI (``gated_delta_linear_b200``); the CPU side
through ``oracle``.  Inputs for both come from ``workloads``.
"""

import numpy as np
import torch

import oracle
import workloads as W
from tests import tolerances as tol


def f64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def phis(w):
    return W.feature_maps(w)


def oracle_state_from_prior_frames(w, phi64):
    """The initial state of a streaming workload: `prior_frames` clean-pass
    updates of S from 0, computed by the oracle's update steps."""
    phq, phk, phv = phi64
    S = W.zero_state(w)
    for j in range(w.prior_frames):
        q, k, v, g, bl = W.prior_frame_inputs(w, j).as_f64()
        for b in range(w.B):
            for h in range(w.H):
                ku = oracle.l2_normalise_rows(oracle.feature_map(k[b, :, h], phk[h]), 1e-6)
                vf = oracle.feature_map(v[b, :, h], phv[h])
                alpha, beta = oracle.frame_gates(g[b, h], bl[b, h])
                S[b, h] = oracle.gated_delta_update(S[b, h], ku, vf, beta, alpha)
    return S


class Run:
    """One workload through the GPU layer, with the oracle checking sampled
    (b, h) pairs after every pass."""

    def __init__(self, w, heads=None, state0=None, check_branches=True):
        import gated_delta_linear_b200 as G
        self.G = G
        self.w = w
        self.heads = heads
        self.check_branches = check_branches
        ph = phis(w)
        self.phi64 = [f64(p) for p in ph]
        self.layer = G.HybridAttention(w.B, w.H, w.T, w.d, w.torch_dtype, *ph)
        if state0 is not None:
            self.layer.state.copy_(torch.from_numpy(state0).to(torch.float32))
        # the oracle starts from exactly what the GPU holds
        self.S_ref = f64(self.layer.state)
        self.worst = {"out": (0.0, 0.0), "intra": (0.0, 0.0), "inter": (0.0, 0.0), "state": 0.0}

    def _track(self, key, errs):
        a, b = self.worst[key]
        self.worst[key] = (max(a, errs[0]), max(b, errs[1]))

    def step(self, frame, pass_idx, clean, check=True):
        w = self.w
        inp = W.pass_inputs(w, frame, pass_idx)
        dev = self.layer.device
        q, k, v = (t.to(dev) for t in (inp.q, inp.k, inp.v))
        g, bl = inp.gate_logits.to(dev), inp.beta_logits.to(dev)
        if self.check_branches:
            out, oi, oe = self.layer.forward_branches(q, k, v, g, bl, clean)
        else:
            out = self.layer.forward(q, k, v, g, bl, clean)
            oi = oe = None
        if not check:
            return
        q64, k64, v64, g64, bl64 = inp.as_f64()
        ref_out, ref_oi, ref_oe, S_new = oracle.layer_pass(
            q64, k64, v64, *self.phi64, g64, bl64, self.S_ref, clean, heads=self.heads)
        got_out = f64(out)
        got_oi = f64(oi) if oi is not None else None
        got_oe = f64(oe) if oe is not None else None
        bf16 = w.dtype == "bf16"
        pairs = self.heads or [(b, h) for b in range(w.B) for h in range(w.H)]
        for b, h in pairs:
            tag = f"frame {frame} pass {pass_idx} b {b} h {h}"
            e = tol.scaled_errors(got_out[b, :, h], ref_out[b, :, h])
            self._track("out", e)
            tol.check(e, tol.OUT_BF16 if bf16 else tol.OUT_FP32, "out " + tag)
            if got_oi is not None:
                e = tol.relative_errors(got_oi[b, :, h], ref_oi[b, :, h])
                self._track("intra", e)
                tol.check(e, tol.INTRA_BF16 if bf16 else tol.BRANCH_FP32, "intra " + tag)
                if np.any(ref_oe[b, :, h] != 0):
                    e = tol.relative_errors(got_oe[b, :, h], ref_oe[b, :, h])
                    self._track("inter", e)
                    tol.check(e, tol.INTER_BF16 if bf16 else tol.BRANCH_FP32, "inter " + tag)
                else:
                    assert np.all(got_oe[b, :, h] == 0), "inter must be exactly 0 " + tag
        if clean:
            got_S = f64(self.layer.state)
            for b, h in pairs:
                r = tol.rel_frobenius(got_S[b, h], S_new[b, h])
                self.worst["state"] = max(self.worst["state"], r)
            self.S_ref = S_new
        return got_out

    def state_error(self):
        got_S = f64(self.layer.state)
        pairs = self.heads or [(b, h) for b in range(self.w.B) for h in range(self.w.H)]
        return max(tol.rel_frobenius(got_S[b, h], self.S_ref[b, h]) for b, h in pairs)
