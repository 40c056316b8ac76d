"""hyb_attn_forward_frames: several frames in one call, bit-identical to the
per-frame loop of hyb_attn_forward (clean passes), checked on the GPU through
the C ABI; and its host-side argument checks (CPU)."""

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from tests import tolerances as tol

FAKE = 0x10000


def _stack(w, frames):
    xs = [W.pass_inputs(w, n, 0) for n in range(frames)]
    cat = lambda ts: torch.stack(ts).contiguous()
    return xs, [cat([getattr(x, f) for x in xs]) for f in ("q", "k", "v", "gate_logits", "beta_logits")]


def _compare(w, frames, check_oracle=False):
    import gated_delta_linear_b200 as G
    phi = [p.cuda() for p in W.feature_maps(w)]
    dt = G.HYB_BF16 if w.dtype == "bf16" else G.HYB_FP32
    desc = G.make_desc(w.B, w.H, w.T, w.d, dt)
    xs, (q, k, v, g, bl) = _stack(w, frames)
    q, k, v, g, bl = (t.cuda() for t in (q, k, v, g, bl))
    # the per-frame loop
    ws1 = torch.zeros(G.hyb_attn_workspace_bytes(desc), dtype=torch.uint8, device="cuda")
    s1 = torch.zeros(w.B, w.H, w.d, w.d, dtype=torch.float32, device="cuda")
    o1 = torch.empty_like(q)
    for n in range(frames):
        assert G.hyb_attn_forward(desc, q[n], k[n], v[n], *phi, g[n], bl[n], s1, 1, o1[n], ws1) == G.HYB_OK
    # one call
    nb = G.hyb_attn_frames_workspace_bytes(desc, frames)
    assert nb >= ws1.numel()
    ws2 = torch.zeros(nb, dtype=torch.uint8, device="cuda")
    s2 = torch.zeros_like(s1)
    o2 = torch.full_like(q, 3.0)
    assert G.hyb_attn_forward_frames(desc, frames, q, k, v, *phi, g, bl, s2, o2, ws2) == G.HYB_OK
    torch.cuda.synchronize()
    assert G.hyb_attn_get_device_status(ws2) in (G.HYB_OK, G.HYB_WARN_NONFINITE)
    assert torch.equal(o1, o2), "outputs differ from the per-frame loop"
    assert torch.equal(s1, s2), "state differs from the per-frame loop"
    if check_oracle:
        phi64 = [p.double().cpu().numpy() for p in phi]
        S = W.zero_state(w)
        got = o2.double().cpu().numpy()
        for n, x in enumerate(xs):
            ref, _, _, S = oracle.layer_pass(*x.as_f64()[:3], *phi64, *x.as_f64()[3:], S, True)
            for b in range(w.B):
                for h in range(w.H):
                    tol.check(tol.scaled_errors(got[n, b, :, h], ref[b, :, h]),
                              tol.OUT_BF16 if w.dtype == "bf16" else tol.OUT_FP32, f"frame {n} h {h}")
        Sg = s2.double().cpu().numpy()
        assert max(tol.rel_frobenius(Sg[b, h], S[b, h]) for b in range(w.B) for h in range(w.H)) <= \
            (tol.STATE_BF16 if w.dtype == "bf16" else tol.STATE_FP32)


@pytest.mark.gpu
def test_frames_call_equals_loop_480p():
    _compare(W.WORKLOADS[1], 21)


@pytest.mark.gpu
def test_frames_call_matches_oracle_480p_first_frames():
    _compare(W.small_workload(W.WORKLOADS[1], frames=3), 3, check_oracle=True)


@pytest.mark.gpu
def test_frames_call_small_grid_matches_oracle():
    _compare(W.small_workload(W.WORKLOADS[1], H=2, T=200, frames=6), 6, check_oracle=True)


@pytest.mark.gpu
def test_frames_call_ragged_length():
    _compare(W.small_workload(W.WORKLOADS[1], H=4, T=129, frames=4), 4, check_oracle=True)


@pytest.mark.gpu
def test_frames_call_fp32_path():
    w = W.small_workload(W.WORKLOADS[0], passes=(True,))
    _compare(w, w.frames, check_oracle=True)


def test_frames_call_host_validation():
    import gated_delta_linear_b200 as G
    d = G.make_desc(1, 12, 1560, 128)
    need = G.hyb_attn_frames_workspace_bytes(d, 21)
    assert need > G.hyb_attn_frames_workspace_bytes(d, 1) > 0
    assert G.hyb_attn_frames_workspace_bytes(d, 0) == 0
    args = [FAKE] * 10
    assert G.hyb_attn_forward_frames(d, 0, *args, FAKE, 1 << 40, 0) == G.HYB_ERR_INVALID
    assert G.hyb_attn_forward_frames(d, 21, *args, FAKE, need - 1, 0) == G.HYB_ERR_WORKSPACE
    bad = list(args)
    bad[0] = None
    assert G.hyb_attn_forward_frames(d, 21, *bad, FAKE, need, 0) == G.HYB_ERR_INVALID
    # B*H*T = 17: the second frame's gate logits are not 16-byte aligned
    d17 = G.make_desc(1, 1, 17, 128)
    assert G.hyb_attn_forward_frames(d17, 2, *args, FAKE, 1 << 40, 0) == G.HYB_ERR_ALIGN
