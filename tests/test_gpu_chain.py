"""hyb_attn_forward_next: one call per pass, each clean pass's delta update
writing the next frame's W = phi_q^T S_N so the next call skips the prep kernel
and its attention kernel starts while the update still runs.  Checked on the
GPU through the C ABI: bit-identical outputs and state to the per-pass loop of
hyb_attn_forward (the same arithmetic in the same order), with every pass
enqueued back to back on one stream and no host synchronisation in between, and
on small grids against the oracle (ARL2 summary §2.2: every token of frame N
reads the pre-update S_{N-1}, which a chained pass must still see)."""

import pytest
import torch

import oracle
import workloads as W
from tests import tolerances as tol


def _setup(w):
    import gated_delta_linear_b200 as G
    phi = [p.cuda() for p in W.feature_maps(w)]
    dt = G.HYB_BF16 if w.dtype == "bf16" else G.HYB_FP32
    desc = G.make_desc(w.B, w.H, w.T, w.d, dt)
    passes = [(n, p, bool(c)) for n in range(w.frames) for p, c in enumerate(w.passes)]
    xs = [W.pass_inputs(w, n, p) for n, p, _ in passes]
    dev = [[getattr(x, f).cuda() for f in ("q", "k", "v", "gate_logits", "beta_logits")] for x in xs]
    return G, phi, desc, passes, xs, dev


def _initial_state(G, w, phi, desc):
    """S_0: zero, or the state the layer builds from the workload's prior frames."""
    s = torch.zeros(w.B, w.H, w.d, w.d, dtype=torch.float32, device="cuda")
    if w.prior_frames:
        ws = torch.zeros(G.hyb_attn_workspace_bytes(desc), dtype=torch.uint8, device="cuda")
        for j in range(w.prior_frames):
            x = W.prior_frame_inputs(w, j)
            q, k, v, g, b = (getattr(x, f).cuda() for f in ("q", "k", "v", "gate_logits", "beta_logits"))
            assert G.hyb_attn_forward(desc, q, k, v, *phi, g, b, s, 1, torch.empty_like(q), ws) == G.HYB_OK
        torch.cuda.synchronize()
    return s


def _run(G, fn, desc, phi, passes, dev, s0, ws=None):
    ws = ws if ws is not None else torch.zeros(G.hyb_attn_workspace_bytes(desc), dtype=torch.uint8, device="cuda")
    s = s0.clone()
    outs = []
    for (n, p, clean), (q, k, v, g, b) in zip(passes, dev):
        o = torch.empty_like(q)
        assert fn(desc, q, k, v, *phi, g, b, s, int(clean), o, ws) == G.HYB_OK
        outs.append(o)
    return outs, s, ws


def _check_oracle(w, phi, passes, xs, outs, s_final, s0):
    phi64 = [p.double().cpu().numpy() for p in phi]
    S = s0.double().cpu().numpy()
    for (n, p, clean), x, o in zip(passes, xs, outs):
        ref, _, _, S = oracle.layer_pass(*x.as_f64()[:3], *phi64, *x.as_f64()[3:], S, clean)
        got = o.double().cpu().numpy()
        for b in range(w.B):
            for h in range(w.H):
                tol.check(tol.scaled_errors(got[b, :, h], ref[b, :, h]),
                          tol.OUT_BF16 if w.dtype == "bf16" else tol.OUT_FP32, f"frame {n} pass {p} h {h}")
    Sg = s_final.double().cpu().numpy()
    assert max(tol.rel_frobenius(Sg[b, h], S[b, h]) for b in range(w.B) for h in range(w.H)) <= \
        (tol.STATE_BF16 if w.dtype == "bf16" else tol.STATE_FP32)


def _compare(w, check_oracle=False):
    G, phi, desc, passes, xs, dev = _setup(w)
    s0 = _initial_state(G, w, phi, desc)
    o1, s1, _ = _run(G, G.hyb_attn_forward, desc, phi, passes, dev, s0)
    o2, s2, ws2 = _run(G, G.hyb_attn_forward_next, desc, phi, passes, dev, s0)
    torch.cuda.synchronize()
    assert G.hyb_attn_get_device_status(ws2) in (G.HYB_OK, G.HYB_WARN_NONFINITE)
    for i, (a, b) in enumerate(zip(o1, o2)):
        assert torch.equal(a, b), f"pass {i}: output differs from the per-pass loop"
    assert torch.equal(s1, s2), "state differs from the per-pass loop"
    if check_oracle:
        _check_oracle(w, phi, passes, xs, o2, s2, s0)


@pytest.mark.gpu
def test_chain_equals_loop_480p_21_frames():
    _compare(W.WORKLOADS[1])


@pytest.mark.gpu
def test_chain_small_grid_matches_oracle_21_frames():
    # 2 heads x 2 query tiles: every attention CTA is resident at once, so a
    # chained attention kernel and the next update run beside the previous update
    _compare(W.small_workload(W.WORKLOADS[1], H=2, T=200), check_oracle=True)


@pytest.mark.gpu
def test_chain_ragged_length_matches_oracle():
    _compare(W.small_workload(W.WORKLOADS[1], H=4, T=129, frames=6), check_oracle=True)


@pytest.mark.gpu
def test_chain_two_query_tiles_per_cta_ragged_matches_oracle():
    # 12 heads x 13 query tiles (the last holding one row): chained passes run
    # two consecutive query tiles per attention CTA, 7 CTAs per head, the last
    # with one tile
    _compare(W.small_workload(W.WORKLOADS[1], T=1537, frames=3), check_oracle=True)


@pytest.mark.gpu
def test_chain_streaming_passes_equal_loop():
    # 4 query-only passes and a clean pass per frame on a pre-filled state
    _compare(W.small_workload(W.WORKLOADS[2], H=12, frames=3, prior_frames=4))


@pytest.mark.gpu
def test_chain_streaming_passes_small_grid_matches_oracle():
    _compare(W.small_workload(W.WORKLOADS[2], H=2, T=200, frames=4, prior_frames=3), check_oracle=True)


@pytest.mark.gpu
def test_chain_fp32_path_equals_loop():
    _compare(W.WORKLOADS[0], check_oracle=True)


@pytest.mark.gpu
def test_chain_restarts_after_state_reset():
    """Resetting the state ends the chain only through another pass on the
    workspace: a hyb_attn_forward call after the reset, then chained calls."""
    w = W.small_workload(W.WORKLOADS[1], H=4, T=300, frames=6)
    G, phi, desc, passes, xs, dev = _setup(w)
    s0 = torch.zeros(w.B, w.H, w.d, w.d, dtype=torch.float32, device="cuda")
    ref_o, ref_s, _ = _run(G, G.hyb_attn_forward, desc, phi, passes, dev, s0)
    ws = torch.zeros(G.hyb_attn_workspace_bytes(desc), dtype=torch.uint8, device="cuda")
    s = s0.clone()
    for (n, p, clean), (q, k, v, g, b) in zip(passes[:3], dev[:3]):
        assert G.hyb_attn_forward_next(desc, q, k, v, *phi, g, b, s, int(clean), torch.empty_like(q), ws) == G.HYB_OK
    s.zero_()  # the caller restores S_0 ...
    outs = []
    for i, ((n, p, clean), (q, k, v, g, b)) in enumerate(zip(passes, dev)):
        o = torch.empty_like(q)
        fn = G.hyb_attn_forward if i == 0 else G.hyb_attn_forward_next  # ... and restarts with a plain pass
        assert fn(desc, q, k, v, *phi, g, b, s, int(clean), o, ws) == G.HYB_OK
        outs.append(o)
    torch.cuda.synchronize()
    assert G.hyb_attn_get_device_status(ws) == G.HYB_OK
    for a, b in zip(ref_o, outs):
        assert torch.equal(a, b)
    assert torch.equal(ref_s, s)


@pytest.mark.gpu
def test_chain_two_layers_interleaved():
    """Two layers (own state and workspace) called in turn: each keeps its chain."""
    wa = W.small_workload(W.WORKLOADS[1], H=4, T=300, frames=5)
    wb = W.small_workload(W.WORKLOADS[1], H=4, T=300, frames=5, wid=wa.wid + 100)
    Ga, phia, desca, pa, _, deva = _setup(wa)
    _, phib, descb, pb, _, devb = _setup(wb)
    s0 = torch.zeros(wa.B, wa.H, wa.d, wa.d, dtype=torch.float32, device="cuda")
    ref_a = _run(Ga, Ga.hyb_attn_forward, desca, phia, pa, deva, s0)
    ref_b = _run(Ga, Ga.hyb_attn_forward, descb, phib, pb, devb, s0)
    wsa = torch.zeros(Ga.hyb_attn_workspace_bytes(desca), dtype=torch.uint8, device="cuda")
    wsb = torch.zeros_like(wsa)
    sa, sb = s0.clone(), s0.clone()
    oa, ob = [], []
    for (n, p, ca), xa, (_, _, cb), xb in zip(pa, deva, pb, devb):
        for (phi, desc, x, c, s, ws, outs) in ((phia, desca, xa, ca, sa, wsa, oa), (phib, descb, xb, cb, sb, wsb, ob)):
            o = torch.empty_like(x[0])
            assert Ga.hyb_attn_forward_next(desc, *x[:3], *phi, *x[3:], s, int(c), o, ws) == Ga.HYB_OK
            outs.append(o)
    torch.cuda.synchronize()
    for ref, got, s in ((ref_a, oa, sa), (ref_b, ob, sb)):
        for a, b in zip(ref[0], got):
            assert torch.equal(a, b)
        assert torch.equal(ref[1], s)
    assert Ga.hyb_attn_get_device_status(wsa) == Ga.HYB_OK
    assert Ga.hyb_attn_get_device_status(wsb) == Ga.HYB_OK


@pytest.mark.gpu
def test_chain_other_stream_starts_a_new_chain():
    """A call on another stream (ordered by an event) does not continue the chain."""
    w = W.small_workload(W.WORKLOADS[1], H=4, T=300, frames=4)
    G, phi, desc, passes, xs, dev = _setup(w)
    s0 = torch.zeros(w.B, w.H, w.d, w.d, dtype=torch.float32, device="cuda")
    ref_o, ref_s, _ = _run(G, G.hyb_attn_forward, desc, phi, passes, dev, s0)
    ws = torch.zeros(G.hyb_attn_workspace_bytes(desc), dtype=torch.uint8, device="cuda")
    s = s0.clone()
    streams = [torch.cuda.current_stream(), torch.cuda.Stream()]
    outs = []
    for i, ((n, p, clean), (q, k, v, g, b)) in enumerate(zip(passes, dev)):
        st = streams[(i // 2) % 2]
        prev = streams[((i - 1) // 2) % 2] if i else st
        if prev is not st:
            st.wait_stream(prev)
        o = torch.empty_like(q)
        with torch.cuda.stream(st):
            assert G.hyb_attn_forward_next(desc, q, k, v, *phi, g, b, s, int(clean), o, ws,
                                           stream=st) == G.HYB_OK
        outs.append(o)
    streams[0].wait_stream(streams[1])
    torch.cuda.synchronize()
    for a, b in zip(ref_o, outs):
        assert torch.equal(a, b)
    assert torch.equal(ref_s, s)
    assert G.hyb_attn_get_device_status(ws) == G.HYB_OK


@pytest.mark.gpu
def test_chain_interleaved_with_a_frames_call():
    """Chained passes, then a frames call on the same state and workspace (it
    ends the chain and writes the state), then chained passes again: every
    output and the final state equal the per-pass loop of hyb_attn_forward."""
    w = W.small_workload(W.WORKLOADS[1], H=4, T=300, frames=9)
    G, phi, desc, passes, xs, dev = _setup(w)
    s0 = torch.zeros(w.B, w.H, w.d, w.d, dtype=torch.float32, device="cuda")
    ref_o, ref_s, _ = _run(G, G.hyb_attn_forward, desc, phi, passes, dev, s0)
    nb = G.hyb_attn_frames_workspace_bytes(desc, 3)
    ws = torch.zeros(nb, dtype=torch.uint8, device="cuda")
    s = s0.clone()
    outs = []
    for i in range(3):
        q, k, v, g, b = dev[i]
        o = torch.empty_like(q)
        assert G.hyb_attn_forward_next(desc, q, k, v, *phi, g, b, s, 1, o, ws) == G.HYB_OK
        outs.append(o)
    stk = [torch.stack([dev[i][f] for i in range(3, 6)]).contiguous() for f in range(5)]
    of = torch.empty_like(stk[0])
    assert G.hyb_attn_forward_frames(desc, 3, *stk[:3], *phi, *stk[3:], s, of, ws) == G.HYB_OK
    outs += [of[i] for i in range(3)]
    for i in range(6, 9):
        q, k, v, g, b = dev[i]
        o = torch.empty_like(q)
        assert G.hyb_attn_forward_next(desc, q, k, v, *phi, g, b, s, 1, o, ws) == G.HYB_OK
        outs.append(o)
    torch.cuda.synchronize()
    assert G.hyb_attn_get_device_status(ws) == G.HYB_OK
    for i, (a, b) in enumerate(zip(ref_o, outs)):
        assert torch.equal(a, b), f"pass {i}"
    assert torch.equal(ref_s, s)
