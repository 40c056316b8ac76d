"""Token Radius Attention on the intra-frame branch (hyb_tra_forward;
"Technical summary: Token Radius Attention" §2), checked through the C ABI
against the float64 oracle (oracle.tra) on seeded tile-major inputs.

The block mask is decided from fp32 entropies on the GPU.  The oracle takes
the GPU's entropies (after checking them against its own float64 ones) and
decides the mask in fp32 too; a decision whose squared distance lies within
1e-5 of a radius could round either way, so the oracle brackets the mask with
the radii scaled by (1 - 1e-5) and (1 + 1e-5), and each query block's output is
compared only where the two brackets agree (and the count of such blocks is
bounded)."""

import math

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from oracle import tra as R
from tests import tolerances as tol

pytestmark = pytest.mark.gpu

BLOCK = 128


def _setup(w, tau, votes_min, grid, tiles):
    import gated_delta_linear_b200 as G
    gh, gw = grid
    params = G.HybTraParams(gh, gw, tiles[0], tiles[1], tau, votes_min)
    desc = G.make_desc(w.B, w.H, w.T, w.d, G.HYB_BF16)
    phi = [p.cuda() for p in W.feature_maps(w)]
    ws = torch.zeros(G.hyb_tra_workspace_bytes(desc), dtype=torch.uint8, device="cuda")
    ent = torch.zeros(w.B, w.H, w.T, dtype=torch.float32, device="cuda")
    return G, params, desc, phi, ws, ent


def _oracle_mask(ent32, tau, T, pos, votes_min, scale):
    # fp32 radius as the kernel forms it: clamp(tau exp(H), 1, T) / pi
    H = np.asarray(ent32, dtype=np.float32)
    k = np.clip(np.float32(tau) * np.exp(H), np.float32(1.0), np.float32(T)).astype(np.float32)
    r2 = (k * np.float32(0.31830988618379067)).astype(np.float64) * scale
    return R.block_mask(R.block_votes(pos, np.sqrt(r2), BLOCK), votes_min)


def _run(w, tau, votes_min, grid, tiles, frames=2):
    G, params, desc, phi, ws, ent = _setup(w, tau, votes_min, grid, tiles)
    phi64 = [p.double().cpu().numpy() for p in phi]
    pos = R.tile_major_positions(grid[0], grid[1], tiles[0], tiles[1])
    S_gpu = torch.zeros(w.B, w.H, w.d, w.d, dtype=torch.float32, device="cuda")
    S_ref = W.zero_state(w)
    sc = 1.0 / math.sqrt(w.d)
    kept, skipped, total = 0, 0, 0
    for n in range(frames):
        x = W.pass_inputs(w, n, 0)
        q, k, v, g, bl = (t.cuda() for t in (x.q, x.k, x.v, x.gate_logits, x.beta_logits))
        q64, k64, v64, g64, bl64 = x.as_f64()
        # warm-up: the dense pass, bit-identical to hyb_attn_forward, plus entropies
        ws_ref = torch.zeros(G.hyb_attn_workspace_bytes(desc), dtype=torch.uint8, device="cuda")
        S_chk = S_gpu.clone()
        o_ref = torch.empty_like(q)
        assert G.hyb_attn_forward(desc, q, k, v, *phi, g, bl, S_chk, 0, o_ref, ws_ref) == G.HYB_OK
        o_w = torch.empty_like(q)
        assert G.hyb_tra_forward(desc, params, 1, q, k, v, *phi, g, bl, S_gpu, 0, o_w, ent, ws) == G.HYB_OK
        torch.cuda.synchronize()
        assert torch.equal(o_w, o_ref), "the warm-up pass must equal the dense pass"
        e_gpu = ent.cpu().numpy()
        for b in range(w.B):
            for h in range(w.H):
                e_ref = R.attention_entropy(q64[b, :, h], k64[b, :, h], sc)
                err = np.abs(e_gpu[b, h] - e_ref).max()
                assert err <= 1e-4 * max(1.0, np.abs(e_ref).max()), (n, b, h, err)
        # sparse clean pass
        out = torch.empty_like(q)
        assert G.hyb_tra_forward(desc, params, 0, q, k, v, *phi, g, bl, S_gpu, 1, out, ent, ws) == G.HYB_OK
        torch.cuda.synchronize()
        assert G.hyb_attn_get_device_status(ws) in (G.HYB_OK, G.HYB_WARN_NONFINITE)
        got = out.double().cpu().numpy()
        for b in range(w.B):
            for h in range(w.H):
                lo = _oracle_mask(e_gpu[b, h], tau, w.T, pos, votes_min, 1 - 1e-5)
                hi = _oracle_mask(e_gpu[b, h], tau, w.T, pos, votes_min, 1 + 1e-5)
                oi = R.block_sparse_attention(q64[b, :, h], k64[b, :, h], v64[b, :, h], sc, hi, BLOCK)
                qf = oracle.feature_map(q64[b, :, h], phi64[0][h])
                ref = oi + oracle.inter_frame_read(qf, S_ref[b, h])
                for qb in range(hi.shape[0]):
                    total += 1
                    if not np.array_equal(lo[qb], hi[qb]):
                        skipped += 1
                        continue
                    kept += int(hi[qb].sum())
                    rows = slice(qb * BLOCK, min(w.T, (qb + 1) * BLOCK))
                    tol.check(tol.scaled_errors(got[b, rows, h], ref[rows]), tol.OUT_BF16,
                              f"frame {n} b {b} h {h} query block {qb}")
        # the state update is the dense layer's
        _, _, _, S_ref = oracle.layer_pass(q64, k64, v64, *phi64, g64, bl64, S_ref, True)
        Sg = S_gpu.double().cpu().numpy()
        assert max(tol.rel_frobenius(Sg[b, hh], S_ref[b, hh]) for b in range(w.B) for hh in range(w.H)) <= \
            tol.STATE_BF16
    assert skipped <= max(1, total // 20), (skipped, total)
    return kept, total


def test_tra_480p_grid():
    """30 x 52 patches (480p), tiles of 8 x 16, tau 0.15, two votes."""
    w = W.small_workload(W.WORKLOADS[1], H=4)
    kept, total = _run(w, 0.15, 2, (30, 52), (8, 16))
    nb = math.ceil(w.T / BLOCK)
    print("retained key blocks", kept / (total * nb))
    assert kept < total * nb        # some blocks were pruned


def test_tra_small_radius_keeps_own_block_only():
    w = W.small_workload(W.WORKLOADS[1], H=2, T=24 * 20)
    _run(w, 1e-6, 1, (24, 20), (8, 16), frames=1)


def test_tra_huge_budget_is_the_dense_layer():
    import gated_delta_linear_b200 as G
    w = W.small_workload(W.WORKLOADS[1], H=2, T=17 * 19, frames=1)
    G_, params, desc, phi, ws, ent = _setup(w, 1e6, 1, (17, 19), (4, 8))
    x = W.pass_inputs(w, 0, 0)
    q, k, v, g, bl = (t.cuda() for t in (x.q, x.k, x.v, x.gate_logits, x.beta_logits))
    S1 = torch.zeros(w.B, w.H, w.d, w.d, dtype=torch.float32, device="cuda")
    S2 = S1.clone()
    assert G.hyb_tra_forward(desc, params, 1, q, k, v, *phi, g, bl, S1, 0, torch.empty_like(q), ent, ws) == G.HYB_OK
    o1 = torch.empty_like(q)
    assert G.hyb_tra_forward(desc, params, 0, q, k, v, *phi, g, bl, S1, 1, o1, ent, ws) == G.HYB_OK
    ws2 = torch.zeros(G.hyb_attn_workspace_bytes(desc), dtype=torch.uint8, device="cuda")
    o2 = torch.empty_like(q)
    assert G.hyb_attn_forward(desc, q, k, v, *phi, g, bl, S2, 1, o2, ws2) == G.HYB_OK
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(S1, S2)


def test_tra_sparse_pass_before_any_warmup_is_dense():
    """No mask built on a fresh workspace: the block-sparse pass is the dense pass."""
    import gated_delta_linear_b200 as G
    w = W.small_workload(W.WORKLOADS[1], H=3, T=30 * 52, frames=1)
    G_, params, desc, phi, ws, ent = _setup(w, 0.15, 2, (30, 52), (8, 16))
    x = W.pass_inputs(w, 0, 0)
    q, k, v, g, bl = (t.cuda() for t in (x.q, x.k, x.v, x.gate_logits, x.beta_logits))
    S1 = torch.randn(w.B, w.H, w.d, w.d, dtype=torch.float32, device="cuda")
    S2 = S1.clone()
    o1 = torch.empty_like(q)
    assert G.hyb_tra_forward(desc, params, 0, q, k, v, *phi, g, bl, S1, 1, o1, ent, ws) == G.HYB_OK
    ws2 = torch.zeros(G.hyb_attn_workspace_bytes(desc), dtype=torch.uint8, device="cuda")
    o2 = torch.empty_like(q)
    assert G.hyb_attn_forward(desc, q, k, v, *phi, g, bl, S2, 1, o2, ws2) == G.HYB_OK
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(S1, S2)
