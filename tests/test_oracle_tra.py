"""Pins of the Token Radius Attention oracle (oracle/tra.py; "Technical
summary: Token Radius Attention" §2, with the readings stated in the module),
each against something other than the oracle's own formula, and planted
mistakes the pins must catch."""

import math

import numpy as np
import pytest
import torch

from oracle import tra as R


def _qkv(seed, T, d=8):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((T, d)) for _ in range(3))


def pin_entropy_closed_forms():
    # uniform scores: H = ln T; two keys with scores (0, s): the binary entropy
    T, d = 37, 4
    q = np.zeros((3, d))
    k = np.random.default_rng(1).standard_normal((T, d))
    np.testing.assert_allclose(R.attention_entropy(q, k, 1.0), math.log(T), rtol=1e-12)
    s = 1.7
    q2 = np.array([[1.0, 0.0]])
    k2 = np.array([[0.0, 0.0], [s, 0.0]])
    p1 = math.exp(s) / (1 + math.exp(s))
    h = -(p1 * math.log(p1) + (1 - p1) * math.log(1 - p1))
    np.testing.assert_allclose(R.attention_entropy(q2, k2, 1.0), h, rtol=1e-12)


def pin_budget_and_radius_closed_forms():
    # tau exp(H) = 9 pi keys -> a disk of radius 3; clamped to [1, T]
    H = np.array([math.log(9 * math.pi), -50.0, 50.0])
    b = R.token_budget(H, 1.0, 100)
    np.testing.assert_allclose(b, [9 * math.pi, 1.0, 100.0], rtol=1e-12)
    np.testing.assert_allclose(R.token_radius(b[:1]), [3.0], rtol=1e-12)
    np.testing.assert_allclose(R.token_budget(np.array([0.0]), 0.25, 10), [1.0])  # 0.25 -> clamped


def pin_tile_major_order_by_hand():
    # a 3 x 5 grid in 2 x 2 tiles: tiles (0,0) (0,1) (0,2) (1,0) (1,1) (1,2), edges cut
    got = [tuple(p) for p in R.tile_major_positions(3, 5, 2, 2)]
    want = [(0, 0), (0, 1), (1, 0), (1, 1), (0, 2), (0, 3), (1, 2), (1, 3), (0, 4), (1, 4),
            (2, 0), (2, 1), (2, 2), (2, 3), (2, 4)]
    assert got == want
    # the order is a bijection onto the grid for the 480p shape
    p = R.tile_major_positions(30, 52, 8, 16)
    assert len({tuple(x) for x in p}) == 30 * 52 == len(p)


def pin_voting_on_a_line_by_hand():
    # one row of 10 patches, blocks of 4: [0..3] [4..7] [8, 9]; radius 1.5 for
    # every query reaches its neighbours within distance 1
    pos = R.tile_major_positions(1, 10, 1, 10)
    v = R.block_votes(pos, np.full(10, 1.5), 4)
    # block 0: queries 0..3 reach block 1 only from query 3 (3 -> 4)
    # block 1: queries 4..7; 4 reaches block 0 (4 -> 3), 7 reaches block 2 (7 -> 8)
    # block 2: queries 8, 9; 8 reaches block 1 (8 -> 7)
    np.testing.assert_array_equal(v, [[4, 1, 0], [1, 4, 1], [0, 1, 2]])
    np.testing.assert_array_equal(R.block_mask(v, 2), np.eye(3, dtype=bool))
    np.testing.assert_array_equal(R.block_mask(v, 1), [[1, 1, 0], [1, 1, 1], [0, 1, 1]])
    # more votes than a block has queries: only the block itself is kept
    np.testing.assert_array_equal(R.block_mask(v, 5), np.eye(3, dtype=bool))
    # a key exactly on the radius counts (distance 1, radius 1)
    np.testing.assert_array_equal(R.block_votes(pos, np.full(10, 1.0), 4), v)


def pin_radius_limits():
    pos = R.tile_major_positions(6, 9, 2, 4)
    T = len(pos)
    big = R.block_votes(pos, np.full(T, 100.0), 8)
    sizes = np.array([min(8, T - 8 * b) for b in range(big.shape[0])])
    np.testing.assert_array_equal(big, np.repeat(sizes[:, None], big.shape[1], 1))  # every query votes everywhere
    assert R.block_mask(big, 1).all()
    small = R.block_votes(pos, np.full(T, 0.5), 8)
    np.testing.assert_array_equal(R.block_mask(small, 1), np.eye(small.shape[0], dtype=bool))


def pin_block_sparse_equals_sdpa():
    T, blk = 23, 8
    q, k, v = _qkv(3, T)
    nb = (T + blk - 1) // blk
    sc = 1 / math.sqrt(q.shape[1])
    t = lambda x: torch.from_numpy(x)[None, None]
    dense = torch.nn.functional.scaled_dot_product_attention(t(q), t(k), t(v), scale=sc)[0, 0].numpy()
    np.testing.assert_allclose(R.block_sparse_attention(q, k, v, sc, np.ones((nb, nb), bool), blk), dense,
                               rtol=1e-10, atol=1e-12)
    # a keep pattern as a boolean SDPA mask over tokens
    keep = np.array([[1, 0, 1], [0, 1, 0], [1, 1, 1]], bool)
    tok = np.repeat(np.repeat(keep, blk, 0), blk, 1)[:T, :T]
    masked = torch.nn.functional.scaled_dot_product_attention(t(q), t(k), t(v), attn_mask=torch.from_numpy(tok),
                                                              scale=sc)[0, 0].numpy()
    np.testing.assert_allclose(R.block_sparse_attention(q, k, v, sc, keep, blk), masked, rtol=1e-10, atol=1e-12)


def pin_large_tau_is_dense_attention():
    # a budget of every key gives a radius past the grid: TRA reduces to the dense layer
    gh, gw, blk = 5, 7, 8
    T = gh * gw
    q, k, v = _qkv(4, T)
    sc = 1 / math.sqrt(q.shape[1])
    H = R.attention_entropy(q, k, sc)
    r = R.token_radius(R.token_budget(H, 1e6, T))
    keep = R.block_mask(R.block_votes(R.tile_major_positions(gh, gw, 2, 4), r, blk), 1)
    assert keep.all()
    t = lambda x: torch.from_numpy(x)[None, None]
    dense = torch.nn.functional.scaled_dot_product_attention(t(q), t(k), t(v), scale=sc)[0, 0].numpy()
    np.testing.assert_allclose(R.block_sparse_attention(q, k, v, sc, keep, blk), dense, rtol=1e-10, atol=1e-12)


PINS = [pin_entropy_closed_forms, pin_budget_and_radius_closed_forms, pin_tile_major_order_by_hand,
        pin_voting_on_a_line_by_hand, pin_radius_limits, pin_block_sparse_equals_sdpa,
        pin_large_tau_is_dense_attention]


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin()


def _mutants():
    def entropy_log2(q, k, sm_scale):
        s = (np.asarray(q) @ np.asarray(k).T) * sm_scale
        p = np.exp(s - s.max(1, keepdims=True))
        p /= p.sum(1, keepdims=True)
        return -(p * np.log2(np.where(p > 0, p, 1))).sum(1)

    def radius_no_pi(budget):
        return np.sqrt(np.asarray(budget, dtype=np.float64))

    def col_major_tiles(gh, gw, th, tw):
        pos = []
        for t0 in range(0, gh, th):
            for c0 in range(0, gw, tw):
                for c in range(c0, min(gw, c0 + tw)):
                    for r in range(t0, min(gh, t0 + th)):
                        pos.append((r, c))
        return np.array(pos, dtype=np.int64)

    def mask_without_diagonal(votes, votes_min):
        return np.asarray(votes) >= votes_min

    def votes_strict(pos, radius, block):
        pos = np.asarray(pos, dtype=np.float64)
        T = pos.shape[0]
        nb = (T + block - 1) // block
        out = np.zeros((nb, nb), dtype=np.int64)
        for i in range(T):
            for kb in range(nb):
                keys = pos[kb * block:min(T, (kb + 1) * block)]
                if np.any(((keys - pos[i]) ** 2).sum(1) < radius[i] ** 2):
                    out[i // block, kb] += 1
        return out

    return {"attention_entropy": entropy_log2, "token_radius": radius_no_pi,
            "tile_major_positions": col_major_tiles, "block_mask": mask_without_diagonal,
            "block_votes": votes_strict}


@pytest.mark.parametrize("name", sorted(_mutants()))
def test_planted_mistakes_are_caught(name, monkeypatch):
    monkeypatch.setattr(R, name, _mutants()[name])
    caught = 0
    for pin in PINS:
        try:
            pin()
        except AssertionError:
            caught += 1
    assert caught >= 1, f"no pin caught the planted mistake in {name}"
