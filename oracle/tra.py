"""Float64 CPU oracle of Token Radius Attention (TRA) applied to the
intra-frame branch.

TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only ``tests/``,
``__graft_entry__.smoke()`` and ``bench.py`` (its CPU-baseline and reference
legs) may import this module.  The CUDA library never calls it, and it never
calls the CUDA library.

Source: "Technical summary: Token Radius Attention" (gist.science/ar/paper/
2608.02504), §2 (methodology): a dense warm-up pass gives every query its
attention entropy; the entropy maps to a per-token budget
``B_i ~ tau exp(H_i) / N`` (a retained density); the budget becomes a spatial
radius around the query, shrunk on other frames by ``exp(-gamma delta)``; the
token-radius masks are turned into a regular block-sparse mask over a
tile-major token order by distance tests, radius comparison, block pruning and
token voting; attention then runs block-sparse.

Readings taken where the page leaves a step open (each is also stated in the
library's API header):

* entropy: ``H_i = -sum_j p_ij ln p_ij`` of the dense softmax row of query i
  over the tokens of its frame (natural log);
* budget: the number of keys ``k_i = clamp(tau exp(H_i), 1, T)``, i.e. the
  page's density ``tau exp(H_i) / N`` times the N = T keys of the frame;
* radius: the disk of ``k_i`` patches, ``r_i = sqrt(k_i / pi)``, in patch units
  on the frame's 2D patch grid; the intra-frame branch attends within the
  current frame only, where the temporal decay ``exp(-gamma * 0)`` is 1;
* tile-major order: tokens ordered tile after tile (tiles of th x tw patches,
  tiles row-major over the grid, patches row-major inside a tile; edge tiles are
  cut by the grid), and blocks are runs of ``block`` consecutive tokens of that
  order;
* voting: query i votes for key block K if some key of K lies within
  distance r_i of it (Euclidean on patch coordinates); key block K is kept for
  query block Q if at least ``votes_min`` of Q's queries vote for it, and a
  block is always kept for itself;
* attention: the original softmax attention of each query over the keys of the
  key blocks kept for its query block (the block-sparse result, not the
  token-level disk).

Everything is float64 NumPy with explicit loops or library matrix products.
"""

from __future__ import annotations

import numpy as np

__all__ = [
    "attention_entropy",
    "token_budget",
    "token_radius",
    "tile_major_positions",
    "block_votes",
    "block_mask",
    "block_sparse_attention",
]


def attention_entropy(q, k, sm_scale):
    """Entropy (nats) of each query's dense softmax row over the frame's keys.

    TRA summary §2, "entropy to budget": computed during the dense warm-up.
    q, k: [T, d] of one head.  Returns [T].
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    s = (q @ k.T) * sm_scale
    s = s - s.max(axis=1, keepdims=True)
    p = np.exp(s)
    p = p / p.sum(axis=1, keepdims=True)
    with np.errstate(divide="ignore", invalid="ignore"):
        plogp = np.where(p > 0, p * np.log(p), 0.0)
    return -plogp.sum(axis=1)


def token_budget(entropy, tau, T):
    """Keys kept per query: ``clamp(tau exp(H), 1, T)`` (TRA summary §2, the
    entropy-to-budget map ``B ~ tau exp(H) / N`` as a density, times N = T)."""
    return np.clip(tau * np.exp(np.asarray(entropy, dtype=np.float64)), 1.0, float(T))


def token_radius(budget):
    """Radius of the disk of ``budget`` patches: ``sqrt(budget / pi)`` (TRA
    summary §2, "budget to radius")."""
    return np.sqrt(np.asarray(budget, dtype=np.float64) / np.pi)


def tile_major_positions(grid_h, grid_w, tile_h, tile_w):
    """(row, col) of every token of a grid_h x grid_w frame in tile-major order
    (TRA summary §2, "tile-major layout"): tiles of tile_h x tile_w patches taken
    row-major over the grid, patches row-major inside each tile, edge tiles cut by
    the grid.  Returns an int array [grid_h * grid_w, 2]."""
    pos = []
    for t0 in range(0, grid_h, tile_h):
        for c0 in range(0, grid_w, tile_w):
            for r in range(t0, min(grid_h, t0 + tile_h)):
                for c in range(c0, min(grid_w, c0 + tile_w)):
                    pos.append((r, c))
    return np.array(pos, dtype=np.int64)


def block_votes(pos, radius, block):
    """votes[Q, K]: the number of queries of block Q that have at least one key
    of block K within their radius (distance on patch coordinates).  A plain
    double loop over queries and key blocks."""
    pos = np.asarray(pos, dtype=np.float64)
    T = pos.shape[0]
    nb = (T + block - 1) // block
    votes = np.zeros((nb, nb), dtype=np.int64)
    for i in range(T):
        qb = i // block
        for kb in range(nb):
            keys = pos[kb * block:min(T, (kb + 1) * block)]
            d2 = ((keys - pos[i]) ** 2).sum(axis=1)
            if np.any(d2 <= radius[i] ** 2):
                votes[qb, kb] += 1
    return votes


def block_mask(votes, votes_min):
    """Kept key blocks per query block: at least ``votes_min`` votes, and the
    block itself always (TRA summary §2, block pruning and token voting)."""
    keep = np.asarray(votes) >= votes_min
    np.fill_diagonal(keep, True)
    return keep


def block_sparse_attention(q, k, v, sm_scale, keep, block):
    """Softmax attention of each query over the keys of the blocks kept for its
    query block (TRA summary §2: the block-sparse mask replaces the dense one).
    q, k, v: [T, d]; keep: [nb, nb] bool.  Returns [T, d]."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    T = q.shape[0]
    out = np.empty_like(q)
    for qb in range(keep.shape[0]):
        rows = slice(qb * block, min(T, (qb + 1) * block))
        cols = np.concatenate([np.arange(kb * block, min(T, (kb + 1) * block))
                               for kb in range(keep.shape[1]) if keep[qb, kb]])
        s = (q[rows] @ k[cols].T) * sm_scale
        s = s - s.max(axis=1, keepdims=True)
        p = np.exp(s)
        out[rows] = (p / p.sum(axis=1, keepdims=True)) @ v[cols]
    return out
