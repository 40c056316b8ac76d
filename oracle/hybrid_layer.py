"""Float64 CPU oracle of the ARL2 hybrid attention layer.

TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only ``tests/``,
``__graft_entry__.smoke()`` and ``bench.py`` (its CPU-baseline and reference
legs) may import this module.  The CUDA library never calls it, and it never
calls the CUDA library.

What it computes, per batch element b, head h and pass of frame N
(source: "Technical summary: Attend Locally, Remember Linearly (ARL2)",
gist.science/ar/paper/2605.16579):

* §2.1, intra-frame branch: the original bidirectional softmax attention,
  restricted to the tokens of the current frame,
  ``O_intra = softmax(Q K^T / sqrt(d)) V``.
* §2.1, inter-frame branch: per-head 1x1 feature maps phi_q, phi_k, phi_v
  adapt Q, K, V; the output is ``O_inter = Q' S_{N-1}``.
* §2.1, state update (printed garbled; read as the only shape-consistent
  form): ``S_N = alpha_N S_{N-1} + K'^T diag(beta_N) (V' - K' S_{N-1})``,
  with K' the L2-normalised feature-mapped keys, beta a per-token sigmoid and
  alpha the frame mean of the per-token sigmoid forget gate (headwise gating,
  §4 ablations).
* §2.2, frame-level access: every token of frame N reads the same
  pre-update S_{N-1}.  Clean-pass updates: denoising passes read S and never
  write it; the final clean pass of a frame writes S once, after the reads.
* Layer output: the pages do not say how the two branches combine; this
  oracle takes the plain sum ``O = O_intra + O_inter``.

Readings taken where the pages are silent (all also stated in the library's
API header): the 1x1 feature map acts as ``x'[o] = sum_i phi[o, i] x[i]``
(so ``X' = X phi^T``), with no bias and no nonlinearity; only K' is
L2-normalised, as ``k / sqrt(sum k^2 + eps)``; the softmax scale is
``1/sqrt(d_k)``; alpha is ``mean_t sigmoid(g_t)``, not ``sigmoid(mean_t g_t)``.

Everything is NumPy float64, one (b, h) at a time, with library matrix
products as the only primitive; there is no blocking, fusion or reordering.
"""

from __future__ import annotations

import numpy as np

__all__ = [
    "sigmoid",
    "feature_map",
    "l2_normalise_rows",
    "intra_frame_attention",
    "inter_frame_read",
    "frame_gates",
    "gated_delta_update",
    "head_pass",
    "layer_pass",
    "run_frames",
]


def sigmoid(x):
    """Logistic function 1 / (1 + exp(-x)), float64.

    ARL2 summary §2.1: alpha (forget gate) and beta (learning rate) are
    learned per-token projections; the sigmoid maps their logits into (0, 1).
    """
    x = np.asarray(x, dtype=np.float64)
    return 1.0 / (1.0 + np.exp(-x))


def feature_map(x, phi):
    """Per-head grouped 1x1 feature map, ARL2 summary §2.1 ("adaptation").

    x: [T, d] tokens of one head; phi: [d, d].  A 1x1 convolution maps input
    channel i to output channel o with weight phi[o, i], so row t of the
    result is ``phi @ x[t]`` and the whole map is ``x @ phi^T``.
    """
    x = np.asarray(x, dtype=np.float64)
    phi = np.asarray(phi, dtype=np.float64)
    return x @ phi.T


def l2_normalise_rows(x, eps):
    """Row-wise L2 normalisation ``x / sqrt(sum x^2 + eps)``.

    The pages do not state it; the layer's specification normalises the
    feature-mapped keys K' so that each token writes a unit-norm key, as in
    the gated delta rule (GDN) that §2.1 names.
    """
    x = np.asarray(x, dtype=np.float64)
    return x / np.sqrt(np.sum(x * x, axis=1, keepdims=True) + eps)


def intra_frame_attention(q, k, v, sm_scale):
    """Bidirectional softmax attention over the tokens of one frame.

    ARL2 summary §2.1, intra-frame branch ("attend locally"): the original
    softmax attention, kept bidirectional within the frame; all tokens of the
    frame are decoded together, so there is no causal mask.
    q, k, v: [T, d] of one head.  Returns [T, d].
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    scores = (q @ k.T) * sm_scale
    scores = scores - scores.max(axis=1, keepdims=True)
    weights = np.exp(scores)
    weights = weights / weights.sum(axis=1, keepdims=True)
    return weights @ v


def inter_frame_read(q_feat, state):
    """Inter-frame readout ``O_inter = Q' S_{N-1}``, ARL2 summary §2.1 ("outputs").

    q_feat: [T, d_k] feature-mapped queries; state: [d_k, d_v].
    §2.2 frame-level access: every token reads the same pre-update state.
    """
    return np.asarray(q_feat, dtype=np.float64) @ np.asarray(state, dtype=np.float64)


def frame_gates(gate_logits, beta_logits):
    """Gates of one head for one frame.

    ARL2 summary §2.1 (state update) and §4 (headwise gating): beta_t =
    sigmoid(beta logit) per token; the forget gate is reduced to one scalar per
    head and frame as the mean over the frame's tokens of the per-token
    sigmoid.  gate_logits, beta_logits: [T].  Returns (alpha, beta[T]).
    """
    alpha = float(np.mean(sigmoid(gate_logits)))
    beta = sigmoid(beta_logits)
    return alpha, beta


def gated_delta_update(state, k_unit, v_feat, beta, alpha):
    """Frame-level gated delta rule, ARL2 summary §2.1 ("state update").

    ``S_N = alpha S_{N-1} + K'^T diag(beta) (V' - K' S_{N-1})``.
    state: [d_k, d_v] (the pre-update S_{N-1}, not modified); k_unit: [T, d_k]
    L2-normalised feature-mapped keys; v_feat: [T, d_v]; beta: [T]; alpha:
    scalar.  Returns a new array S_N.
    """
    state = np.asarray(state, dtype=np.float64)
    residual = v_feat - k_unit @ state
    return alpha * state + k_unit.T @ (beta[:, None] * residual)


def head_pass(q, k, v, phi_q, phi_k, phi_v, gate_logits, beta_logits, state,
              clean_pass, sm_scale=None, l2_eps=1e-6):
    """One pass of one (batch, head) pair through the hybrid layer.

    q, k, v: [T, d]; phi_*: [d, d]; gate_logits, beta_logits: [T] (used only
    when clean_pass); state: [d, d], read-only here.
    Returns (out, out_intra, out_inter, new_state); new_state is ``state``
    itself (the same object, untouched) on a query-only pass, per ARL2 summary
    §2.2 ("clean-pass updates").
    """
    d = q.shape[1]
    if sm_scale is None:
        sm_scale = 1.0 / np.sqrt(d)
    out_intra = intra_frame_attention(q, k, v, sm_scale)
    out_inter = inter_frame_read(feature_map(q, phi_q), state)
    out = out_intra + out_inter
    if not clean_pass:
        return out, out_intra, out_inter, state
    k_unit = l2_normalise_rows(feature_map(k, phi_k), l2_eps)
    v_feat = feature_map(v, phi_v)
    alpha, beta = frame_gates(gate_logits, beta_logits)
    new_state = gated_delta_update(state, k_unit, v_feat, beta, alpha)
    return out, out_intra, out_inter, new_state


def layer_pass(q, k, v, phi_q, phi_k, phi_v, gate_logits, beta_logits, state,
               clean_pass, sm_scale=None, l2_eps=1e-6, heads=None):
    """One pass of the whole layer, looping over (batch, head) pairs.

    Layouts (the library's): q, k, v, out: [B, T, H, d]; phi_*: [H, d, d];
    gate_logits, beta_logits: [B, H, T]; state: [B, H, d_k, d_v].
    ``heads``: optional list of (b, h) pairs to evaluate (others are left as
    NaN in the outputs and carried unchanged in the state), so that large
    configurations can be checked on sampled heads.
    Returns (out, out_intra, out_inter, new_state); ``state`` is never written.
    """
    B, T, H, d = q.shape
    out = np.full((B, T, H, state.shape[3]), np.nan)
    out_intra = np.full_like(out, np.nan)
    out_inter = np.full_like(out, np.nan)
    new_state = state if not clean_pass else np.array(state, dtype=np.float64, copy=True)
    pairs = heads if heads is not None else [(b, h) for b in range(B) for h in range(H)]
    for b, h in pairs:
        g = gate_logits[b, h] if clean_pass else None
        bl = beta_logits[b, h] if clean_pass else None
        o, oi, oe, s_new = head_pass(q[b, :, h, :], k[b, :, h, :], v[b, :, h, :],
                                     phi_q[h], phi_k[h], phi_v[h], g, bl, state[b, h],
                                     clean_pass, sm_scale, l2_eps)
        out[b, :, h, :] = o
        out_intra[b, :, h, :] = oi
        out_inter[b, :, h, :] = oe
        if clean_pass:
            new_state[b, h] = s_new
    return out, out_intra, out_inter, new_state


def run_frames(frame_source, phi_q, phi_k, phi_v, state0, n_frames, passes,
               sm_scale=None, l2_eps=1e-6, heads=None, on_pass=None):
    """Autoregressive frame loop over a persistent state (ARL2 summary §2.2).

    frame_source(frame, pass_index) -> (q, k, v, gate_logits, beta_logits).
    ``passes`` is a sequence of booleans, one per pass of every frame
    (False = query-only denoising pass, True = clean pass).  Only the state is
    carried between frames, so memory does not grow with the frame count.
    ``on_pass(frame, pass_index, out, out_intra, out_inter, state_before,
    state_after)`` receives each pass's results.  Returns the final state.
    """
    state = np.array(state0, dtype=np.float64, copy=True)
    for n in range(n_frames):
        for p, clean in enumerate(passes):
            q, k, v, g, bl = frame_source(n, p)
            out, oi, oe, new_state = layer_pass(q, k, v, phi_q, phi_k, phi_v, g, bl, state,
                                                clean, sm_scale, l2_eps, heads)
            if on_pass is not None:
                on_pass(n, p, out, oi, oe, state, new_state)
            state = new_state
    return state


def kvcache_attention(q, k_frames, v_frames, sm_scale):
    """The softmax baseline with a key/value cache, for one frame of one head.

    ARL2 summary §1 (problem statement): the softmax attention of an
    autoregressive video DiT keeps the keys and values of every generated chunk
    in a cache that grows linearly with the video; §4 compares the hybrid layer's
    memory and wall-clock time against it.  The queries of frame N attend,
    with one softmax, over the keys of frames 0..N (bidirectional within frame
    N, no mask): the cache is the frames' keys and values stacked in order.
    q: [T, d] of frame N; k_frames, v_frames: sequences of [T_f, d] for frames
    0..N.  Returns [T, d].
    """
    k = np.concatenate([np.asarray(x, dtype=np.float64) for x in k_frames], axis=0)
    v = np.concatenate([np.asarray(x, dtype=np.float64) for x in v_frames], axis=0)
    q = np.asarray(q, dtype=np.float64)
    scores = (q @ k.T) * sm_scale
    scores = scores - scores.max(axis=1, keepdims=True)
    weights = np.exp(scores)
    weights = weights / weights.sum(axis=1, keepdims=True)
    return weights @ v


def mixed_output(o_intra, o_inter, a, c):
    """Weighted combination of the two branches, ``a O_intra + c O_inter``.

    The adjacent methods combine a softmax-type branch with a linear one by a
    scalar: "LinVideo: A Post-Training Framework towards O(n) Attention in
    Efficient Video Generation" §2(b) mixes ``r SoftmaxAttn + (1 - r)
    LinearAttn`` (a = r, c = 1 - r); "SALAD: Achieve High-Sparsity Attention via
    Efficient Linear Attention Tuning for Video Diffusion Transformer" §2 scales
    the linear branch by a static gain or a sigmoid-bounded factor (a = 1).
    a, c: scalars of one (batch, head); o_intra, o_inter: [T, d].
    """
    return a * np.asarray(o_intra, dtype=np.float64) + c * np.asarray(o_inter, dtype=np.float64)


def token_level_head_pass(q, k, v, phi_q, phi_k, phi_v, gate_logits, beta_logits, state,
                          clean_pass, sm_scale=None, l2_eps=1e-6):
    """The token-level access variant of one pass of one (batch, head) pair.

    ARL2 summary §4 (ablations) compares the layer's frame-level access with a
    token-level one.  The pages give no formulas for it; the readings taken:
    on a clean pass the tokens of the frame update the state one after another
    by the single-token gated delta rule with a per-token forget gate (§2.1
    calls the forget gate a per-token projection),

        S <- alpha_t S + beta_t k'_t (v'_t^T - k'_t^T S),
        alpha_t = sigmoid(g_t), beta_t = sigmoid(beta_logit_t),

    and token t reads the state before its own update, O_inter[t] = q'_t S
    (causal within the frame, the analogue of the frame-level rule's read of
    S_{N-1}).  The residual v'_t - k'_t^T S is taken against the undecayed
    state, exactly as in the frame-level rule of §2.1 (so a one-token frame
    gives the same update under both accesses).  This is a reading, not the
    form of "Gated Delta Networks", whose rule S <- alpha S (I - beta k k^T) +
    beta v k^T decays the state inside the residual; the two differ whenever
    alpha_t < 1.  A query-only pass updates nothing, so every token reads the
    frame-start state, as in the frame-level layer.  The intra-frame branch
    and the combination out = O_intra + O_inter are unchanged.
    q, k, v: [T, d]; phi_*: [d, d]; gate_logits, beta_logits: [T]; state:
    [d, d] (not modified).  Returns (out, out_intra, out_inter, new_state).
    """
    d = q.shape[1]
    if sm_scale is None:
        sm_scale = 1.0 / np.sqrt(d)
    out_intra = intra_frame_attention(q, k, v, sm_scale)
    q_feat = feature_map(q, phi_q)
    if not clean_pass:
        out_inter = inter_frame_read(q_feat, state)
        return out_intra + out_inter, out_intra, out_inter, state
    k_unit = l2_normalise_rows(feature_map(k, phi_k), l2_eps)
    v_feat = feature_map(v, phi_v)
    alpha = sigmoid(np.asarray(gate_logits, dtype=np.float64))
    beta = sigmoid(np.asarray(beta_logits, dtype=np.float64))
    S = np.array(state, dtype=np.float64, copy=True)
    out_inter = np.empty_like(q_feat)
    for t in range(q.shape[0]):
        out_inter[t] = q_feat[t] @ S
        kt = k_unit[t]
        S = alpha[t] * S + beta[t] * np.outer(kt, v_feat[t] - kt @ S)
    return out_intra + out_inter, out_intra, out_inter, S
