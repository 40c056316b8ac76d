"""Pins of the CPU oracle to facts fixed outside the oracle itself.

Each pin checks the oracle against something it does not compute itself: a
library routine (PyTorch's scaled-dot-product attention), a hand-derived
worked example under tests/golden/, a closed form, an invariant of the gated
delta rule, or a brute-force token loop.  ``test_planted_mistakes_are_caught``
then plants plausible mistakes in the oracle (on the CPU) and checks that at
least one pin fails for each.

Source of the method: "Technical summary: Attend Locally, Remember Linearly
(ARL2)", gist.science/ar/paper/2605.16579, §2.1 and §2.2.
"""

import json
import math
import os
import tracemalloc

import numpy as np
import pytest
import torch

from oracle import hybrid_layer as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
INF = float("inf")


def _rng(seed):
    return np.random.default_rng(seed)


def _eye_phi(d):
    return np.eye(d)


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _arr(x):
    return np.asarray(x, dtype=np.float64)


# --------------------------------------------------------------------------- pins

def pin_intra_matches_library_sdpa():
    """§2.1 intra-frame branch == full softmax attention with a block-diagonal
    per-frame mask, computed by torch's SDPA (float64, default 1/sqrt(d) scale)."""
    rng = _rng(1)
    d, lens = 8, (5, 7, 1, 4)
    L = sum(lens)
    q, k, v = (rng.standard_normal((L, d)) * 1.5 for _ in range(3))
    mask = torch.zeros(L, L, dtype=torch.bool)
    s = 0
    for n in lens:
        mask[s:s + n, s:s + n] = True
        s += n
    t = lambda a: torch.from_numpy(a)[None, None]
    ref = torch.nn.functional.scaled_dot_product_attention(t(q), t(k), t(v), attn_mask=mask)[0, 0].numpy()
    got = np.zeros_like(ref)
    s = 0
    for n in lens:
        got[s:s + n] = O.intra_frame_attention(q[s:s + n], k[s:s + n], v[s:s + n], 1.0 / math.sqrt(d))
        s += n
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


def pin_intra_special_cases():
    """T = 1 returns v; identical keys give the mean of v; a key far ahead of
    the others (score gap >> 1) selects its value (softmax limit)."""
    rng = _rng(2)
    d = 4
    q, k, v = (rng.standard_normal((1, d)) for _ in range(3))
    np.testing.assert_allclose(O.intra_frame_attention(q, k, v, 0.5), v, rtol=0, atol=1e-15)
    q = rng.standard_normal((3, d))
    k = np.repeat(rng.standard_normal((1, d)), 6, axis=0)
    v = rng.standard_normal((6, d))
    np.testing.assert_allclose(O.intra_frame_attention(q, k, v, 0.5),
                               np.repeat(v.mean(0, keepdims=True), 3, axis=0), rtol=1e-13, atol=1e-13)
    q = np.array([[1.0, 0.0, 0.0, 0.0]])
    k = np.array([[100.0, 0, 0, 0], [0, 1.0, 0, 0], [-3.0, 0, 0, 0]])
    v = np.array([[1.0, 2, 3, 4], [9.0, 9, 9, 9], [5.0, 5, 5, 5]])
    np.testing.assert_allclose(O.intra_frame_attention(q, k, v, 1.0), v[:1], rtol=0, atol=1e-30)
    # the scale multiplies the scores: scale 0 gives the plain mean
    q, k = rng.standard_normal((2, d)), rng.standard_normal((5, d))
    v = rng.standard_normal((5, d))
    np.testing.assert_allclose(O.intra_frame_attention(q, k, v, 0.0),
                               np.repeat(v.mean(0, keepdims=True), 2, axis=0), rtol=1e-13, atol=1e-13)


def pin_golden_single_token():
    """Hand-derived single-token GDN step (tests/golden/gdn_single_token_d2.json)."""
    g = _load("gdn_single_token_d2.json")
    out, oi, oe, s1 = O.head_pass(_arr(g["q"]), _arr(g["k"]), _arr(g["v"]), _arr(g["phi_q"]),
                                  _arr(g["phi_k"]), _arr(g["phi_v"]), _arr(g["gate_logits"]),
                                  _arr(g["beta_logits"]), _arr(g["state0"]), True,
                                  l2_eps=g["l2_eps"])
    np.testing.assert_allclose(s1, _arr(g["expected_state1"]), rtol=0, atol=1e-15)
    np.testing.assert_allclose(out, _arr(g["expected_out"]), rtol=0, atol=1e-15)
    np.testing.assert_allclose(oe, _arr(g["expected_out_inter"]), rtol=0, atol=1e-15)
    np.testing.assert_allclose(oi, _arr(g["expected_out_intra"]), rtol=0, atol=1e-15)


def pin_golden_two_tokens_feature_maps():
    """Hand-derived two-token frame update with non-symmetric phi maps
    (tests/golden/frame_update_two_tokens_d2.json): pins the 1x1-map
    orientation, the residual's sign and the transpose of K'."""
    g = _load("frame_update_two_tokens_d2.json")
    out, oi, oe, s1 = O.head_pass(_arr(g["q"]), _arr(g["k"]), _arr(g["v"]), _arr(g["phi_q"]),
                                  _arr(g["phi_k"]), _arr(g["phi_v"]), _arr(g["gate_logits"]),
                                  _arr(g["beta_logits"]), _arr(g["state0"]), True,
                                  l2_eps=g["l2_eps"])
    np.testing.assert_allclose(s1, _arr(g["expected_state1"]), rtol=0, atol=1e-14)
    np.testing.assert_allclose(oe, _arr(g["expected_out_inter"]), rtol=0, atol=1e-14)
    np.testing.assert_allclose(oi[0], _arr(g["expected_out_intra_row0"]), rtol=0, atol=1e-14)
    w = 1.0 / (1.0 + math.exp(-8.0 / math.sqrt(2.0)))
    v = _arr(g["v"])
    np.testing.assert_allclose(oi[1], (1 - w) * v[0] + w * v[1], rtol=0, atol=1e-14)
    np.testing.assert_allclose(out, oi + oe, rtol=0, atol=0)


def pin_zero_state_gives_zero_inter():
    """§2.1 O_inter = Q' S_{N-1}: with S_0 = 0, frame 0's inter output is exactly 0."""
    rng = _rng(3)
    T, d = 9, 6
    args = [rng.standard_normal((T, d)) for _ in range(3)] + \
           [np.eye(d) + 0.1 * rng.standard_normal((d, d)) for _ in range(3)]
    out, oi, oe, _ = O.head_pass(*args, rng.standard_normal(T), rng.standard_normal(T),
                                 np.zeros((d, d)), True)
    assert np.all(oe == 0.0)
    assert np.array_equal(out, oi)


def pin_state_invariance_and_forget_closed_form():
    """alpha = 1, beta = 0 keeps S exactly; beta = 0 alone scales S by the
    product of the frames' alphas; alpha is the frame mean of sigmoid(g)."""
    rng = _rng(4)
    T, d = 7, 5
    phis = [np.eye(d) + 0.1 * rng.standard_normal((d, d)) for _ in range(3)]
    S0 = rng.standard_normal((d, d))
    qkv = [rng.standard_normal((T, d)) for _ in range(3)]
    _, _, _, s1 = O.head_pass(*qkv, *phis, np.full(T, INF), np.full(T, -INF), S0, True)
    assert np.array_equal(s1, S0)
    # gate logits 0 and ln 3 give sigmoids 1/2 and 3/4: alpha = 5/8
    g = np.array([0.0, math.log(3.0)] * 3 + [0.0])
    alpha = (4 * 0.5 + 3 * 0.75) / 7
    S = S0
    for _ in range(3):
        _, _, _, S = O.head_pass(*qkv, *phis, g, np.full(T, -INF), S, True)
    np.testing.assert_allclose(S, alpha ** 3 * S0, rtol=1e-14, atol=0)
    # mean of sigmoids, not sigmoid of the mean: logits (0, 40) give alpha = 3/4
    _, _, _, s1 = O.head_pass(*[x[:2] for x in qkv], *phis, np.array([0.0, 40.0]),
                              np.full(2, -INF), S0, True)
    np.testing.assert_allclose(s1, 0.75 * S0, rtol=1e-15, atol=0)


def pin_query_only_pass_does_not_write():
    """§2.2 clean-pass updates: a query-only pass returns the state object
    untouched (bit-identical), whatever the gates."""
    rng = _rng(5)
    B, T, H, d = 2, 6, 3, 4
    q, k, v = (rng.standard_normal((B, T, H, d)) for _ in range(3))
    phis = [np.eye(d)[None].repeat(H, 0) + 0.1 * rng.standard_normal((H, d, d)) for _ in range(3)]
    S = rng.standard_normal((B, H, d, d))
    keep = S.copy()
    _, _, _, s_after = O.layer_pass(q, k, v, *phis, rng.standard_normal((B, H, T)),
                                    rng.standard_normal((B, H, T)), S, False)
    assert s_after is S
    assert np.array_equal(S, keep)
    # and a clean pass does change it without writing the input buffer
    _, _, _, s_after = O.layer_pass(q, k, v, *phis, rng.standard_normal((B, H, T)),
                                    rng.standard_normal((B, H, T)), S, True)
    assert np.array_equal(S, keep)
    assert not np.array_equal(s_after, keep)


def pin_update_equals_token_loop_bruteforce():
    """spec check: the frame-level update equals the brute-force sum over
    tokens of beta_t k'_t (v'_t - S^T k'_t)^T, written as explicit loops."""
    rng = _rng(6)
    T, d, eps = 5, 3, 1e-6
    q, k, v = (rng.standard_normal((T, d)) for _ in range(3))
    phq, phk, phv = (np.eye(d) + 0.3 * rng.standard_normal((d, d)) for _ in range(3))
    g, bl = rng.standard_normal(T), rng.standard_normal(T)
    S = rng.standard_normal((d, d))
    _, _, _, s1 = O.head_pass(q, k, v, phq, phk, phv, g, bl, S, True, l2_eps=eps)
    alpha = sum(1.0 / (1.0 + math.exp(-x)) for x in g) / T
    ref = [[alpha * S[i][j] for j in range(d)] for i in range(d)]
    for t in range(T):
        kt = [sum(phk[o][i] * k[t][i] for i in range(d)) for o in range(d)]
        nrm = math.sqrt(sum(x * x for x in kt) + eps)
        kt = [x / nrm for x in kt]
        vt = [sum(phv[o][i] * v[t][i] for i in range(d)) for o in range(d)]
        bt = 1.0 / (1.0 + math.exp(-bl[t]))
        for i in range(d):
            for j in range(d):
                read = sum(kt[m] * S[m][j] for m in range(d))
                ref[i][j] += bt * kt[i] * (vt[j] - read)
    np.testing.assert_allclose(s1, np.array(ref), rtol=1e-12, atol=1e-12)


def pin_delta_rule_stores_value():
    """Textbook property of the delta rule (GDN, §2.1): with alpha = beta = 1
    and one token, reading the new state with that token's unit key returns its
    value exactly: k'^T S_N = v'^T, whatever S_{N-1}."""
    rng = _rng(7)
    d = 6
    phk, phv = (np.eye(d) + 0.2 * rng.standard_normal((d, d)) for _ in range(2))
    k, v, q = (rng.standard_normal((1, d)) for _ in range(3))
    S = rng.standard_normal((d, d)) * 3
    _, _, _, s1 = O.head_pass(q, k, v, np.eye(d), phk, phv, np.array([INF]), np.array([INF]),
                              S, True, l2_eps=0.0)
    ku = (k @ phk.T) / np.linalg.norm(k @ phk.T)
    np.testing.assert_allclose(ku @ s1, v @ phv.T, rtol=1e-12, atol=1e-12)


def pin_orthonormal_keys_store_all_values():
    """With orthonormal unit keys (T <= d), alpha = beta = 1, the frame update
    stores every value: K' S_N = V'; it then equals the token-by-token delta
    rule applied in any order."""
    rng = _rng(8)
    T, d = 4, 6
    Qm, _ = np.linalg.qr(rng.standard_normal((d, d)))
    k = Qm[:T] * rng.uniform(0.5, 3.0, size=(T, 1))       # orthogonal, not unit
    v = rng.standard_normal((T, d))
    S = rng.standard_normal((d, d))
    I = np.eye(d)
    _, _, _, s1 = O.head_pass(v, k, v, I, I, I, np.full(T, INF), np.full(T, INF), S, True, l2_eps=0.0)
    ku = k / np.linalg.norm(k, axis=1, keepdims=True)
    np.testing.assert_allclose(ku @ s1, v, rtol=1e-12, atol=1e-12)
    for order in ([0, 1, 2, 3], [3, 1, 0, 2]):
        s_seq = S.copy()
        for t in order:
            s_seq = s_seq + np.outer(ku[t], v[t] - ku[t] @ s_seq)
        np.testing.assert_allclose(s1, s_seq, rtol=1e-12, atol=1e-12)


def pin_permutation_and_linearity():
    """Permuting a frame's tokens permutes the output rows and leaves S_N
    unchanged; with S_0 = 0, S_1 is linear in the values."""
    rng = _rng(9)
    T, d = 11, 5
    q, k, v = (rng.standard_normal((T, d)) for _ in range(3))
    phis = [np.eye(d) + 0.2 * rng.standard_normal((d, d)) for _ in range(3)]
    g, bl = rng.standard_normal(T), rng.standard_normal(T)
    S = rng.standard_normal((d, d))
    perm = rng.permutation(T)
    o1, _, _, s1 = O.head_pass(q, k, v, *phis, g, bl, S, True)
    o2, _, _, s2 = O.head_pass(q[perm], k[perm], v[perm], *phis, g[perm], bl[perm], S, True)
    np.testing.assert_allclose(o2, o1[perm], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(s2, s1, rtol=1e-12, atol=1e-12)
    Z = np.zeros((d, d))
    v2 = rng.standard_normal((T, d))
    sa = O.head_pass(q, k, v, *phis, g, bl, Z, True)[3]
    sb = O.head_pass(q, k, v2, *phis, g, bl, Z, True)[3]
    sc = O.head_pass(q, k, 2.0 * v - 3.0 * v2, *phis, g, bl, Z, True)[3]
    np.testing.assert_allclose(sc, 2.0 * sa - 3.0 * sb, rtol=1e-12, atol=1e-12)


def pin_feature_map_orientation_and_key_scale():
    """A 1x1 map with phi[o][i] = 1 iff i = pi(o) routes input channel pi(o)
    to output o; phi = I is the identity; scaling the raw keys by c > 0 does
    not change S_N (K' is L2-normalised)."""
    rng = _rng(10)
    T, d = 3, 5
    pi = np.array([2, 0, 4, 1, 3])
    P = np.zeros((d, d))
    P[np.arange(d), pi] = 1.0
    x = rng.standard_normal((T, d))
    np.testing.assert_array_equal(O.feature_map(x, P), x[:, pi])
    np.testing.assert_array_equal(O.feature_map(x, np.eye(d)), x)
    # the inter read uses the mapped queries: with S = I it returns x[:, pi]
    q = x
    out, _, oe, _ = O.head_pass(q, q, q, P, np.eye(d), np.eye(d), None, None, np.eye(d), False)
    np.testing.assert_allclose(oe, x[:, pi], rtol=0, atol=0)
    k, v = rng.standard_normal((T, d)), rng.standard_normal((T, d))
    g, bl = rng.standard_normal(T), rng.standard_normal(T)
    S = rng.standard_normal((d, d))
    s_a = O.head_pass(q, k, v, P, P, P, g, bl, S, True, l2_eps=0.0)[3]
    s_b = O.head_pass(q, 7.5 * k, v, P, P, P, g, bl, S, True, l2_eps=0.0)[3]
    np.testing.assert_allclose(s_a, s_b, rtol=1e-12, atol=1e-12)
    # the value map is applied: S_1 from S_0 = 0 with unit orthogonal keys is K'^T diag(beta) V phi_v^T
    ku = np.eye(d)[:T]
    s1 = O.head_pass(q, ku, v, np.eye(d), np.eye(d), P, np.zeros(T), np.full(T, INF),
                     np.zeros((d, d)), True, l2_eps=0.0)[3]
    np.testing.assert_allclose(s1[:T], v[:, pi], rtol=0, atol=1e-15)


def pin_memory_constant_in_frames():
    """Only the state is carried between frames: the oracle's peak traced
    memory for 40 frames equals that for 4 frames (within a small slack)."""
    rng = _rng(11)
    B, T, H, d = 1, 32, 2, 8
    data = [rng.standard_normal((B, T, H, d)) for _ in range(3)]
    gates = [rng.standard_normal((B, H, T)) for _ in range(2)]
    phis = [np.eye(d)[None].repeat(H, 0) for _ in range(3)]

    def src(n, p):
        return data[0], data[1], data[2], gates[0], gates[1]

    def peak(F):
        tracemalloc.start()
        O.run_frames(src, *phis, np.zeros((B, H, d, d)), F, (False, True))
        _, pk = tracemalloc.get_traced_memory()
        tracemalloc.stop()
        return pk

    p4, p40 = peak(4), peak(40)
    assert p40 <= p4 * 1.05 + 4096, (p4, p40)


PINS = [
    pin_intra_matches_library_sdpa,
    pin_intra_special_cases,
    pin_golden_single_token,
    pin_golden_two_tokens_feature_maps,
    pin_zero_state_gives_zero_inter,
    pin_state_invariance_and_forget_closed_form,
    pin_query_only_pass_does_not_write,
    pin_update_equals_token_loop_bruteforce,
    pin_delta_rule_stores_value,
    pin_orthonormal_keys_store_all_values,
    pin_permutation_and_linearity,
    pin_feature_map_orientation_and_key_scale,
    pin_memory_constant_in_frames,
]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_pin(pin):
    pin()


# ---------------------------------------------------------------- planted mistakes

def _mut_phi_transposed(x, phi):
    return np.asarray(x, dtype=np.float64) @ np.asarray(phi, dtype=np.float64)


def _mut_no_scale(q, k, v, sm_scale):
    return _ORIG["intra_frame_attention"](q, k, v, 1.0)


def _mut_softmax_wrong_axis(q, k, v, sm_scale):
    s = (q @ k.T) * sm_scale
    w = np.exp(s - s.max(axis=0, keepdims=True))
    return (w / w.sum(axis=0, keepdims=True)) @ v


def _mut_residual_sign(state, k_unit, v_feat, beta, alpha):
    return alpha * state + k_unit.T @ (beta[:, None] * (k_unit @ state - v_feat))


def _mut_no_alpha(state, k_unit, v_feat, beta, alpha):
    return _ORIG["gated_delta_update"](state, k_unit, v_feat, beta, 1.0)


def _mut_alpha_on_all(state, k_unit, v_feat, beta, alpha):
    return alpha * _ORIG["gated_delta_update"](state, k_unit, v_feat, beta, 1.0)


def _mut_no_beta(state, k_unit, v_feat, beta, alpha):
    return _ORIG["gated_delta_update"](state, k_unit, v_feat, np.ones_like(beta), alpha)


def _mut_sigmoid_of_mean(gate_logits, beta_logits):
    return float(O.sigmoid(np.mean(gate_logits))), O.sigmoid(beta_logits)


def _mut_no_l2(x, eps):
    return np.asarray(x, dtype=np.float64)


def _mut_inter_transposed_state(q_feat, state):
    return q_feat @ np.asarray(state).T


def _mut_inter_reads_nothing(q_feat, state):
    return np.zeros((q_feat.shape[0], state.shape[1]))


def _mut_sigmoid_sign(x):
    return 1.0 / (1.0 + np.exp(np.asarray(x, dtype=np.float64)))


_ORIG = {name: getattr(O, name) for name in
         ("feature_map", "intra_frame_attention", "gated_delta_update", "frame_gates",
          "l2_normalise_rows", "inter_frame_read", "sigmoid")}

MUTANTS = {
    "phi_transposed": ("feature_map", _mut_phi_transposed),
    "softmax_no_scale": ("intra_frame_attention", _mut_no_scale),
    "softmax_wrong_axis": ("intra_frame_attention", _mut_softmax_wrong_axis),
    "residual_sign": ("gated_delta_update", _mut_residual_sign),
    "forget_gate_dropped": ("gated_delta_update", _mut_no_alpha),
    "forget_gate_on_update": ("gated_delta_update", _mut_alpha_on_all),
    "beta_dropped": ("gated_delta_update", _mut_no_beta),
    "alpha_sigmoid_of_mean": ("frame_gates", _mut_sigmoid_of_mean),
    "key_not_normalised": ("l2_normalise_rows", _mut_no_l2),
    "inter_state_transposed": ("inter_frame_read", _mut_inter_transposed_state),
    "inter_branch_dropped": ("inter_frame_read", _mut_inter_reads_nothing),
    "sigmoid_sign": ("sigmoid", _mut_sigmoid_sign),
}


@pytest.mark.parametrize("mutant", sorted(MUTANTS))
def test_planted_mistakes_are_caught(mutant, monkeypatch):
    name, fn = MUTANTS[mutant]
    monkeypatch.setattr(O, name, fn)
    failed = []
    for pin in PINS:
        try:
            pin()
        except AssertionError:
            failed.append(pin.__name__)
    assert failed, f"no pin caught the planted mistake {mutant}"
