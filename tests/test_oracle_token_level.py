"""Pins of the oracle's token-level access variant (``token_level_head_pass``,
"Technical summary: Attend Locally, Remember Linearly (ARL2)" §4 ablation; the
readings are stated in its docstring), each checked against something other
than its token loop, and planted mistakes the pins must catch."""

import numpy as np
import pytest

from oracle import hybrid_layer as O

BIG = 40.0  # sigmoid(40) = 1 to double precision


def _inputs(seed, T=5, d=8, state_scale=1.0):
    rng = np.random.default_rng(seed)
    q, k, v = (rng.standard_normal((T, d)) for _ in range(3))
    phi = [np.eye(d) + 0.05 * rng.standard_normal((d, d)) for _ in range(3)]
    g, bl = rng.standard_normal(T) + 1.0, rng.standard_normal(T)
    S = state_scale * rng.standard_normal((d, d))
    return q, k, v, phi, g, bl, S


def pin_one_token_is_the_frame_level_rule():
    q, k, v, phi, g, bl, S = _inputs(1, T=1)
    a = O.token_level_head_pass(q, k, v, *phi, g, bl, S, True)
    b = O.head_pass(q, k, v, *phi, g, bl, S, True)
    for x, y in zip(a, b):
        np.testing.assert_allclose(x, y, rtol=1e-12, atol=1e-12)


def pin_single_token_stores_its_value():
    # alpha = beta = 1, unit key: k^T S_new = v^T exactly (the delta rule)
    rng = np.random.default_rng(2)
    d = 6
    k = rng.standard_normal((1, d))
    v = rng.standard_normal((1, d))
    eye = np.eye(d)
    _, _, _, S = O.token_level_head_pass(k, k, v, eye, eye, eye, np.array([BIG]), np.array([BIG]),
                                         rng.standard_normal((d, d)), True, l2_eps=0.0)
    ku = k[0] / np.linalg.norm(k[0])
    np.testing.assert_allclose(ku @ S, v[0], rtol=1e-12, atol=1e-12)


def pin_orthonormal_keys_match_the_frame_level_update():
    # alpha = 1 and K'K'^T = I: the token-sequential updates commute and equal the batch rule
    rng = np.random.default_rng(3)
    d, T = 8, 5
    basis = np.linalg.qr(rng.standard_normal((d, d)))[0][:T]
    q, v = rng.standard_normal((T, d)), rng.standard_normal((T, d))
    eye = np.eye(d)
    g, bl = np.full(T, BIG), rng.standard_normal(T)
    S0 = rng.standard_normal((d, d))
    _, _, _, a = O.token_level_head_pass(q, basis, v, eye, eye, eye, g, bl, S0, True, l2_eps=0.0)
    _, _, _, b = O.head_pass(q, basis, v, eye, eye, eye, g, bl, S0, True, l2_eps=0.0)
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-12)


def pin_query_only_pass_is_the_frame_level_pass():
    q, k, v, phi, g, bl, S = _inputs(4)
    a = O.token_level_head_pass(q, k, v, *phi, g, bl, S, False)
    b = O.head_pass(q, k, v, *phi, g, bl, S, False)
    for x, y in zip(a, b):
        np.testing.assert_allclose(x, y, rtol=0, atol=0)


def pin_each_step_is_non_expansive():
    # ||alpha I - beta k k^T||_2 <= 1 for unit k and alpha, beta in (0, 1]:
    # ||S'||_2 <= ||S||_2 + beta ||v'||, token after token (one-token frames)
    rng = np.random.default_rng(5)
    d = 8
    eye = np.eye(d)
    S = 3.0 * rng.standard_normal((d, d))
    for _ in range(40):
        k, v = rng.standard_normal((1, d)), rng.standard_normal((1, d))
        g, bl = rng.standard_normal(1), rng.standard_normal(1)
        _, _, _, S2 = O.token_level_head_pass(k, k, v, eye, eye, eye, g, bl, S, True)
        beta = 1 / (1 + np.exp(-bl[0]))
        assert np.linalg.norm(S2, 2) <= np.linalg.norm(S, 2) + beta * np.linalg.norm(v) + 1e-9
        S = S2


def pin_product_form_of_the_recurrence():
    # S_t = A_{t-1} ... A_0 S_0 + sum_s A_{t-1} ... A_{s+1} beta_s k_s v_s^T,
    # A_s = alpha_s I - beta_s k_s k_s^T: reads O_inter[t] = q'_t S_t and the final state
    q, k, v, phi, g, bl, S0 = _inputs(6, T=4)
    out, oi, oe, S = O.token_level_head_pass(q, k, v, *phi, g, bl, S0, True)
    d = q.shape[1]
    kf = k @ phi[1].T
    ku = kf / np.sqrt((kf ** 2).sum(axis=1, keepdims=True) + 1e-6)
    vf = v @ phi[2].T
    qf = q @ phi[0].T
    al, be = 1 / (1 + np.exp(-g)), 1 / (1 + np.exp(-bl))
    A = [al[s] * np.eye(d) - be[s] * np.outer(ku[s], ku[s]) for s in range(4)]
    for t in range(5):
        St = np.eye(d)
        for s in range(t):
            St = A[s] @ St
        St = St @ S0
        for s in range(t):
            P = np.eye(d)
            for r in range(s + 1, t):
                P = A[r] @ P
            St = St + P @ (be[s] * np.outer(ku[s], vf[s]))
        if t < 4:
            np.testing.assert_allclose(oe[t], qf[t] @ St, rtol=1e-10, atol=1e-10)
        else:
            np.testing.assert_allclose(S, St, rtol=1e-10, atol=1e-10)


def _chunked_pass(q, k, v, phi, g, bl, S0, C, dtype):
    """The token-level recurrence in chunks of C tokens, as a kernel computes it,
    with only relative decays (every factor exp(Lambda_a - Lambda_b) <= 1,
    Lambda_t = sum_{r <= t} log alpha_r; nothing is divided by a gate).
    Inside a chunk that starts from state S, with u_t the row beta_t (v'_t - k'_t S_{t-1}):
      (I + L) U = diag(beta) V - diag(beta * gprev) K S,
      L[t, s] = beta_t exp(Lambda_{t-1} - Lambda_s) (k_t . k_s)      for s < t,
      gprev_t = exp(Lambda_{t-1})  (the decay from the chunk start to token t's read),
      read_t  = gprev_t q_t S + sum_{s<t} exp(Lambda_{t-1} - Lambda_s) (q_t . k_s) u_s,
      S_end   = exp(Lambda_{C-1}) S + sum_s exp(Lambda_{C-1} - Lambda_s) k_s u_s."""
    f = lambda x: np.asarray(x, dtype=dtype)
    kf = k @ phi[1].T
    ku = f(kf / np.sqrt((kf ** 2).sum(axis=1, keepdims=True) + 1e-6))
    vf, qf = f(v @ phi[2].T), f(q @ phi[0].T)
    logal = f(-np.logaddexp(0.0, -np.asarray(g, dtype=np.float64)))  # log sigmoid(g), no overflow
    be = f(1 / (1 + np.exp(-np.asarray(bl, dtype=np.float64))))
    T = q.shape[0]
    Sc = f(S0)
    reads = np.empty((T, S0.shape[1]), dtype=dtype)
    for c0 in range(0, T, C):
        sl = slice(c0, min(T, c0 + C))
        K, V, Q, la, bt = ku[sl], vf[sl], qf[sl], logal[sl], be[sl]
        n = len(la)
        Lam = np.cumsum(la)                                   # Lambda_t within the chunk
        Lprev = np.concatenate([np.zeros(1, dtype=dtype), Lam[:-1]])
        dec = np.exp(np.minimum(Lprev[:, None] - Lam[None, :], 0.0))  # exp(Lambda_{t-1} - Lambda_s)
        strict = np.tril(np.ones((n, n), dtype=dtype), -1)
        A = strict * dec * (K @ K.T)
        gprev = np.exp(Lprev)
        U = np.linalg.solve(np.eye(n, dtype=dtype) + bt[:, None] * A,
                            bt[:, None] * V - (bt * gprev)[:, None] * (K @ Sc))
        reads[sl] = gprev[:, None] * (Q @ Sc) + (strict * dec * (Q @ K.T)) @ U
        Sc = np.exp(Lam[-1]) * Sc + K.T @ (np.exp(Lam[-1] - Lam)[:, None] * U)
    return reads, Sc


def pin_chunked_triangular_solve_form():
    # float64, chunks of 4 over 11 tokens: the chunked form equals the token loop
    q, k, v, phi, g, bl, S0 = _inputs(7, T=11)
    _, _, oe, S = O.token_level_head_pass(q, k, v, *phi, g, bl, S0, True)
    reads, Sc = _chunked_pass(q, k, v, phi, g, bl, S0, 4, np.float64)
    np.testing.assert_allclose(oe, reads, rtol=1e-9, atol=1e-9)
    np.testing.assert_allclose(S, Sc, rtol=1e-9, atol=1e-9)


def pin_chunked_form_in_fp32_with_strong_forgetting():
    # fp32, chunks of 64 over 150 tokens (a ragged last chunk), gate logits down to
    # -6 (alpha ~ 2.5e-3): the relative-decay form stays finite and accurate
    rng = np.random.default_rng(8)
    T, d = 150, 32
    q, k, v = (rng.standard_normal((T, d)) for _ in range(3))
    phi = [np.eye(d) + 0.02 * rng.standard_normal((d, d)) for _ in range(3)]
    g = rng.uniform(-6.0, 3.0, T)
    g[::7] = -6.0
    bl = rng.standard_normal(T)
    S0 = rng.standard_normal((d, d))
    _, _, oe, S = O.token_level_head_pass(q, k, v, *phi, g, bl, S0, True)
    reads, Sc = _chunked_pass(q, k, v, phi, g, bl, S0, 64, np.float32)
    assert np.isfinite(reads).all() and np.isfinite(Sc).all()
    rel = lambda a, b: np.linalg.norm(a - b) / np.linalg.norm(b)
    assert rel(reads.astype(np.float64), oe) < 1e-4, rel(reads.astype(np.float64), oe)
    assert rel(Sc.astype(np.float64), S) < 1e-4, rel(Sc.astype(np.float64), S)


PINS = [pin_chunked_triangular_solve_form, pin_chunked_form_in_fp32_with_strong_forgetting, pin_one_token_is_the_frame_level_rule, pin_single_token_stores_its_value,
        pin_orthonormal_keys_match_the_frame_level_update, pin_query_only_pass_is_the_frame_level_pass,
        pin_each_step_is_non_expansive, pin_product_form_of_the_recurrence]


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin()


def _mutant(kind):
    def f(q, k, v, phi_q, phi_k, phi_v, gate_logits, beta_logits, state, clean_pass, sm_scale=None,
          l2_eps=1e-6):
        d = q.shape[1]
        sm = 1.0 / np.sqrt(d) if sm_scale is None else sm_scale
        oi = O.intra_frame_attention(q, k, v, sm)
        qf = O.feature_map(q, phi_q)
        if not clean_pass:
            oe = O.inter_frame_read(qf, state)
            return oi + oe, oi, oe, state
        ku = O.l2_normalise_rows(O.feature_map(k, phi_k), l2_eps)
        vf = O.feature_map(v, phi_v)
        al = O.sigmoid(np.asarray(gate_logits, dtype=np.float64))
        if kind == "frame_mean_gate":
            al = np.full_like(al, al.mean())
        be = O.sigmoid(np.asarray(beta_logits, dtype=np.float64))
        if kind == "no_beta":
            be = np.ones_like(be)
        S = np.array(state, dtype=np.float64)
        oe = np.empty_like(qf)
        for t in range(q.shape[0]):
            if kind != "read_after_update":
                oe[t] = qf[t] @ S
            upd = np.outer(vf[t] - ku[t] @ S, ku[t]) if kind == "transposed_outer" else np.outer(ku[t], vf[t] - ku[t] @ S)
            S = al[t] * S + be[t] * upd
            if kind == "read_after_update":
                oe[t] = qf[t] @ S
        return oi + oe, oi, oe, S
    f.__name__ = kind
    return f


@pytest.mark.parametrize("kind", ["read_after_update", "frame_mean_gate", "no_beta", "transposed_outer"])
def test_planted_mistakes_are_caught(kind, monkeypatch):
    monkeypatch.setattr(O, "token_level_head_pass", _mutant(kind))
    caught = 0
    for pin in PINS:
        try:
            pin()
        except AssertionError:
            caught += 1
    assert caught >= 1, f"no pin caught {kind}"
