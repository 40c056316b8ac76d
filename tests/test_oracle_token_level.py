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


def pin_chunked_triangular_solve_form():
    # The same recurrence in chunks of C tokens, as a kernel would compute it.
    # With gamma_t = alpha_1 ... alpha_t and the normalised state S^_t = S_t / gamma_t,
    #   S^_t = S^_{t-1} + k_t u_t^T,  u_t = c_t v'_t - b_t S^_{t-1}^T k_t,
    #   b_t = beta_t / alpha_t, c_t = beta_t / gamma_t,
    # so per chunk (I + diag(b) tril(K K^T, -1)) U = diag(c) V - diag(b) K S^_0,
    # S^_C = S^_0 + K^T U, and token t reads gamma_{t-1} (q_t S^_0 + sum_{r<t} (q_t . k_r) u_r).
    q, k, v, phi, g, bl, S0 = _inputs(7, T=11)
    _, _, oe, S = O.token_level_head_pass(q, k, v, *phi, g, bl, S0, True)
    kf = k @ phi[1].T
    ku = kf / np.sqrt((kf ** 2).sum(axis=1, keepdims=True) + 1e-6)
    vf, qf = v @ phi[2].T, q @ phi[0].T
    al, be = 1 / (1 + np.exp(-g)), 1 / (1 + np.exp(-bl))
    Sc = S0.copy()
    reads = np.empty_like(oe)
    C = 4
    for c0 in range(0, 11, C):
        sl = slice(c0, min(11, c0 + C))
        K, V, Q, a, bt = ku[sl], vf[sl], qf[sl], al[sl], be[sl]
        gam = np.cumprod(a)
        gam_prev = np.concatenate([[1.0], gam[:-1]])
        b, cc = bt / a, bt / gam
        L = np.eye(len(a)) + np.diag(b) @ np.tril(K @ K.T, -1)
        U = np.linalg.solve(L, np.diag(cc) @ V - np.diag(b) @ K @ Sc)
        reads[sl] = gam_prev[:, None] * (Q @ Sc + np.tril(Q @ K.T, -1) @ U)
        Sc = gam[-1] * (Sc + K.T @ U)
    np.testing.assert_allclose(oe, reads, rtol=1e-9, atol=1e-9)
    np.testing.assert_allclose(S, Sc, rtol=1e-9, atol=1e-9)


PINS = [pin_chunked_triangular_solve_form, pin_one_token_is_the_frame_level_rule, pin_single_token_stores_its_value,
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
