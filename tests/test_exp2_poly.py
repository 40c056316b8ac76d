"""The FMA-pipe exp2 of the attention softmax, simulated step by step in
float32 on the CPU against numpy's exp2 (the device function follows the same
operations: clamp, Cody-Waite split with the 1.5 * 2^23 shift, degree-3
polynomial, exponent-field add)."""

import numpy as np

C = np.array([0.9999280571937561, 0.6932609677314758, 0.2426111251115799, 0.0551716685295105],
             dtype=np.float32)


def exp2_fma(x):
    x = np.maximum(x.astype(np.float32), np.float32(-125.0))
    t = (x + np.float32(12582912.0)).astype(np.float32)
    f = (x - (t - np.float32(12582912.0))).astype(np.float32)
    p = np.float32(C[3]) * f + C[2]
    p = (p * f + C[1]).astype(np.float32)
    p = (p * f + C[0]).astype(np.float32)
    bits = p.view(np.int32) + (t.view(np.int32) << 23)
    return bits.astype(np.int32).view(np.float32)


def test_relative_error_over_the_softmax_range():
    x = np.linspace(-125.0, 8.0, 2_000_001, dtype=np.float32)
    got = exp2_fma(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got - ref) / ref
    # well inside a bf16 half-ulp (2^-9 ~ 2e-3), where the result is rounded next
    assert rel.max() < 1.2e-4, rel.max()


def test_integers_and_clamp():
    for n in range(-125, 9):
        v = exp2_fma(np.array([n], dtype=np.float32))[0]
        assert abs(v / 2.0 ** n - 1) < 1.2e-4
    tiny = exp2_fma(np.array([-np.inf, -1e30, -300.0], dtype=np.float32))
    assert np.all(tiny > 0) and np.all(tiny < 3e-38)


def test_coefficients_match_the_fit_script():
    import importlib.util
    import os
    path = os.path.join(os.path.dirname(os.path.dirname(__file__)), "gated_delta_linear_b200", "csrc",
                        "gen_exp2_poly.py")
    spec = importlib.util.spec_from_file_location("gen_exp2_poly", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    c, err = mod.remez()
    assert np.allclose(c.astype(np.float32), C, rtol=0, atol=0), (c, C)
    assert err < 8e-5
