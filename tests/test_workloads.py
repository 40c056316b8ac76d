"""The seeded input generators: determinism, shapes, distributions, rounding."""

import numpy as np
import torch

import workloads as W


def test_inputs_are_deterministic_and_per_pass():
    w = W.small_workload(W.WORKLOADS[0], frames=2)
    a = W.pass_inputs(w, 1, 2)
    b = W.pass_inputs(w, 1, 2)
    c = W.pass_inputs(w, 1, 1)
    assert torch.equal(a.q, b.q) and torch.equal(a.gate_logits, b.gate_logits)
    assert not torch.equal(a.q, c.q)
    assert not torch.equal(a.q, a.k)


def test_shapes_dtypes_and_rounding():
    w = W.WORKLOADS[1]
    p = W.pass_inputs(w, 0, 0)
    assert p.q.shape == (1, 1560, 12, 128) and p.q.dtype == torch.bfloat16
    assert p.gate_logits.shape == (1, 12, 1560) and p.gate_logits.dtype == torch.float32
    q64 = p.as_f64()[0]
    # the float64 view is exactly the bf16 values
    assert np.array_equal(torch.from_numpy(q64).to(torch.bfloat16).to(torch.float64).numpy(), q64)
    assert abs(q64.mean()) < 0.01 and abs(q64.std() - 1.0) < 0.01
    g = p.gate_logits.numpy()
    assert abs(g.mean() - 2.0) < 0.05 and abs(g.std() - 1.0) < 0.05
    phq, phk, phv = W.feature_maps(w)
    assert phq.shape == (12, 128, 128)
    off = phq.to(torch.float64).numpy() - np.eye(128)[None]
    assert abs(off.std() - 0.02) < 0.002
    assert not torch.equal(phq, phk)


def test_long_stream_pool_cycles():
    w = W.WORKLOADS[4]
    assert torch.equal(W.pass_inputs(w, 3, 0).gate_logits, W.pass_inputs(w, 11, 0).gate_logits)
    assert not torch.equal(W.pass_inputs(w, 3, 0).gate_logits, W.pass_inputs(w, 4, 0).gate_logits)
    g = W.pass_inputs(w, 0, 0)
    assert abs(g.gate_logits.mean().item() - 3.0) < 0.05
    assert abs(g.beta_logits.mean().item() + 1.0) < 0.05


def test_prior_frames_distinct_from_stream():
    w = W.WORKLOADS[2]
    a = W.prior_frame_inputs(w, 0)
    b = W.pass_inputs(w, 0, 0)
    assert not torch.equal(a.q, b.q)
