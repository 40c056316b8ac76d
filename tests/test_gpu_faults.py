"""Failure detection on the GPU without a GPU fault.

Every device wait of the attention kernel and of the delta update is bounded.
The library's fault test switches off the attention kernel's value-tile loads
and shortens the limit to a few milliseconds, so that the MMA issuer's first
wait for a value tile runs out: nothing arrives on that barrier, and no copy is
in flight.  The kernel must then set the TIMEOUT flag, store nothing, drain its
issued products and free its tensor memory and return; the host reads
HYB_ERR_TIMEOUT, and the next normal pass on the same device must be correct.
The chained update's wait for the previous update's flag words is made to run
out the same way, by clearing those words.
"""

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from tests import tolerances as tol


def test_fault_test_knob_validates_its_arguments():
    import gated_delta_linear_b200 as G
    assert G.hyb_attn_set_fault_test(2, 0) == G.HYB_ERR_INVALID
    assert G.hyb_attn_set_fault_test(0, 20 * 1000 * 1000) == G.HYB_ERR_INVALID
    assert G.hyb_attn_set_fault_test(0, 0) == G.HYB_OK


@pytest.mark.gpu
def test_expired_wait_reports_timeout_and_device_stays_usable():
    import gated_delta_linear_b200 as G
    w = W.small_workload(W.WORKLOADS[1], H=2, T=300, frames=2)
    phi = W.feature_maps(w)
    layer = G.HybridAttention(w.B, w.H, w.T, w.d, w.torch_dtype, *phi)
    x = W.pass_inputs(w, 0, 0)
    dev = [t.cuda() for t in (x.q, x.k, x.v, x.gate_logits, x.beta_logits)]
    out = torch.full_like(dev[0], 7.0)
    assert layer.device_status() == G.HYB_OK
    assert G.hyb_attn_set_fault_test(1, 5000) == G.HYB_OK   # no V loads, 5 ms limit
    try:
        layer.forward(*dev, 0, out=out)                     # query-only: the state is not touched
        st = layer.device_status()                          # synchronises; returns
    finally:
        assert G.hyb_attn_set_fault_test(0, 0) == G.HYB_OK
    assert st == G.HYB_ERR_TIMEOUT, G.hyb_attn_status_string(st)
    assert torch.all(out == 7.0), "no output tile may be stored after an expired wait"
    assert layer.device_status() == G.HYB_OK                # the flag was cleared by the read

    # the same device, the same layer: a normal clean pass is correct
    phi64 = [p.to(torch.float64).numpy() for p in phi]
    layer.state.zero_()
    got = layer.forward(*dev, 1)
    torch.cuda.synchronize()
    assert layer.device_status() == G.HYB_OK
    q, k, v, g, bl = x.as_f64()
    ref, _, _, S = oracle.layer_pass(q, k, v, *phi64, g, bl, W.zero_state(w), True)
    gotn = got.to("cpu", torch.float64).numpy()
    for h in range(w.H):
        tol.check(tol.scaled_errors(gotn[0, :, h], ref[0, :, h]), tol.OUT_BF16, f"head {h}")
    Sg = layer.state.to("cpu", torch.float64).numpy()
    assert max(tol.rel_frobenius(Sg[0, h], S[0, h]) for h in range(w.H)) <= tol.STATE_BF16


@pytest.mark.gpu
def test_expired_chain_wait_reports_timeout_and_device_stays_usable():
    """A chained delta update waits, bounded, for the previous update's flag
    words before it reads the state.  Zeroing the workspace between two chained
    calls (a write the chain's contract rules out) leaves those words unset: the
    wait runs out, the update leaves the state as it was, the host reads
    HYB_ERR_TIMEOUT, and a normal pass afterwards is correct."""
    import gated_delta_linear_b200 as G
    w = W.small_workload(W.WORKLOADS[1], H=2, T=300, frames=3)
    phi = W.feature_maps(w)
    layer = G.HybridAttention(w.B, w.H, w.T, w.d, w.torch_dtype, *phi)
    xs = [W.pass_inputs(w, n, 0) for n in range(3)]
    dev = [[t.cuda() for t in (x.q, x.k, x.v, x.gate_logits, x.beta_logits)] for x in xs]
    layer.forward(*dev[0], 1)
    layer.forward_next(*dev[1], 1)      # starts a chain; its update raises the flags
    torch.cuda.synchronize()
    assert layer.device_status() == G.HYB_OK
    s_before = layer.state.clone()
    layer.workspace.zero_()             # clears the words the next chained update waits for
    assert G.hyb_attn_set_fault_test(0, 5000) == G.HYB_OK   # 5 ms limit
    try:
        layer.forward_next(*dev[2], 1)  # continues the chain: its flag wait runs out
        st = layer.device_status()      # synchronises; returns
    finally:
        assert G.hyb_attn_set_fault_test(0, 0) == G.HYB_OK
    assert st == G.HYB_ERR_TIMEOUT, G.hyb_attn_status_string(st)
    assert torch.equal(layer.state, s_before), "an update whose wait ran out must leave the state"
    assert layer.device_status() == G.HYB_OK

    # the same layer: a normal clean pass (which ends the chain) is correct
    phi64 = [p.to(torch.float64).numpy() for p in phi]
    layer.state.zero_()
    got = layer.forward(*dev[0], 1)
    torch.cuda.synchronize()
    assert layer.device_status() == G.HYB_OK
    q, k, v, g, bl = xs[0].as_f64()
    ref, _, _, S = oracle.layer_pass(q, k, v, *phi64, g, bl, W.zero_state(w), True)
    gotn = got.to("cpu", torch.float64).numpy()
    for h in range(w.H):
        tol.check(tol.scaled_errors(gotn[0, :, h], ref[0, :, h]), tol.OUT_BF16, f"head {h}")
    Sg = layer.state.to("cpu", torch.float64).numpy()
    assert max(tol.rel_frobenius(Sg[0, h], S[0, h]) for h in range(w.H)) <= tol.STATE_BF16
