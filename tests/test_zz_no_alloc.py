"""hyb_attn_forward_noalloc: the workspace-free entry point.

Some callers cannot allocate device memory at the point where they run the
layer (a stream being captured into a CUDA graph under a strict capture mode,
an allocator callback, a serving loop whose memory is fixed up front), so they
cannot hand the library a workspace.  This entry point runs the same pass on a
scratch array the library keeps on each GPU.  The tests call it through the C
ABI on consecutive passes and compare its outputs and states with
hyb_attn_forward given a caller-owned workspace.  Both run the same kernels in
the same order on the same data, so the results must agree bit for bit, on the
bf16 tensor-core path and on the fp32 path (whose update keeps its split
partials and its copy of S_{N-1} in the scratch array).  This file is named to
be collected last.
"""

import numpy as np
import pytest
import torch

import workloads as W



def _inputs(w, n, p):
    x = W.pass_inputs(w, n, p)
    return [t.cuda() for t in (x.q, x.k, x.v, x.gate_logits, x.beta_logits)]


def _compare(w, frames):
    import gated_delta_linear_b200 as G
    phi = [p.cuda() for p in W.feature_maps(w)]
    desc = G.make_desc(w.B, w.H, w.T, w.d, G.HYB_BF16 if w.dtype == "bf16" else G.HYB_FP32)
    need = G.hyb_attn_workspace_bytes(desc)
    assert 0 < need <= G.HYB_NOALLOC_SCRATCH_BYTES
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    s_ref = torch.zeros(w.B, w.H, w.d, w.d, dtype=torch.float32, device="cuda")
    s_new = torch.zeros_like(s_ref)
    calls = 0
    for n in range(frames):
        for p, clean in enumerate(w.passes):
            q, k, v, g, bl = _inputs(w, n, p)
            o_ref = torch.empty_like(q)
            o_new = torch.empty_like(q)
            assert G.hyb_attn_forward(desc, q, k, v, *phi, g, bl, s_ref, int(clean), o_ref, ws) == G.HYB_OK
            assert G.hyb_attn_forward_noalloc(desc, q, k, v, *phi, g, bl, s_new, int(clean), o_new) == G.HYB_OK
            torch.cuda.synchronize()
            assert torch.equal(o_new, o_ref), f"frame {n} pass {p}: outputs differ"
            assert torch.equal(s_new, s_ref), f"frame {n} pass {p}: states differ"
            calls += 1
    assert calls >= 2
    assert np.isfinite(s_new.cpu().numpy()).all()
    assert s_new.abs().sum().item() > 0


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_on_two_calls():
    """bf16, d = 128 (tensor-core path): two full 480p frames, each a clean pass."""
    _compare(W.WORKLOADS[1], frames=2)


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_fp32_path():
    """fp32, d = 32: every pass of the tiny workload (2 query-only + 1 clean per frame)."""
    _compare(W.WORKLOADS[0], frames=W.WORKLOADS[0].frames)


def test_noalloc_rejects_descriptors_beyond_its_scratch():
    """Host path: the size check comes before any CUDA call."""
    import gated_delta_linear_b200 as G
    big = G.make_desc(1, 512, 1560, 128, G.HYB_BF16)
    assert G.hyb_attn_workspace_bytes(big) > G.HYB_NOALLOC_SCRATCH_BYTES
    fake = 0x10000
    st = G.hyb_attn_forward_noalloc(big, fake, fake, fake, fake, fake, fake, fake, fake, fake, 1,
                                    fake, 0)
    assert st == G.HYB_ERR_WORKSPACE


@pytest.mark.parametrize("what", ["null", "misaligned", "bad_flag"])
def test_noalloc_rejects_bad_arguments_before_any_cuda_call(what):
    """Argument errors come back before the scratch address is looked up or
    anything is enqueued, so these host-path checks need no GPU."""
    import gated_delta_linear_b200 as G
    desc = G.make_desc(1, 2, 64, 128, G.HYB_BF16)
    fake = 0x10000
    args = [fake] * 9 + [1, fake]
    if what == "null":
        args[0] = None
        want = G.HYB_ERR_INVALID
    elif what == "misaligned":
        args[1] = fake + 2
        want = G.HYB_ERR_ALIGN
    else:
        args[9] = 3
        want = G.HYB_ERR_INVALID
    assert G.hyb_attn_forward_noalloc(desc, *args, 0) == want



@pytest.mark.gpu
def test_noalloc_status_getter_reports_the_last_call():
    """The no-allocation entry point's device flags: HYB_OK after a normal call;
    after a call whose bounded wait is made to run out (the fault test), the
    getter reports HYB_ERR_TIMEOUT, and a normal call afterwards is HYB_OK again."""
    import gated_delta_linear_b200 as G
    w = W.small_workload(W.WORKLOADS[1], H=2, T=300, frames=1)
    phi = [p.cuda() for p in W.feature_maps(w)]
    desc = G.make_desc(w.B, w.H, w.T, w.d, G.HYB_BF16)
    q, k, v, g, bl = _inputs(w, 0, 0)
    S = torch.zeros(w.B, w.H, w.d, w.d, dtype=torch.float32, device="cuda")
    out = torch.empty_like(q)
    assert G.hyb_attn_forward_noalloc(desc, q, k, v, *phi, g, bl, S, 0, out) == G.HYB_OK
    assert G.hyb_attn_noalloc_device_status() == G.HYB_OK
    assert G.hyb_attn_set_fault_test(1, 5000) == G.HYB_OK
    try:
        assert G.hyb_attn_forward_noalloc(desc, q, k, v, *phi, g, bl, S, 0, out) == G.HYB_OK
        assert G.hyb_attn_noalloc_device_status() == G.HYB_ERR_TIMEOUT
    finally:
        G.hyb_attn_set_fault_test(0, 0)
    assert G.hyb_attn_forward_noalloc(desc, q, k, v, *phi, g, bl, S, 0, out) == G.HYB_OK
    assert G.hyb_attn_noalloc_device_status() == G.HYB_OK
