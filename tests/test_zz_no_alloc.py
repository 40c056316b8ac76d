"""hyb_attn_forward_noalloc: the workspace-free entry point.

Some callers cannot allocate device memory at the point where they run the
layer (a stream being captured into a CUDA graph under a strict capture mode,
an allocator callback, a serving loop whose memory is fixed up front), so they
cannot hand the library a workspace.  This entry point runs the same pass on a
scratch array the library keeps on each GPU.  The test calls it through the C
ABI twice in a row (two frames, each a clean pass that updates the state) and
checks its outputs and states against hyb_attn_forward with a caller-owned
workspace, within the parity tolerances of the other GPU tests.  This file is
named to be collected last.
"""

import numpy as np
import pytest
import torch

import workloads as W
from tests import tolerances as tol

pytestmark = pytest.mark.gpu


def _inputs(w, n):
    x = W.pass_inputs(w, n, 0)
    return [t.cuda() for t in (x.q, x.k, x.v, x.gate_logits, x.beta_logits)]


def test_noalloc_matches_workspace_entry_point_on_two_calls():
    import gated_delta_linear_b200 as G
    w = W.WORKLOADS[1]
    phi = [p.cuda() for p in W.feature_maps(w)]
    desc = G.make_desc(w.B, w.H, w.T, w.d, G.HYB_BF16)
    need = G.hyb_attn_workspace_bytes(desc)
    assert 0 < need <= G.HYB_NOALLOC_SCRATCH_BYTES
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    s_ref = torch.zeros(w.B, w.H, w.d, w.d, dtype=torch.float32, device="cuda")
    s_new = torch.zeros_like(s_ref)
    for n in range(2):
        q, k, v, g, bl = _inputs(w, n)
        o_ref = torch.empty_like(q)
        o_new = torch.empty_like(q)
        assert G.hyb_attn_forward(desc, q, k, v, *phi, g, bl, s_ref, 1, o_ref, ws) == G.HYB_OK
        assert G.hyb_attn_forward_noalloc(desc, q, k, v, *phi, g, bl, s_new, 1, o_new) == G.HYB_OK
        torch.cuda.synchronize()
        got = o_new.to(torch.float64).cpu().numpy()
        ref = o_ref.to(torch.float64).cpu().numpy()
        for h in range(w.H):
            tol.check(tol.scaled_errors(got[0, :, h], ref[0, :, h]), tol.OUT_BF16, f"call {n} head {h}")
        for h in range(w.H):
            r = tol.rel_frobenius(s_new[0, h].double().cpu().numpy(), s_ref[0, h].double().cpu().numpy())
            assert r <= tol.STATE_BF16, (n, h, r)
    assert np.isfinite(s_new.cpu().numpy()).all()


def test_noalloc_rejects_descriptors_beyond_its_scratch():
    import gated_delta_linear_b200 as G
    big = G.make_desc(1, 512, 1560, 128, G.HYB_BF16)
    assert G.hyb_attn_workspace_bytes(big) > G.HYB_NOALLOC_SCRATCH_BYTES
    fake = 0x10000
    st = G.hyb_attn_forward_noalloc(big, fake, fake, fake, fake, fake, fake, fake, fake, fake, 1,
                                    fake, 0)
    assert st == G.HYB_ERR_WORKSPACE
