"""C-ABI checks that need no GPU: the library loads, exports every declared
symbol, sizes its workspace, and rejects bad arguments on the host before
anything is launched."""

import ctypes
import os
import re

import pytest

import gated_delta_linear_b200 as G
import workloads as W

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "hyb_attn.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(hyb_attn_\w+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    names = declared_functions()
    assert len(names) >= 5, names
    for n in names:
        assert hasattr(G.lib, n), f"{n} declared in hyb_attn.h but not exported"


def test_status_strings():
    for code in (G.HYB_OK, G.HYB_WARN_NONFINITE, G.HYB_ERR_INVALID, G.HYB_ERR_UNSUPPORTED,
                 G.HYB_ERR_ALIGN, G.HYB_ERR_WORKSPACE, G.HYB_ERR_CUDA, G.HYB_ERR_TIMEOUT):
        s = G.hyb_attn_status_string(code)
        assert s.startswith("HYB_")
    assert "unknown" in G.hyb_attn_status_string(42)


def _desc(w):
    return G.make_desc(w.B, w.H, w.T, w.d, G.HYB_BF16 if w.dtype == "bf16" else G.HYB_FP32)


def test_workspace_sizes():
    for w in W.WORKLOADS.values():
        n = G.hyb_attn_workspace_bytes(_desc(w))
        BH = w.B * w.H
        assert n >= 256 + BH * w.d * w.d * 4 * 2, (w.name, n)   # W split + S_{N-1} copy
        assert n % 256 == 0
        # does not grow with the frame count: nothing in the descriptor names frames
        assert n < 64 * 2**20, (w.name, n)
    # unsupported (dtype, d) pairs and bad descriptors size to 0
    assert G.hyb_attn_workspace_bytes(G.make_desc(1, 2, 64, 32, G.HYB_BF16)) == 0
    assert G.hyb_attn_workspace_bytes(G.make_desc(1, 2, 64, 128, G.HYB_FP32)) == 0
    d = G.make_desc(1, 2, 64, 128)
    d.d_v = 64
    assert G.hyb_attn_workspace_bytes(d) == 0
    assert G.hyb_attn_workspace_bytes(G.make_desc(0, 2, 64, 128)) == 0
    assert G.hyb_attn_workspace_bytes(G.make_desc(1, 2, 0, 128)) == 0
    assert G.hyb_attn_workspace_bytes(G.make_desc(1, 2, 64, 128, dtype=7)) == 0
    assert G.hyb_attn_workspace_bytes(G.make_desc(1, 2, 64, 128, l2_eps=-1.0)) == 0


FAKE = 0x10000  # 16-byte aligned fake addresses: never dereferenced on these paths


def _call(desc, **over):
    args = dict(q=FAKE, k=FAKE, v=FAKE, phi_q=FAKE, phi_k=FAKE, phi_v=FAKE, gate_logits=FAKE,
                beta_logits=FAKE, state=FAKE, clean_pass=1, out=FAKE, workspace=FAKE,
                workspace_bytes=1 << 40, stream=0)
    args.update(over)
    return G.hyb_attn_forward(desc, **args)


def test_host_validation_rejects_before_launch():
    d = G.make_desc(1, 12, 1560, 128)
    assert G.lib.hyb_attn_forward(None, *([None] * 9), 0, None, None, 0, None) == G.HYB_ERR_INVALID
    assert _call(G.make_desc(1, 12, 1560, 64)) == G.HYB_ERR_UNSUPPORTED
    assert _call(G.make_desc(1, 12, 0, 128)) == G.HYB_ERR_INVALID
    assert _call(d, q=None) == G.HYB_ERR_INVALID
    assert _call(d, out=None) == G.HYB_ERR_INVALID
    assert _call(d, state=None) == G.HYB_ERR_INVALID
    assert _call(d, gate_logits=None) == G.HYB_ERR_INVALID
    assert _call(d, clean_pass=2) == G.HYB_ERR_INVALID
    assert _call(d, k=FAKE + 2) == G.HYB_ERR_ALIGN
    assert _call(d, state=FAKE + 8) == G.HYB_ERR_ALIGN
    assert _call(d, workspace=None) == G.HYB_ERR_WORKSPACE
    need = G.hyb_attn_workspace_bytes(d)
    assert _call(d, workspace_bytes=need - 1) == G.HYB_ERR_WORKSPACE
    # query-only passes do not need gates
    assert _call(d, clean_pass=0, gate_logits=None, beta_logits=None,
                 workspace_bytes=need - 1) == G.HYB_ERR_WORKSPACE
    # the branch entry point needs both fp32 outputs
    assert G.hyb_attn_forward_branches(d, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1,
                                       FAKE, None, FAKE, FAKE, 1 << 40, 0) == G.HYB_ERR_INVALID
    assert G.hyb_attn_get_device_status(None, 0) == G.HYB_ERR_INVALID
    assert G.hyb_attn_get_device_status(FAKE + 4, 0) == G.HYB_ERR_ALIGN


def test_chained_entry_point_validates_like_the_plain_one():
    """hyb_attn_forward_next checks every argument before anything is enqueued,
    with the statuses of hyb_attn_forward (no chain record is kept for a call
    that fails its checks)."""
    d = G.make_desc(1, 12, 1560, 128)

    def nxt(desc=d, **over):
        args = dict(q=FAKE, k=FAKE, v=FAKE, phi_q=FAKE, phi_k=FAKE, phi_v=FAKE, gate_logits=FAKE,
                    beta_logits=FAKE, state=FAKE, clean_pass=1, out=FAKE, workspace=FAKE,
                    workspace_bytes=1 << 40, stream=0)
        args.update(over)
        return G.hyb_attn_forward_next(desc, **args)

    assert G.lib.hyb_attn_forward_next(None, *([None] * 9), 0, None, None, 0, None) == G.HYB_ERR_INVALID
    assert nxt(desc=G.make_desc(1, 12, 1560, 64)) == G.HYB_ERR_UNSUPPORTED
    assert nxt(q=None) == G.HYB_ERR_INVALID
    assert nxt(out=None) == G.HYB_ERR_INVALID
    assert nxt(gate_logits=None) == G.HYB_ERR_INVALID
    assert nxt(clean_pass=2) == G.HYB_ERR_INVALID
    assert nxt(v=FAKE + 2) == G.HYB_ERR_ALIGN
    assert nxt(workspace=None) == G.HYB_ERR_WORKSPACE
    need = G.hyb_attn_workspace_bytes(d)
    assert nxt(workspace_bytes=need - 1) == G.HYB_ERR_WORKSPACE


def test_desc_layout_matches_header():
    # eight 4-byte fields, in the header's order
    assert ctypes.sizeof(G.HybAttnDesc) == 32
    names = [f[0] for f in G.HybAttnDesc._fields_]
    assert names == ["B", "H", "T", "d_k", "d_v", "dtype", "sm_scale", "l2_eps"]


def test_kvcache_host_validation_rejects_before_launch():
    d = G.make_desc(1, 12, 1560, 128)
    ws = FAKE

    def call(desc=d, cache=4 * 1560, cached=0, **over):
        args = dict(q=FAKE, k=FAKE, v=FAKE, kc=FAKE, vc=FAKE, out=FAKE, ws=ws, nbytes=256)
        args.update(over)
        return G.lib.hyb_kvcache_attn_forward(ctypes.byref(desc), args["q"], args["k"], args["v"], args["kc"],
                                              args["vc"], cache, cached, args["out"], args["ws"],
                                              args["nbytes"], None)

    assert G.lib.hyb_kvcache_attn_forward(None, *([None] * 5), 1, 0, None, None, 0, None) == G.HYB_ERR_INVALID
    assert call(cached=3 * 1560 + 1) == G.HYB_ERR_INVALID      # the frame would overflow the cache
    assert call(cached=-1) == G.HYB_ERR_INVALID
    assert call(q=None) == G.HYB_ERR_INVALID
    assert call(vc=None) == G.HYB_ERR_INVALID
    assert call(desc=G.make_desc(1, 12, 1560, 64)) == G.HYB_ERR_UNSUPPORTED
    assert call(desc=G.make_desc(1, 2, 64, 32, G.HYB_FP32)) == G.HYB_ERR_UNSUPPORTED
    assert call(kc=FAKE + 8) == G.HYB_ERR_ALIGN
    assert call(ws=None) == G.HYB_ERR_WORKSPACE
    assert call(nbytes=255) == G.HYB_ERR_WORKSPACE


def test_mixed_entry_requires_weights():
    d = G.make_desc(1, 12, 1560, 128)
    args = [FAKE] * 9
    assert G.lib.hyb_attn_forward_mixed(ctypes.byref(d), *args, 1, None, FAKE, FAKE, 1 << 40, None) \
        == G.HYB_ERR_INVALID
    assert G.lib.hyb_attn_forward_mixed(ctypes.byref(d), *args, 1, FAKE, None, FAKE, 1 << 40, None) \
        == G.HYB_ERR_INVALID
    assert G.lib.hyb_attn_forward_mixed(ctypes.byref(d), *args, 1, FAKE + 8, FAKE, FAKE, 1 << 40, None) \
        == G.HYB_ERR_ALIGN


def test_tra_host_validation_rejects_before_launch():
    d = G.make_desc(1, 12, 1560, 128)
    ok = G.HybTraParams(30, 52, 8, 16, 0.15, 2)
    need = G.hyb_tra_workspace_bytes(d)
    assert need > G.hyb_attn_workspace_bytes(d)
    assert G.hyb_tra_workspace_bytes(G.make_desc(1, 2, 64, 32, G.HYB_FP32)) == 0

    def call(params=ok, warmup=0, ent=FAKE, nbytes=need, desc=d):
        return G.hyb_tra_forward(desc, params, warmup, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1,
                                 FAKE, ent, FAKE, nbytes, 0)

    assert call(params=G.HybTraParams(30, 51, 8, 16, 0.15, 2)) == G.HYB_ERR_INVALID   # grid != T
    assert call(params=G.HybTraParams(30, 52, 8, 16, 0.0, 2)) == G.HYB_ERR_INVALID
    assert call(params=G.HybTraParams(30, 52, 8, 16, 0.15, 0)) == G.HYB_ERR_INVALID
    assert call(warmup=2) == G.HYB_ERR_INVALID
    assert call(ent=None) == G.HYB_ERR_INVALID
    assert call(ent=FAKE + 4) == G.HYB_ERR_ALIGN
    assert call(nbytes=need - 1) == G.HYB_ERR_WORKSPACE
    assert call(desc=G.make_desc(1, 2, 64, 32, G.HYB_FP32)) == G.HYB_ERR_UNSUPPORTED
    # the mask kernel's shared memory holds at most 221 key blocks (T <= 28288)
    big = G.make_desc(1, 1, 28289, 128)
    assert call(desc=big, params=G.HybTraParams(1, 28289, 1, 16, 0.15, 2), nbytes=1 << 40) == \
        G.HYB_ERR_UNSUPPORTED
