"""ctypes marshalling for libhyb_attn.so (names follow include/hyb_attn.h)."""

from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
library_path = os.path.join(_HERE, "libhyb_attn.so")

HYB_OK = 0
HYB_WARN_NONFINITE = 1
HYB_ERR_INVALID = -1
HYB_ERR_UNSUPPORTED = -2
HYB_ERR_ALIGN = -3
HYB_ERR_WORKSPACE = -4
HYB_ERR_CUDA = -5
HYB_ERR_TIMEOUT = -6

HYB_BF16 = 0
HYB_FP32 = 1


class HybAttnError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {hyb_attn_status_string(status)} ({status})")
        self.status = status


class HybAttnDesc(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int), ("H", ctypes.c_int), ("T", ctypes.c_int),
        ("d_k", ctypes.c_int), ("d_v", ctypes.c_int), ("dtype", ctypes.c_int),
        ("sm_scale", ctypes.c_float), ("l2_eps", ctypes.c_float),
    ]


class HybTraParams(ctypes.Structure):
    _fields_ = [("grid_h", ctypes.c_int), ("grid_w", ctypes.c_int), ("tile_h", ctypes.c_int),
                ("tile_w", ctypes.c_int), ("tau", ctypes.c_float), ("votes_min", ctypes.c_int)]


HYB_NUM_KERNELS = 7


class HybAttnTiming(ctypes.Structure):
    _fields_ = [("launches", ctypes.c_int * HYB_NUM_KERNELS),
                ("total_ms", ctypes.c_double * HYB_NUM_KERNELS),
                ("dropped", ctypes.c_int)]


def _load():
    if not os.path.exists(library_path):
        raise ImportError(
            f"{library_path} is missing: build it with `python gated_delta_linear_b200/build.py`")
    L = ctypes.CDLL(library_path)
    vp, sz, i = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
    dp = ctypes.POINTER(HybAttnDesc)
    L.hyb_attn_workspace_bytes.argtypes = [dp]
    L.hyb_attn_workspace_bytes.restype = sz
    L.hyb_attn_forward.argtypes = [dp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i, vp, vp, sz, vp]
    L.hyb_attn_forward.restype = i
    L.hyb_attn_forward_next.argtypes = [dp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i, vp, vp, sz, vp]
    L.hyb_attn_forward_next.restype = i
    L.hyb_attn_forward_branches.argtypes = [dp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i, vp,
                                            vp, vp, vp, sz, vp]
    L.hyb_attn_forward_branches.restype = i
    L.hyb_attn_forward_noalloc.argtypes = [dp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i, vp, vp]
    L.hyb_attn_forward_noalloc.restype = i
    L.hyb_attn_forward_mixed.argtypes = [dp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i, vp, vp, vp, sz, vp]
    L.hyb_attn_forward_mixed.restype = i
    L.hyb_tra_workspace_bytes.argtypes = [dp]
    L.hyb_tra_workspace_bytes.restype = sz
    L.hyb_tra_forward.argtypes = [dp, ctypes.POINTER(HybTraParams), i, vp, vp, vp, vp, vp, vp, vp, vp, vp, i, vp,
                                  vp, vp, sz, vp]
    L.hyb_tra_forward.restype = i
    L.hyb_attn_frames_workspace_bytes.argtypes = [dp, i]
    L.hyb_attn_frames_workspace_bytes.restype = sz
    L.hyb_attn_forward_frames.argtypes = [dp, i, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    L.hyb_attn_forward_frames.restype = i
    L.hyb_attn_token_level_workspace_bytes.argtypes = [dp]
    L.hyb_attn_token_level_workspace_bytes.restype = sz
    L.hyb_attn_forward_token_level.argtypes = [dp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i, vp, vp, sz, vp]
    L.hyb_attn_forward_token_level.restype = i
    L.hyb_kvcache_attn_forward.argtypes = [dp, vp, vp, vp, vp, vp, i, i, vp, vp, sz, vp]
    L.hyb_kvcache_attn_forward.restype = i
    L.hyb_attn_get_device_status.argtypes = [vp, vp]
    L.hyb_attn_get_device_status.restype = i
    L.hyb_attn_set_fault_test.argtypes = [i, ctypes.c_uint]
    L.hyb_attn_set_fault_test.restype = i
    L.hyb_attn_noalloc_device_status.argtypes = [vp]
    L.hyb_attn_noalloc_device_status.restype = i
    L.hyb_attn_timing_begin.argtypes = [i]
    L.hyb_attn_timing_begin.restype = i
    L.hyb_attn_timing_end.argtypes = [ctypes.POINTER(HybAttnTiming)]
    L.hyb_attn_timing_end.restype = i
    L.hyb_attn_kernel_name.argtypes = [i]
    L.hyb_attn_kernel_name.restype = ctypes.c_char_p
    L.hyb_attn_status_string.argtypes = [i]
    L.hyb_attn_status_string.restype = ctypes.c_char_p
    return L


lib = _load()


def make_desc(B, H, T, d, dtype=HYB_BF16, sm_scale=0.0, l2_eps=1e-6) -> HybAttnDesc:
    return HybAttnDesc(B, H, T, d, d, dtype, sm_scale, l2_eps)


def _ptr(x):
    """A device or host address: None, an int, or a tensor's data pointer."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def hyb_attn_workspace_bytes(desc: HybAttnDesc) -> int:
    return lib.hyb_attn_workspace_bytes(ctypes.byref(desc))


def hyb_attn_forward(desc, q, k, v, phi_q, phi_k, phi_v, gate_logits, beta_logits, state,
                     clean_pass, out, workspace, workspace_bytes=None, stream=None) -> int:
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    return lib.hyb_attn_forward(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(phi_q),
                                _ptr(phi_k), _ptr(phi_v), _ptr(gate_logits), _ptr(beta_logits),
                                _ptr(state), int(clean_pass), _ptr(out), _ptr(workspace),
                                workspace_bytes, _stream(stream))


def hyb_attn_forward_branches(desc, q, k, v, phi_q, phi_k, phi_v, gate_logits, beta_logits,
                              state, clean_pass, out, out_intra, out_inter, workspace,
                              workspace_bytes=None, stream=None) -> int:
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    return lib.hyb_attn_forward_branches(
        ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(phi_q), _ptr(phi_k), _ptr(phi_v),
        _ptr(gate_logits), _ptr(beta_logits), _ptr(state), int(clean_pass), _ptr(out),
        _ptr(out_intra), _ptr(out_inter), _ptr(workspace), workspace_bytes, _stream(stream))


HYB_NOALLOC_SCRATCH_BYTES = 32 << 20


def hyb_attn_forward_noalloc(desc, q, k, v, phi_q, phi_k, phi_v, gate_logits, beta_logits, state,
                             clean_pass, out, stream=None) -> int:
    """hyb_attn_forward without a workspace argument, for callers that cannot
    allocate device memory; uses the library's fixed scratch array instead."""
    return lib.hyb_attn_forward_noalloc(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v),
                                        _ptr(phi_q), _ptr(phi_k), _ptr(phi_v), _ptr(gate_logits),
                                        _ptr(beta_logits), _ptr(state), int(clean_pass), _ptr(out),
                                        _stream(stream))


def hyb_tra_workspace_bytes(desc: HybAttnDesc) -> int:
    return lib.hyb_tra_workspace_bytes(ctypes.byref(desc))


def hyb_tra_forward(desc, params, warmup, q, k, v, phi_q, phi_k, phi_v, gate_logits, beta_logits, state,
                    clean_pass, out, entropy, workspace, workspace_bytes=None, stream=None) -> int:
    """Token Radius Attention pass: warmup=1 is the dense pass that also writes the
    per-query entropies; warmup=0 attends over the key blocks those entropies keep."""
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    return lib.hyb_tra_forward(ctypes.byref(desc), ctypes.byref(params), int(warmup), _ptr(q), _ptr(k), _ptr(v),
                               _ptr(phi_q), _ptr(phi_k), _ptr(phi_v), _ptr(gate_logits), _ptr(beta_logits),
                               _ptr(state), int(clean_pass), _ptr(out), _ptr(entropy), _ptr(workspace),
                               workspace_bytes, _stream(stream))


def hyb_attn_frames_workspace_bytes(desc: HybAttnDesc, n_frames: int) -> int:
    return lib.hyb_attn_frames_workspace_bytes(ctypes.byref(desc), int(n_frames))


def hyb_attn_forward_frames(desc, n_frames, q, k, v, phi_q, phi_k, phi_v, gate_logits, beta_logits, state,
                            out, workspace, workspace_bytes=None, stream=None) -> int:
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    return lib.hyb_attn_forward_frames(ctypes.byref(desc), int(n_frames), _ptr(q), _ptr(k), _ptr(v), _ptr(phi_q),
                                       _ptr(phi_k), _ptr(phi_v), _ptr(gate_logits), _ptr(beta_logits),
                                       _ptr(state), _ptr(out), _ptr(workspace), workspace_bytes, _stream(stream))


def hyb_attn_token_level_workspace_bytes(desc: HybAttnDesc) -> int:
    return lib.hyb_attn_token_level_workspace_bytes(ctypes.byref(desc))


def hyb_attn_forward_token_level(desc, q, k, v, phi_q, phi_k, phi_v, gate_logits, beta_logits, state,
                                 clean_pass, out, workspace, workspace_bytes=None, stream=None) -> int:
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    return lib.hyb_attn_forward_token_level(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(phi_q),
                                            _ptr(phi_k), _ptr(phi_v), _ptr(gate_logits), _ptr(beta_logits),
                                            _ptr(state), int(clean_pass), _ptr(out), _ptr(workspace),
                                            workspace_bytes, _stream(stream))


def hyb_attn_forward_mixed(desc, q, k, v, phi_q, phi_k, phi_v, gate_logits, beta_logits, state,
                           clean_pass, mix, out, workspace, workspace_bytes=None, stream=None) -> int:
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    return lib.hyb_attn_forward_mixed(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(phi_q),
                                      _ptr(phi_k), _ptr(phi_v), _ptr(gate_logits), _ptr(beta_logits),
                                      _ptr(state), int(clean_pass), _ptr(mix), _ptr(out), _ptr(workspace),
                                      workspace_bytes, _stream(stream))


def hyb_kvcache_attn_forward(desc, q, k, v, k_cache, v_cache, cache_tokens, cached_tokens, out,
                             workspace, workspace_bytes=None, stream=None) -> int:
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    return lib.hyb_kvcache_attn_forward(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(k_cache),
                                        _ptr(v_cache), int(cache_tokens), int(cached_tokens), _ptr(out),
                                        _ptr(workspace), workspace_bytes, _stream(stream))


def hyb_attn_get_device_status(workspace, stream=None) -> int:
    return lib.hyb_attn_get_device_status(_ptr(workspace), _stream(stream))


def hyb_attn_status_string(status: int) -> str:
    return lib.hyb_attn_status_string(int(status)).decode()


def hyb_attn_noalloc_device_status(stream=None) -> int:
    """Status flags of the last hyb_attn_forward_noalloc call on the current device."""
    return lib.hyb_attn_noalloc_device_status(_stream(stream))


def hyb_attn_set_fault_test(skip_v_loads: int, wait_limit_us: int) -> int:
    """Test hook (off by default): shorten the attention kernel's bounded waits
    and/or switch off its value-tile loads so that a wait expires."""
    return lib.hyb_attn_set_fault_test(int(skip_v_loads), int(wait_limit_us))


def hyb_attn_timing_begin(max_launches: int) -> int:
    return lib.hyb_attn_timing_begin(int(max_launches))


def hyb_attn_timing_end():
    """Returns (status, {kernel name: (launches, total ms)}, dropped)."""
    t = HybAttnTiming()
    st = lib.hyb_attn_timing_end(ctypes.byref(t))
    per = {hyb_attn_kernel_name(i): (t.launches[i], t.total_ms[i]) for i in range(HYB_NUM_KERNELS)}
    return st, per, t.dropped


def hyb_attn_kernel_name(kernel: int):
    n = lib.hyb_attn_kernel_name(int(kernel))
    return n.decode() if n is not None else None

def hyb_attn_forward_next(desc, q, k, v, phi_q, phi_k, phi_v, gate_logits, beta_logits, state,
                          clean_pass, out, workspace, workspace_bytes=None, stream=None) -> int:
    """hyb_attn_forward continuing the chain of passes on ``workspace`` (the
    next frame's W comes from the previous clean pass's update)."""
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    return lib.hyb_attn_forward_next(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(phi_q),
                                     _ptr(phi_k), _ptr(phi_v), _ptr(gate_logits), _ptr(beta_logits),
                                     _ptr(state), int(clean_pass), _ptr(out), _ptr(workspace),
                                     workspace_bytes, _stream(stream))


class HybridAttention:
    """Owns the device buffers of one layer instance and drives its passes.

    Holds phi_q/phi_k/phi_v, the persistent fp32 state [B, H, d, d] and the
    zero-filled workspace, all allocated with PyTorch on one CUDA device;
    ``forward`` marshals one pass into ``hyb_attn_forward``.
    """

    def __init__(self, B, H, T, d, dtype, phi_q, phi_k, phi_v, device="cuda", sm_scale=0.0,
                 l2_eps=1e-6):
        import torch
        self.desc = make_desc(B, H, T, d, HYB_BF16 if dtype == torch.bfloat16 else HYB_FP32,
                              sm_scale, l2_eps)
        nbytes = hyb_attn_workspace_bytes(self.desc)
        if nbytes == 0:
            raise HybAttnError(HYB_ERR_UNSUPPORTED, "hyb_attn_workspace_bytes")
        self.device = torch.device(device)
        self.dtype = dtype
        self.phi = [p.to(self.device, dtype).contiguous() for p in (phi_q, phi_k, phi_v)]
        self.state = torch.zeros(B, H, d, d, dtype=torch.float32, device=self.device)
        self.workspace = torch.zeros(nbytes, dtype=torch.uint8, device=self.device)

    def forward(self, q, k, v, gate_logits, beta_logits, clean_pass, out=None, stream=None):
        import torch
        if out is None:
            out = torch.empty_like(q)
        st = hyb_attn_forward(self.desc, q, k, v, *self.phi, gate_logits, beta_logits,
                              self.state, clean_pass, out, self.workspace, stream=stream)
        if st != HYB_OK:
            raise HybAttnError(st, "hyb_attn_forward")
        return out

    def forward_next(self, q, k, v, gate_logits, beta_logits, clean_pass, out=None, stream=None):
        """``forward`` through hyb_attn_forward_next: consecutive calls on this
        layer continue one chain (call ``forward`` after resetting the state)."""
        import torch
        if out is None:
            out = torch.empty_like(q)
        st = hyb_attn_forward_next(self.desc, q, k, v, *self.phi, gate_logits, beta_logits,
                                   self.state, clean_pass, out, self.workspace, stream=stream)
        if st != HYB_OK:
            raise HybAttnError(st, "hyb_attn_forward_next")
        return out

    def forward_branches(self, q, k, v, gate_logits, beta_logits, clean_pass, stream=None):
        import torch
        out = torch.empty_like(q)
        oi = torch.empty(q.shape, dtype=torch.float32, device=q.device)
        oe = torch.empty_like(oi)
        st = hyb_attn_forward_branches(self.desc, q, k, v, *self.phi, gate_logits, beta_logits,
                                       self.state, clean_pass, out, oi, oe, self.workspace,
                                       stream=stream)
        if st != HYB_OK:
            raise HybAttnError(st, "hyb_attn_forward_branches")
        return out, oi, oe

    def forward_mixed(self, q, k, v, gate_logits, beta_logits, clean_pass, mix, out=None, stream=None):
        """out = a O_intra + c O_inter with (a, c) = mix[b, h] ([B, H, 2] fp32 on the device)."""
        import torch
        if out is None:
            out = torch.empty_like(q)
        st = hyb_attn_forward_mixed(self.desc, q, k, v, *self.phi, gate_logits, beta_logits, self.state,
                                    clean_pass, mix, out, self.workspace, stream=stream)
        if st != HYB_OK:
            raise HybAttnError(st, "hyb_attn_forward_mixed")
        return out

    def device_status(self, stream=None) -> int:
        return hyb_attn_get_device_status(self.workspace, stream)


class TokenLevelAttention(HybridAttention):
    """The token-level access variant of the layer (tokens update the state one
    after another on a clean pass); the same buffers as HybridAttention with the
    larger workspace hyb_attn_token_level_workspace_bytes asks for."""

    def __init__(self, B, H, T, d, dtype, phi_q, phi_k, phi_v, device="cuda", sm_scale=0.0, l2_eps=1e-6):
        import torch
        super().__init__(B, H, T, d, dtype, phi_q, phi_k, phi_v, device, sm_scale, l2_eps)
        nbytes = hyb_attn_token_level_workspace_bytes(self.desc)
        if nbytes == 0:
            raise HybAttnError(HYB_ERR_UNSUPPORTED, "hyb_attn_token_level_workspace_bytes")
        self.workspace = torch.zeros(nbytes, dtype=torch.uint8, device=self.device)

    def forward(self, q, k, v, gate_logits, beta_logits, clean_pass, out=None, stream=None):
        import torch
        if out is None:
            out = torch.empty_like(q)
        st = hyb_attn_forward_token_level(self.desc, q, k, v, *self.phi, gate_logits, beta_logits, self.state,
                                          clean_pass, out, self.workspace, stream=stream)
        if st != HYB_OK:
            raise HybAttnError(st, "hyb_attn_forward_token_level")
        return out


class KVCacheAttention:
    """The softmax baseline with a growing key/value cache: owns the bf16 caches
    [B, max_frames * T, H, d] and a status workspace; ``forward`` marshals one
    frame into ``hyb_kvcache_attn_forward`` (which appends the frame's k, v and
    attends over every cached token) and advances the cached-token count."""

    def __init__(self, B, H, T, d, max_frames, device="cuda", sm_scale=0.0):
        import torch
        self.desc = make_desc(B, H, T, d, HYB_BF16, sm_scale)
        self.device = torch.device(device)
        self.capacity = max_frames * T
        self.k_cache = torch.zeros(B, self.capacity, H, d, dtype=torch.bfloat16, device=self.device)
        self.v_cache = torch.zeros_like(self.k_cache)
        self.workspace = torch.zeros(256, dtype=torch.uint8, device=self.device)
        self.cached = 0

    def reset(self):
        self.cached = 0

    def cache_bytes(self) -> int:
        """Bytes of key/value cache in use."""
        return 2 * self.k_cache.shape[0] * self.cached * self.k_cache.shape[2] * self.k_cache.shape[3] * 2

    def forward(self, q, k, v, out=None, stream=None):
        import torch
        if out is None:
            out = torch.empty_like(q)
        st = hyb_kvcache_attn_forward(self.desc, q, k, v, self.k_cache, self.v_cache, self.capacity,
                                      self.cached, out, self.workspace, stream=stream)
        if st != HYB_OK:
            raise HybAttnError(st, "hyb_kvcache_attn_forward")
        self.cached += q.shape[1]
        return out

    def device_status(self, stream=None) -> int:
        return hyb_attn_get_device_status(self.workspace, stream)
