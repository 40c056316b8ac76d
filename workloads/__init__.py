"""Seeded synthetic inputs for the hybrid attention layer's five workloads.

This module only draws random numbers and rounds them to the I/O precision.
It holds none of the layer's arithmetic, so the CPU oracle and the CUDA
library can both be fed from it without sharing any of the method.

Shapes follow the video-DiT settings of the ARL2 summary
(gist.science/ar/paper/2605.16579): §1 (5 s of 480p video) and §4 (a 1.3B
model, up to 921 frames); 480p at Wan's patching gives 30x52 = 1560 tokens per
latent frame and 720p gives 45x80 = 3600.  Values are standard normals; the
per-head 1x1 feature maps start near identity, ``I + N(0, 0.02^2)``.

Every tensor of every pass has its own seed:
``SeedSequence(20261202, spawn_key=(workload, frame, pass, tensor))`` feeding
NumPy's PCG64.  Values are drawn in float32 and, for bf16 workloads, rounded
once to bfloat16 (round-to-nearest-even) by PyTorch.  Gate logits stay fp32.
"""

from __future__ import annotations

from dataclasses import dataclass, field
from typing import Tuple

import numpy as np
import torch

ROOT_SEED = 20261202

# tensor ids inside a seed key
_Q, _K, _V, _G, _BETA, _PHI_Q, _PHI_K, _PHI_V = range(8)


@dataclass(frozen=True)
class Workload:
    """One synthetic workload of the hybrid layer."""
    wid: int
    name: str
    B: int
    H: int
    d: int
    T: int
    frames: int
    dtype: str                     # "bf16" or "fp32": dtype of q/k/v/phi/out
    passes: Tuple[bool, ...]       # per frame: False = query-only, True = clean pass
    gate_mu: float = 2.0
    gate_sd: float = 1.0
    beta_mu: float = 0.0
    beta_sd: float = 1.0
    phi_sd: float = 0.02
    prior_frames: int = 0          # frames folded into the initial state (clean passes)
    pool: int = 0                  # >0: frame n reuses the inputs of frame n % pool
    note: str = field(default="", compare=False)

    @property
    def tokens_per_frame(self) -> int:
        return self.B * self.T

    @property
    def torch_dtype(self):
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32


WORKLOADS = {
    0: Workload(0, "tiny_fp32_B1_H2_d32_4x64", B=1, H=2, d=32, T=64, frames=4, dtype="fp32",
                passes=(False, False, True),
                note="2 query-only denoise passes then 1 clean pass per frame"),
    1: Workload(1, "wan1.3b_480p_B1_H12_d128_21x1560", B=1, H=12, d=128, T=1560, frames=21,
                dtype="bf16", passes=(True,),
                note="480p 5 s: 21 latent frames of 30x52 patches; clean pass every frame"),
    2: Workload(2, "wan14b_stream_step_B1_H40_d128_1x1560", B=1, H=40, d=128, T=1560, frames=1,
                dtype="bf16", passes=(False, False, False, False, True), prior_frames=20,
                note="one frame: 4 query-only passes + 1 clean pass on a state built "
                     "from 20 prior frames"),
    3: Workload(3, "720p_B1_H40_d128_21x3600", B=1, H=40, d=128, T=3600, frames=21,
                dtype="bf16", passes=(True,),
                note="720p: 21 latent frames of 45x80 patches"),
    4: Workload(4, "long_stream_B2_H12_d128_240x1560", B=2, H=12, d=128, T=1560, frames=240,
                dtype="bf16", passes=(True,), gate_mu=3.0, beta_mu=-1.0, pool=8,
                note="240 frames cycling a pool of 8 distinct frames"),
}


def _rng(wid: int, frame: int, pass_idx: int, tensor: int) -> np.random.Generator:
    # frames may be negative (prior frames of workload 2): shift keys to stay >= 0
    ss = np.random.SeedSequence(ROOT_SEED, spawn_key=(wid, frame + 1000, pass_idx, tensor))
    return np.random.Generator(np.random.PCG64(ss))


def _normal(wid, frame, pass_idx, tensor, shape, mu=0.0, sd=1.0) -> np.ndarray:
    x = _rng(wid, frame, pass_idx, tensor).standard_normal(shape, dtype=np.float32)
    if mu != 0.0 or sd != 1.0:
        x = (x * np.float32(sd) + np.float32(mu)).astype(np.float32)
    return x


def _round(x: np.ndarray, dtype: str) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(x))
    return t.to(torch.bfloat16) if dtype == "bf16" else t


@dataclass
class PassInputs:
    """Inputs of one pass, as rounded torch CPU tensors (the values both sides see)."""
    q: torch.Tensor            # [B, T, H, d]
    k: torch.Tensor
    v: torch.Tensor
    gate_logits: torch.Tensor  # [B, H, T] fp32
    beta_logits: torch.Tensor  # [B, H, T] fp32

    def as_f64(self):
        """The same values as float64 NumPy arrays (for the oracle)."""
        f = lambda t: t.to(torch.float64).numpy()
        return f(self.q), f(self.k), f(self.v), f(self.gate_logits), f(self.beta_logits)


def feature_maps(w: Workload):
    """phi_q, phi_k, phi_v: [H, d, d] each, I + N(0, phi_sd^2), rounded to the I/O dtype."""
    eye = np.eye(w.d, dtype=np.float32)[None]
    out = []
    for tid in (_PHI_Q, _PHI_K, _PHI_V):
        x = eye + _normal(w.wid, -1000, 0, tid, (w.H, w.d, w.d), sd=w.phi_sd)
        out.append(_round(x.astype(np.float32), w.dtype))
    return tuple(out)


def pass_inputs(w: Workload, frame: int, pass_idx: int) -> PassInputs:
    """Seeded inputs of one pass of one frame (fresh q/k/v per denoising pass)."""
    src = frame % w.pool if (w.pool and frame >= 0) else frame
    shape = (w.B, w.T, w.H, w.d)
    q = _round(_normal(w.wid, src, pass_idx, _Q, shape), w.dtype)
    k = _round(_normal(w.wid, src, pass_idx, _K, shape), w.dtype)
    v = _round(_normal(w.wid, src, pass_idx, _V, shape), w.dtype)
    gshape = (w.B, w.H, w.T)
    g = torch.from_numpy(_normal(w.wid, src, pass_idx, _G, gshape, w.gate_mu, w.gate_sd))
    bl = torch.from_numpy(_normal(w.wid, src, pass_idx, _BETA, gshape, w.beta_mu, w.beta_sd))
    return PassInputs(q, k, v, g, bl)


def prior_frame_inputs(w: Workload, j: int) -> PassInputs:
    """Inputs of prior frame j (0 <= j < prior_frames) used to build the initial state."""
    return pass_inputs(w, -(w.prior_frames - j), 0)


def zero_state(w: Workload) -> np.ndarray:
    return np.zeros((w.B, w.H, w.d, w.d), dtype=np.float64)


def small_workload(base: Workload, **changes) -> Workload:
    """A reduced copy of a workload (e.g. fewer frames or heads) with its own id space."""
    fields = dict(base.__dict__)
    fields.update(changes)
    return Workload(**fields)
