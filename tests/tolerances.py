"""Parity tolerances between the CUDA library and the float64 oracle.

Stated bounds (the layer's specification): max abs error <= 2e-2 and mean abs
error <= 2e-3 on outputs for bf16 I/O with fp32 accumulation; state relative
Frobenius error <= 1e-3 after 21 frames (bf16 workloads) and <= 1e-4 for the
fp32 workload.

Reading for outputs that are not O(1).  The frame-level delta rule grows S
geometrically on these synthetic inputs (|S|_F ~ 2.5e2 after frame 0 and ~6e17
after frame 20 on the 480p workload), so O_inter and the output reach 1e17 and
no bf16 result can meet an absolute 2e-2.  The bounds are therefore applied
per (frame, pass, batch, head) in units of the output's own magnitude:

    max |got - ref|  <= 2e-2 * max(1, max |ref|)
    mean |got - ref| <= 2e-3 * max(1, mean |ref|)

which is exactly the stated absolute test wherever |ref| <= 1.  The reference
is the unrounded float64 oracle value.  Rounding a correct result once to
bf16 alone costs up to 2^-8 = 3.9e-3 of max|ref| and about 1.4e-3 of mean|ref|
(measured on the 480p workload), so both bounds keep headroom above that
floor, while a dropped term, a transposed map or a wrong sign moves the output
by O(|ref|).  (Scaling by rms(ref) instead leaves no headroom: bf16 rounding
alone reaches 1.6e-2 * rms.)

Branch outputs (fp32, from hyb_attn_forward_branches) get bounds derived from
the tensor-core arithmetic: the intra branch rounds the softmax weights P to
bf16 before P V (relative rounding <= 2^-8, rms ~1.6e-3 of |O_intra|), so
max <= 1e-2 * max|ref| and mean <= 4e-3 * mean|ref|; the inter branch reads the
state through a two-term bf16 split (~2^-16 relative) and a state that itself
agrees to ~1e-5, so max <= 2e-3 * max|ref| and mean <= 5e-4 * mean|ref|.  The
fp32 SIMT workload computes everything in fp32: 1e-4 (max) and 1e-5 (mean)
relative to the same scales.
"""

import numpy as np

OUT_BF16 = (2e-2, 2e-3)
OUT_FP32 = (1e-4, 1e-5)
INTRA_BF16 = (1e-2, 4e-3)
INTER_BF16 = (2e-3, 5e-4)
BRANCH_FP32 = (1e-4, 1e-5)
STATE_BF16 = 1e-3
STATE_FP32 = 1e-4


def scaled_errors(got, ref, floor=1.0):
    """(max|d| / max(floor, max|ref|), mean|d| / max(floor, mean|ref|))."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    d = np.abs(got - ref)
    a = np.abs(ref)
    return d.max() / max(floor, a.max()), d.mean() / max(floor, a.mean())


def relative_errors(got, ref):
    """(max|d| / max|ref|, mean|d| / mean|ref|): no floor (for branch checks)."""
    return scaled_errors(got, ref, floor=np.finfo(np.float64).tiny)


def rel_frobenius(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    n = np.linalg.norm(ref)
    return np.linalg.norm(got - ref) / (n if n > 0 else 1.0)


def check(errs, bounds, what):
    mx, mn = errs
    assert mx <= bounds[0] and mn <= bounds[1], \
        f"{what}: max {mx:.3e} (bound {bounds[0]:.0e}), mean {mn:.3e} (bound {bounds[1]:.0e})"
