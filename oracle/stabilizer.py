"""Stabilizer construction: the frozen full-precision low-rank branch and the
residual weight that is quantized.

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).

FourTune §3.1 isolates a quantization-sensitive low-rank component of each
backbone weight into a frozen full-precision branch (the numerical stabilizer)
and quantizes only what remains; the pages cite SVDQuant for that step and give
no further detail.  Readings (the plainest ones the rest of the pages support):
  * W [N, K] is the backbone weight of y = X W^T.  The stabilizer is the rank-r_s
    truncated SVD of W^T: with W^T = U diag(s) V^T (s descending),
    S_dn = U[:, :r_s] diag(sqrt(s[:r_s]))   [K, r_s]
    S_up = diag(sqrt(s[:r_s])) V[:, :r_s]^T [r_s, N]
    (the singular values split evenly between the two factors).
  * The factors are stored in bf16 (nearest-even), like the layer's other
    low-rank factors; the residual is taken against the rounded factors, so
    that W = R + (S_dn S_up)^T up to R's own rounding:
    R = bf16(W - (S_dn S_up)^T), computed exactly (float64) and rounded once.
  * R is then quantized by the block16 quantizer (block16.quantize).
A library SVD (numpy, float64) is the one primitive used.
"""
import numpy as np

from . import block16, formats


def truncated_factors(W, r_s):
    """Unrounded rank-r_s factors (S_dn [K, r_s], S_up [r_s, N]) of W^T, float64."""
    Wt = np.asarray(W, dtype=np.float64).T
    U, s, Vt = np.linalg.svd(Wt, full_matrices=False)
    root = np.sqrt(s[:r_s])
    return U[:, :r_s] * root[None, :], root[:, None] * Vt[:r_s, :]


def split(W, r_s):
    """Returns dict(S_dn, S_up (bf16 values), R (bf16 values) [N, K], R_codes, R_scales)."""
    S_dn, S_up = truncated_factors(W, r_s)
    S_dn = formats.bf16_round(S_dn)
    S_up = formats.bf16_round(S_up)
    R = residual(W, S_dn, S_up)
    codes, scales = block16.quantize(R.astype(np.float32))
    return dict(S_dn=S_dn, S_up=S_up, R=R, R_codes=codes, R_scales=scales)


def residual(W, S_dn, S_up):
    """R = bf16(W - (S_dn S_up)^T), the subtraction exact before the one rounding."""
    return formats.bf16_round(np.asarray(W, dtype=np.float64) - (np.asarray(S_dn, np.float64) @
                                                                 np.asarray(S_up, np.float64)).T)
