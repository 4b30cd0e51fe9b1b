"""Offline preparation of a frozen backbone weight: the stabilizer split.

FourTune §3.1 isolates a frozen full-precision low-rank component of each
backbone weight (the numerical stabilizer) and quantizes only the remainder;
the pages cite SVDQuant for the split.  Read as the rank-r_s truncated SVD of
W^T with the singular values split evenly between the two factors:
    W^T ~ S_dn S_up,  S_dn = U_r sqrt(s_r) [K, r_s],  S_up = sqrt(s_r) V_r^T [r_s, N]
stored in bf16, and the residual R = bf16(W - (S_dn S_up)^T) that is then
block16-quantized.  This runs once per weight, before training, off the hot
path: the factorization is a library SVD on the GPU (torch.linalg.svd, float32),
the residual and its quantization are this library's kernels
(fourtune_stabilizer_residual, fourtune_quantize_block16).
"""
import torch

from . import fourtune as ft


def stabilizer_split(W, r_s):
    """W [N, K] bf16 on the GPU -> (S_dn [K, r_s], S_up [r_s, N], R [N, K]) bf16."""
    if W.dim() != 2 or not W.is_cuda or W.dtype != torch.bfloat16:
        raise ValueError("W must be a 2-D CUDA bfloat16 tensor")
    N, K = W.shape
    if not 1 <= r_s <= min(N, K, 128):
        raise ValueError(f"r_s must be in 1..min(N, K, 128), got {r_s}")
    U, s, Vh = torch.linalg.svd(W.float().t(), full_matrices=False)      # W^T = U diag(s) Vh
    root = s[:r_s].sqrt()
    S_dn = (U[:, :r_s] * root[None, :]).to(torch.bfloat16).contiguous()
    S_up = (root[:, None] * Vh[:r_s, :]).to(torch.bfloat16).contiguous()
    R = ft.stabilizer_residual(W.contiguous(), S_dn, S_up)
    return S_dn, S_up, R


def linear_from_dense(W, r_s, A, B, bias=None):
    """A 4-bit triple-branch layer from a dense bf16 weight W [N, K]: the stabilizer
    split, the residual's block16 quantization, and the adapter A [K, r], B [r, N]."""
    S_dn, S_up, R = stabilizer_split(W, r_s)
    return ft.Linear.from_weights(R, S_dn, S_up, A, B, bias)
