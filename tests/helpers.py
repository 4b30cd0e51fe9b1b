"""Shared test helpers: seeded inputs, device upload, the normwise error metric."""
import numpy as np

from bit_lora_fine_b200 import synth

# Output/gradient tolerance: max-normwise relative error  ||g - r||_inf / ||r||_inf.
# The layer spec allows 2e-3 (fp32 accumulation vs float64 on identical dequantized
# operands); bf16 outputs are additionally checked as the rounding of the fp32 path.
TOL = 2e-3


def normwise(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    denom = np.abs(ref).max()
    if denom == 0:
        return float(np.abs(got).max())
    return float(np.abs(got - ref).max() / denom)


def bf16_ulps(got, ref):
    """Largest |got - ref| in units of the bf16 spacing at |ref| (for bf16-rounded
    outputs such as L and P: fp32 accumulation vs float64 may flip a rounding)."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    mag = np.maximum(np.abs(ref), 2.0 ** -126)
    ulp = 2.0 ** (np.floor(np.log2(mag)) - 7)
    return float((np.abs(got - ref) / ulp).max())


def to_dev_bf16(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to("cuda").to(torch.bfloat16)


def to_host(t):
    import torch
    if t.dtype == torch.bfloat16:
        return t.float().cpu().numpy().astype(np.float64)
    return t.cpu().numpy()


def random_layer(K, N, r_s, r, seed=0, w_std=0.02, b_std=1e-3, bias=False, M=None, x_outliers=4):
    """Small seeded layer + input/gradient for edge-case tests (bf16-exact float32 arrays)."""
    rng = np.random.default_rng(seed)
    f = lambda shape, s: synth.to_bf16((rng.standard_normal(shape) * s).astype(np.float32))
    p = dict(R=f((N, K), w_std), S_dn=f((K, r_s), w_std), S_up=f((r_s, N), w_std), A=f((K, r), w_std),
             B=f((r, N), b_std), bias=f((N,), 0.02) if bias else None)
    if M is not None:
        X = rng.standard_normal((M, K)).astype(np.float32)
        if x_outliers:
            X[:, rng.choice(K, size=min(x_outliers, K), replace=False)] *= 20
        p["X"] = synth.to_bf16(X)
        p["dY"] = f((M, N), 1.0)
    return p
