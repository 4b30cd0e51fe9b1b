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


def check_bf16_dot(got, ref, absdot, n):
    """A bf16-rounded dot product of length n: the GPU accumulates in fp32, the oracle
    exactly, then both round once.  Elementwise bound: one bf16 ulp of the result plus
    the fp32 accumulation bound n * 2^-24 * sum|a_k b_k| (absdot); and normwise at most
    one bf16 ulp of the largest element's binade (2^-7 of the largest magnitude: a
    rounding flip of an element in the top binade)."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    mag = np.maximum(np.abs(ref), 2.0 ** -126)
    bound = 2.0 ** (np.floor(np.log2(mag)) - 7) + n * 2.0 ** -24 * np.asarray(absdot)
    bad = np.abs(got - ref) > bound
    assert not bad.any(), f"{int(bad.sum())} elements beyond the bf16-dot bound"
    assert normwise(got, ref) <= 2.0 ** -7


# Elementwise bound of an fp32-accumulated sum of n products against its exact
# value: the tensor cores' products of dequantized FP4 or bf16 operands are
# exact, each accumulation step rounds with relative error at most 2^-23 (twice
# the nearest-even unit, for adders that truncate), so the error is at most
# n * 2^-23 * sum_k |a_k b_k| (absdot), plus the final rounding of the stored fp32.
GAMMA_FP32 = 2.0 ** -23


def fp32_dot_bound(absdot, n):
    return n * GAMMA_FP32 * np.asarray(absdot, dtype=np.float64)


def check_fp32_dot(got, ref, absdot, n, extra=0.0, name="output"):
    """fp32 output of an fp32-accumulated product vs the exact (float64) value:
    elementwise |got - ref| <= n 2^-23 absdot + 2^-24 |ref| + extra (extra: a
    caller-stated bound for inputs that were themselves rounded, e.g. a bf16
    intermediate one ulp away).  Returns the largest error / bound ratio (the
    elementwise figure reported next to the normwise one)."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    bound = fp32_dot_bound(absdot, n) + 2.0 ** -24 * np.abs(ref) + np.asarray(extra, dtype=np.float64) + 1e-30
    ratio = np.abs(got - ref) / bound
    worst = float(ratio.max()) if ratio.size else 0.0
    assert worst <= 1.0, f"{name}: {int((ratio > 1).sum())} elements beyond the fp32 accumulation bound " \
                         f"(worst ratio {worst:.3g})"
    return worst


def check_bf16_rounded(got, ref, err_bound, name="output"):
    """bf16 value that is the rounding of a computed quantity whose exact value is
    `ref` and whose error before rounding is at most err_bound (elementwise):
    |got - ref| <= one bf16 ulp at |ref| + err_bound.  Returns the worst ratio."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    mag = np.maximum(np.abs(ref), 2.0 ** -126)
    bound = 2.0 ** (np.floor(np.log2(mag)) - 7) + np.asarray(err_bound, dtype=np.float64) + 1e-38
    ratio = np.abs(got - ref) / bound
    worst = float(ratio.max()) if ratio.size else 0.0
    assert worst <= 1.0, f"{name}: {int((ratio > 1).sum())} elements beyond one bf16 ulp + bound " \
                         f"(worst ratio {worst:.3g})"
    return worst


def nan_dev(shape, dtype=None):
    """Device tensor filled with NaN: an output element a kernel never writes stays NaN."""
    import torch
    return torch.full(shape, float("nan"), dtype=dtype or torch.float32, device="cuda")


def poisoned_ws(nbytes):
    """Workspace filled with 0xFF bytes: the call must clear what it needs (status
    word, counters) and write every intermediate it reads."""
    import torch
    return torch.full((nbytes,), 0xFF, dtype=torch.uint8, device="cuda")


def to_dev_bf16(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to("cuda").to(torch.bfloat16)


def to_host(t):
    import torch
    if t.dtype == torch.bfloat16:
        return t.float().cpu().numpy().astype(np.float64)
    return t.cpu().numpy()


def tie_tensor(rows, cols, seed=0):
    """bf16 values that hit every E2M1 rounding tie exactly: in each 16x16 block
    the largest magnitude is 6 d for an E4M3 value d (so the block scale is d and
    element / scale is exact), the other entries are +-t d for the ties t in
    {0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5} and their bf16 neighbours one ulp
    either side, plus +-0.  d runs over normal and subnormal E4M3 scales."""
    from oracle import formats  # test-side construction only
    rng = np.random.default_rng(seed)
    ties = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
    scodes = [0x01, 0x03, 0x07, 0x08, 0x1B, 0x30, 0x38, 0x3D, 0x4F, 0x66, 0x70]
    t = np.zeros((rows, cols), np.float32)
    for bi in range(rows // 16):
        for bj in range(cols // 16):
            d = formats.E4M3_TABLE[scodes[(bi * 7 + bj) % len(scodes)]]
            vals = np.concatenate([ties * d, -ties * d]).astype(np.float32)
            up = synth.bf16_from_bits(synth.bf16_bits(vals) + np.uint16(1))
            dn = synth.bf16_from_bits(synth.bf16_bits(vals) - np.uint16(1))
            pool = np.concatenate([vals, up, dn, np.float32([0.0, -0.0])])
            blk = rng.choice(pool, size=(16, 16))
            blk[0, 0] = np.float32(6 * d) * rng.choice([-1, 1])
            t[bi * 16:(bi + 1) * 16, bj * 16:(bj + 1) * 16] = blk
    assert np.array_equal(synth.to_bf16(t), t), "tie tensor must be bf16-exact"
    return t


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
