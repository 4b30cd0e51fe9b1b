"""1x16 group-wise NVFP4 quantizer with a per-tensor scale (the ablation format).

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).

FourTune §4.3 "Impact of Quantization Granularity" (Table 5) compares its 16x16
blocks with the finer group-wise layout, 1x16: each row's 16 consecutive
elements along the reduction dimension share one scale.  §2.3 names NVFP4, whose
full form scales twice: one FP32 scale for the whole tensor and one E4M3 scale
per 16 elements, with W~ = Round(W / s).  A transposed operand cannot reuse
these groups (they run along the other dimension), so the backward's R^T is
quantized on its own (§3.2's contrast with the block layout).

Readings (the pages fix neither):
  * per-tensor scale s_t = 2^e, the smallest power of two with
    amax(T) / (6 * 2^e) <= 448 (the E4M3 maximum), i.e. the power of two at or
    above amax / 2688; amax = 0 gives e = 0, and e is at least -126 (so that
    2^-e is a float32 number; only a tensor whose largest magnitude is below
    2688 * 2^-127 ~ 1e-35 meets the bound).  A power of two keeps every step
    below exact: T' = T * 2^-e changes no significand (float32 rounding only
    if an element lands below 2^-126), and the GEMM's output scale
    s_tA * s_tB is an exact multiply.
  * per 1x16 group of T' (the layer's rules of the block layout, one row):
      a  = max |t'| over the group                  (exact)
      s  = fp32(a) / 6                              (IEEE float32 division)
      sc = E4M3(s)   ties-to-even, subnormals kept, saturate at 448
      if value(sc) == 0: every code is +0
      else: code = E2M1(fp32(t') / value(sc))
  * the value of a code: E2M1(code) * value(sc) * 2^e.
Packing: codes[r, c//2] holds column c in the low nibble when c is even, the
high nibble when c is odd; scales[r, c//16] is one E4M3 byte per group.
"""
import numpy as np

from . import block16, formats

GROUP = 16
E4M3_MAX = 448.0
E2M1_MAX = 6.0


def tensor_exponent(amax: float) -> int:
    """The exponent e of the per-tensor scale 2^e: the least integer with
    amax <= 2688 * 2^e (2688 = 6 * 448), and at least -126; 0 for amax = 0."""
    amax = float(amax)
    if amax == 0.0:
        return 0
    if amax <= E2M1_MAX * E4M3_MAX * 2.0 ** -127:
        return -126
    e = int(np.ceil(np.log2(amax / (E2M1_MAX * E4M3_MAX))))
    # guard the log2 rounding on either side of a power of two
    while amax > E2M1_MAX * E4M3_MAX * 2.0 ** e:
        e += 1
    while amax <= E2M1_MAX * E4M3_MAX * 2.0 ** (e - 1):
        e -= 1
    return e


def quantize_codes(t: np.ndarray, e=None):
    """Quantize a float32-exact [rows, cols] array (cols a multiple of 16).

    Returns (code4 uint8 [rows, cols] unpacked, scales uint8 [rows, cols/16], e).
    `e` may force the per-tensor exponent (default: from the tensor's amax)."""
    t = np.asarray(t)
    rows, cols = t.shape
    if cols % GROUP:
        raise ValueError(f"1x16 groups need cols that are a multiple of 16, got {cols}")
    t32 = t.astype(np.float32)
    if not np.array_equal(t32.astype(np.float64), np.asarray(t, dtype=np.float64)):
        raise ValueError("quantize_codes expects float32-exact input")
    if e is None:
        e = tensor_exponent(np.abs(t32).max() if t32.size else 0.0)
    ts = (t32 * np.float32(2.0 ** -e)).astype(np.float32)               # float32 multiply by 2^-e
    groups = ts.reshape(rows, cols // GROUP, GROUP)
    amax = np.abs(groups).max(axis=2)                                    # [rows, cols/16]
    s = (amax.astype(np.float32) / np.float32(6.0)).astype(np.float32)   # float32 division
    scales = formats.e4m3_encode_nonneg(s)
    dec = formats.e4m3_decode(scales).astype(np.float32)                 # exact in float32
    d = np.repeat(dec, GROUP, axis=1)                                    # [rows, cols]
    with np.errstate(divide="ignore", invalid="ignore"):
        q = (ts / np.where(d == 0, np.float32(1.0), d)).astype(np.float32)
    code4 = formats.e2m1_encode(q)
    code4 = np.where(d == 0, np.uint8(0), code4).astype(np.uint8)       # zero scale -> +0 codes
    return code4, scales, e


def quantize(t: np.ndarray, e=None):
    """Quantize and pack: (codes uint8 [rows, cols/2], scales uint8 [rows, cols/16], e)."""
    code4, scales, e = quantize_codes(t, e)
    return block16.pack_codes(code4), scales, e


def dequantize(codes: np.ndarray, scales: np.ndarray, e: int) -> np.ndarray:
    """value = E2M1(code) * E4M3(scale of its group) * 2^e, in float64 (exact)."""
    vals = formats.e2m1_decode(block16.unpack_codes(codes))
    sc = formats.e4m3_decode(scales)
    return vals * np.repeat(sc, GROUP, axis=1) * 2.0 ** e
