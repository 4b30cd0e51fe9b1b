"""16x16 block FP4 quantizer, dequantizer and transposed packing.

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).

Follows FourTune §3.2 (block-wise quantization: each block carries its own
scale, so a transposed read fetches the same block and the same scale, and
Q(G)Q(R)^T needs no dequantize/requantize) and §4.3 "Impact of Quantization
Granularity" (16x16 blocks instead of 1x16 groups), with §2.3's W~ = Round(W/s).

Per 16x16 block of a float32-exact tensor T (the layer's readings of the
pages, which leave the arithmetic open):
  a  = max |t| over the block                      (exact)
  s  = fp32(a) / 6                                 (IEEE float32 division)
  sc = E4M3(s)   ties-to-even, subnormals kept, saturate at 448
  if value(sc) == 0: every code is +0
  else: code = E2M1(fp32(t) / value(sc))  (float32 division, ties-to-even,
        saturate at +-6, sign bit kept so small negatives give 0x8)
Packing: codes[r, c//2] holds column c in the low nibble when c is even, the
high nibble when c is odd.  scales[r//16, c//16] is one E4M3 byte per block.
"""
import numpy as np

from . import formats

BLOCK = 16


def _check_shape(rows: int, cols: int):
    if rows % BLOCK or cols % BLOCK:
        raise ValueError(f"block16 needs rows and cols that are multiples of 16, got {rows}x{cols}")


def quantize_codes(t: np.ndarray):
    """Quantize a float32-exact [rows, cols] array.

    Returns (code4, scales): code4 is uint8 [rows, cols] with one 4-bit code per
    element (unpacked), scales is uint8 [rows/16, cols/16].
    """
    t = np.asarray(t)
    rows, cols = t.shape
    _check_shape(rows, cols)
    t32 = t.astype(np.float32)
    if not np.array_equal(t32.astype(np.float64), np.asarray(t, dtype=np.float64)):
        raise ValueError("quantize_codes expects float32-exact input")
    blocks = t32.reshape(rows // BLOCK, BLOCK, cols // BLOCK, BLOCK)
    amax = np.abs(blocks).max(axis=(1, 3))                               # [rb, cb] float32
    s = (amax.astype(np.float32) / np.float32(6.0)).astype(np.float32)   # float32 division
    scales = formats.e4m3_encode_nonneg(s)
    dec = formats.e4m3_decode(scales).astype(np.float32)                 # exact in float32
    code4 = np.zeros((rows, cols), dtype=np.uint8)
    # process in row stripes to bound memory
    for rb in range(rows // BLOCK):
        stripe = t32[rb * BLOCK:(rb + 1) * BLOCK]                         # [16, cols]
        d = np.repeat(dec[rb], BLOCK)[None, :]                            # [1, cols]
        with np.errstate(divide="ignore", invalid="ignore"):
            q = (stripe / np.where(d == 0, np.float32(1.0), d)).astype(np.float32)
        c = formats.e2m1_encode(q)
        c = np.where(d == 0, np.uint8(0), c)                              # zero scale -> +0 codes
        code4[rb * BLOCK:(rb + 1) * BLOCK] = c
    return code4, scales


def pack_codes(code4: np.ndarray) -> np.ndarray:
    """[rows, cols] 4-bit codes -> [rows, cols/2] bytes, even column in the low nibble."""
    code4 = np.asarray(code4, dtype=np.uint8)
    return (code4[:, 0::2] & 0xF) | ((code4[:, 1::2] & 0xF) << 4)


def unpack_codes(packed: np.ndarray) -> np.ndarray:
    packed = np.asarray(packed, dtype=np.uint8)
    rows, half = packed.shape
    out = np.empty((rows, half * 2), dtype=np.uint8)
    out[:, 0::2] = packed & 0xF
    out[:, 1::2] = packed >> 4
    return out


def quantize(t: np.ndarray):
    """Quantize and pack: returns (codes uint8 [rows, cols/2], scales uint8 [rows/16, cols/16])."""
    code4, scales = quantize_codes(t)
    return pack_codes(code4), scales


def dequantize(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """value = E2M1(code) * E4M3(scale of its block), in float64 (exact)."""
    code4 = unpack_codes(codes)
    vals = formats.e2m1_decode(code4)
    sc = formats.e4m3_decode(scales)
    return vals * np.repeat(np.repeat(sc, BLOCK, axis=0), BLOCK, axis=1)


def transpose_pack(codes: np.ndarray) -> np.ndarray:
    """Codes of T^T from the codes of T: the same 4-bit codes, nibble-transposed.

    The scales of T^T are scales.T (the same bytes): §3.2's point that a
    transposed block reuses its code and scale with no requantization.
    """
    return pack_codes(unpack_codes(codes).T)
