"""E2M1 and E4M3 number formats, written out from their definitions.

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).

FourTune §2.3 names NVFP4 as the hardware format and writes quantization as
W~ = Round(W / s); §3.1 quantizes the residual weights to NVFP4.  NVFP4 elements
are FP4 E2M1 (1 sign, 2 exponent, 1 mantissa bit, bias 1, no inf/NaN) and the
block scale is FP8 E4M3 (1 sign, 4 exponent, 3 mantissa bits, bias 7, the
all-ones pattern 0x7F/0xFF is NaN, no inf, maximum finite 448).

Rounding is round-to-nearest with ties to the even code (the code whose least
significant bit is 0), and values beyond the largest finite magnitude saturate
to it.  Both encoders below are literal "pick the nearest table entry" searches,
so the definition can be checked by eye.
"""
import numpy as np

# --------------------------------------------------------------------------- E2M1
# code c in 0..15: bit 3 = sign, bits 2..1 = exponent e, bit 0 = mantissa m.
#   e == 0  -> subnormal: m * 0.5
#   e >  0  -> normal:    (1 + m/2) * 2**(e-1)


def e2m1_value(code: int) -> float:
    """Exact value of a 4-bit E2M1 code (sign bit honoured, -0 stays -0)."""
    sign = -1.0 if code & 0x8 else 1.0
    e = (code >> 1) & 0x3
    m = code & 0x1
    mag = m * 0.5 if e == 0 else (1.0 + m / 2.0) * 2.0 ** (e - 1)
    return sign * mag


E2M1_TABLE = np.array([e2m1_value(c) for c in range(16)], dtype=np.float64)
E2M1_MAGNITUDES = E2M1_TABLE[:8].copy()          # 0, .5, 1, 1.5, 2, 3, 4, 6
E2M1_MAX = 6.0


def e2m1_encode(v: np.ndarray) -> np.ndarray:
    """Round float values to E2M1 codes: nearest magnitude, ties to the even code,
    saturating at 6; the sign bit is copied from the input (so -0.1 -> 0x8).

    `v` must hold exact float32 values (they are compared in float64).
    """
    v = np.asarray(v, dtype=np.float64)
    mag = np.minimum(np.abs(v), E2M1_MAX)                      # saturate first
    dist = np.abs(mag[..., None] - E2M1_MAGNITUDES)            # [..., 8]
    best = dist.min(axis=-1, keepdims=True)
    tied = dist == best
    # among the nearest candidates prefer an even code; there are at most two
    # candidates and they are adjacent codes, so exactly one is even.
    even = tied & ((np.arange(8) & 1) == 0)
    code = np.where(even.any(axis=-1), even.argmax(axis=-1), tied.argmax(axis=-1))
    sign = np.signbit(v).astype(np.uint8) << 3
    return (code.astype(np.uint8) | sign).astype(np.uint8)


# --------------------------------------------------------------------------- E4M3
# code c in 0..255: bit 7 sign, bits 6..3 exponent e, bits 2..0 mantissa m.
#   e == 0            -> subnormal: m/8 * 2**-6
#   e in 1..15        -> normal:    (1 + m/8) * 2**(e-7)
#   e == 15, m == 7   -> NaN (0x7F, 0xFF)


def e4m3_value(code: int) -> float:
    """Exact value of an 8-bit E4M3 code (the 'fn' variant: no infinities)."""
    sign = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    mag = (m / 8.0) * 2.0 ** -6 if e == 0 else (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return sign * mag


E4M3_TABLE = np.array([e4m3_value(c) for c in range(256)], dtype=np.float64)
E4M3_MAX = 448.0
E4M3_MIN_SUBNORMAL = 2.0 ** -9
# non-negative finite codes 0x00..0x7E in increasing value order
_E4M3_POS = E4M3_TABLE[:0x7F].copy()


def e4m3_encode_nonneg(s: np.ndarray) -> np.ndarray:
    """Round non-negative values to E4M3 codes 0x00..0x7E: nearest finite value,
    ties to the even code, saturating at 448 (code 0x7E).

    Block scales are amax/6 >= 0, so only the non-negative half of the table is
    searched.  `s` must hold exact float32 values.
    """
    s = np.asarray(s, dtype=np.float64)
    if np.any(s < 0) or np.any(np.isnan(s)):
        raise ValueError("e4m3_encode_nonneg expects finite non-negative input")
    flat = np.minimum(s.reshape(-1), E4M3_MAX)                 # saturate first
    out = np.empty(flat.shape, dtype=np.uint8)
    step = 1 << 16
    codes = np.arange(0x7F)
    for i in range(0, flat.size, step):
        chunk = flat[i:i + step]
        dist = np.abs(chunk[:, None] - _E4M3_POS)                 # [n, 127]
        best = dist.min(axis=1, keepdims=True)
        tied = dist == best
        even = tied & ((codes & 1) == 0)
        out[i:i + step] = np.where(even.any(axis=1), even.argmax(axis=1), tied.argmax(axis=1))
    return out.reshape(s.shape)


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    return E4M3_TABLE[np.asarray(codes, dtype=np.uint8)]


def e2m1_decode(codes: np.ndarray) -> np.ndarray:
    return E2M1_TABLE[np.asarray(codes, dtype=np.uint8) & 0xF]


# --------------------------------------------------------------------------- bf16
def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round float64 values to the nearest bfloat16 (ties to even), returned as
    float64.  bfloat16 keeps 8 significant bits and float32's exponent range.

    Written from the definition: scale each value into [2**7, 2**8) by its
    binade, round the significand with numpy's round-half-to-even, scale back.
    Below 2**-126 the spacing stays 2**-133 (bfloat16 subnormals); values past
    the largest finite bfloat16 are not expected and the assert checks it.
    Rounding keeps the sign of zero (IEEE 754): -0.0 stays -0.0, and a negative
    value below half the smallest subnormal rounds to -0.0.
    """
    x = np.asarray(x, dtype=np.float64)
    out = x.copy()                      # zeros pass through with their sign
    nz = x != 0
    if np.any(nz):
        v = x[nz]
        e = np.floor(np.log2(np.abs(v)))
        # guard log2 rounding at exact powers of two
        e = np.where(np.abs(v) >= 2.0 ** (e + 1), e + 1, e)
        e = np.where(np.abs(v) < 2.0 ** e, e - 1, e)
        e = np.maximum(e, -126.0)
        assert np.all(e <= 127), "value outside bf16 range"
        q = np.round(v * 2.0 ** (7 - e)) * 2.0 ** (e - 7)        # numpy rounds half to even
        out[nz] = q
    return out
