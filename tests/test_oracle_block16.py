"""Pins for oracle/block16.py, the 16x16 block quantizer (FourTune §3.2, §4.3).

Pinned by: worked ties and scales (tests/golden), an element-by-element cross
check through library converters (ml_dtypes) on random blocks, exact
representability, idempotence, the transposed-block invariant that makes
Q(G)Q(R)^T work without requantization, and the zero / subnormal / saturated
scale cases.
"""
import os

import ml_dtypes
import numpy as np
import pytest

from oracle import block16, formats

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "e2m1_e4m3_points.txt")


def _golden(section):
    with open(GOLDEN) as f:
        return [l.split()[1:] for l in f if l.startswith(section + " ")]


def _block_with_amax(amax, fill=None):
    b = np.zeros((16, 16), dtype=np.float32) if fill is None else fill.astype(np.float32).copy()
    b[3, 5] = amax
    return b


def test_block_scale_golden():
    for amax, code in _golden("block_scale"):
        _, scales = block16.quantize_codes(_block_with_amax(float(amax)))
        assert int(scales[0, 0]) == int(code, 16), (amax, scales[0, 0], code)


def test_worked_ties_at_unit_scale():
    # amax 6 -> s = 1 -> scale 0x38; the element codes are then the E2M1 ties.
    vals = np.float32([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -0.25])
    want = [0x0, 0x2, 0x2, 0x4, 0x4, 0x6, 0x6, 0x8]
    b = np.zeros((16, 16), dtype=np.float32)
    b[0, 0] = 6.0
    b[1, :8] = vals
    code4, scales = block16.quantize_codes(b)
    assert scales[0, 0] == 0x38
    assert list(code4[1, :8]) == want
    assert code4[0, 0] == 0x7


def test_scale_midpoint_and_saturating_element():
    # amax 6.375 -> s = 1.0625, the E4M3 midpoint of 1 and 1.125 -> 1.0 (even);
    # 6.375 / 1.0 then saturates to code 7 (value 6).
    b = _block_with_amax(6.375)
    code4, scales = block16.quantize_codes(b)
    assert scales[0, 0] == 0x38
    assert code4[3, 5] == 0x7


def test_zero_block_all_positive_zero_codes():
    b = np.zeros((16, 16), dtype=np.float32)
    b[2, 2] = -0.0
    code4, scales = block16.quantize_codes(b)
    assert scales[0, 0] == 0 and np.all(code4 == 0)


def test_tiny_block_scale_rounds_to_zero():
    # amax/6 below half the smallest subnormal (2^-10) -> scale 0 -> +0 codes
    b = _block_with_amax(5e-3)
    b[0, 0] = -1e-3
    code4, scales = block16.quantize_codes(b)
    assert scales[0, 0] == 0 and np.all(code4 == 0)


def test_negative_small_values_keep_sign_bit():
    b = _block_with_amax(6.0)
    b[0, 0] = -0.1
    b[0, 1] = -0.0
    code4, _ = block16.quantize_codes(b)
    assert code4[0, 0] == 0x8 and code4[0, 1] == 0x8


def _reference_quantize_via_ml_dtypes(t):
    """Element-by-element restatement through library converters (ml_dtypes RNE)."""
    rows, cols = t.shape
    code4 = np.zeros((rows, cols), np.uint8)
    scales = np.zeros((rows // 16, cols // 16), np.uint8)
    for bi in range(rows // 16):
        for bj in range(cols // 16):
            blk = t[bi * 16:(bi + 1) * 16, bj * 16:(bj + 1) * 16].astype(np.float32)
            s = np.float32(np.abs(blk).max()) / np.float32(6)
            assert s < 464
            sc = np.float32(s).astype(ml_dtypes.float8_e4m3fn)
            scales[bi, bj] = sc.view(np.uint8)
            d = np.float32(sc.astype(np.float32))
            if d == 0:
                continue
            q = (blk / d).astype(np.float32)
            q = np.clip(q, -6, 6)                     # satfinite
            code4[bi * 16:(bi + 1) * 16, bj * 16:(bj + 1) * 16] = \
                q.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF
    return code4, scales


@pytest.mark.parametrize("std,seed", [(1.0, 0), (0.02, 1), (20.0, 2), (0.0005, 3), (1e-5, 4)])
def test_quantizer_matches_library_restatement(std, seed):
    rng = np.random.default_rng(seed)
    t = (rng.standard_normal((64, 96)) * std).astype(np.float32)
    t[5, :] *= 37.0                                   # an outlier row
    ours = block16.quantize_codes(t)
    ref = _reference_quantize_via_ml_dtypes(t)
    np.testing.assert_array_equal(ours[1], ref[1])
    np.testing.assert_array_equal(ours[0], ref[0])


def test_exact_representability_every_normal_scale():
    grid = np.concatenate([formats.E2M1_MAGNITUDES, -formats.E2M1_MAGNITUDES])
    rng = np.random.default_rng(11)
    for sc in range(0x08, 0x7F):                      # every normal E4M3 scale
        d = formats.E4M3_TABLE[sc]
        blk = rng.choice(grid, size=(16, 16)) * d
        blk[0, 0] = 6.0 * d                           # amax = 6 d -> s = d exactly
        blk = blk.astype(np.float32)
        codes, scales = block16.quantize(blk)
        assert scales[0, 0] == sc
        np.testing.assert_array_equal(block16.dequantize(codes, scales), blk.astype(np.float64))


def test_idempotence_on_max_code_six_blocks():
    rng = np.random.default_rng(5)
    t = (rng.standard_normal((128, 128)) * 0.7).astype(np.float32)
    c1, s1 = block16.quantize(t)
    deq = block16.dequantize(c1, s1).astype(np.float32)
    c2, s2 = block16.quantize(deq)
    code4 = block16.unpack_codes(c1)
    for bi in range(8):
        for bj in range(8):
            blk = code4[bi * 16:(bi + 1) * 16, bj * 16:(bj + 1) * 16] & 0x7
            if blk.max() == 7:                        # max code 6 => Q(deq(Q)) == Q
                assert s2[bi, bj] == s1[bi, bj]
                np.testing.assert_array_equal(c2[bi * 16:(bi + 1) * 16, bj * 8:(bj + 1) * 8],
                                              c1[bi * 16:(bi + 1) * 16, bj * 8:(bj + 1) * 8])


def test_transposed_block_equality():
    # Q(T^T) == nibble-transpose of Q(T) with scales transposed: the same bytes
    rng = np.random.default_rng(9)
    t = (rng.standard_normal((48, 80)) * 3).astype(np.float32)
    t[:, 7] *= 50
    c, s = block16.quantize(t)
    ct, st = block16.quantize(np.ascontiguousarray(t.T))
    np.testing.assert_array_equal(st, s.T)
    np.testing.assert_array_equal(ct, block16.transpose_pack(c))
    np.testing.assert_array_equal(block16.dequantize(ct, st), block16.dequantize(c, s).T)


def test_nibble_order_even_column_low():
    b = np.zeros((16, 16), dtype=np.float32)
    b[0, 0] = 6.0                                     # code 7 at even column 0
    b[0, 1] = -6.0                                    # code 0xF at odd column 1
    codes, _ = block16.quantize(b)
    assert codes[0, 0] == 0xF7


def test_subnormal_and_saturated_scales():
    b = _block_with_amax(6 * 3 * 2.0 ** -9)           # s = 3 * 2^-9 -> subnormal code 0x03
    _, s = block16.quantize_codes(b)
    assert s[0, 0] == 0x03
    b = _block_with_amax(6 * 1000.0)                  # s = 1000 -> saturates to 448
    code4, s = block16.quantize_codes(b)
    assert s[0, 0] == 0x7E and code4[3, 5] == 0x7     # 6000/448 = 13.4 -> saturates to 6


def test_shape_checks():
    with pytest.raises(ValueError):
        block16.quantize(np.zeros((16, 20), np.float32))
