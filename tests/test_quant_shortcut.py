"""The GPU quantizer replaces the per-element IEEE division v / d by
snap19(v * (1/d)) followed by a nearest-even E2M1 conversion (see the comment on
quantize_2blocks in the CUDA sources).  This test restates that arithmetic in
NumPy float32 and checks it against the oracle's definition, fp32(v / d) then
E2M1 nearest-even, exhaustively: every finite bf16 value v and every nonzero
E4M3 scale d, over the reachable range |v / d| <= 8 (in a block |v| <= amax and
d >= amax / 6.375).  It pins the argument that v / d is either exactly an E2M1
tie or at least 1/255 (relative) away from all of them.
"""
import numpy as np

from oracle import formats


def test_division_free_quantization_is_exact():
    bits = np.arange(0, 1 << 16, dtype=np.uint32) << 16
    v = bits.view(np.float32)
    v = v[np.isfinite(v)]
    mismatches = 0
    checked = 0
    with np.errstate(over="ignore", invalid="ignore"):
        for sc in range(1, 0x7F):
            d = np.float32(formats.E4M3_TABLE[sc])
            q_def = (v / d).astype(np.float32)                   # IEEE float32 division
            keep = np.abs(q_def) <= 8
            vv, qd = v[keep], q_def[keep]
            rd = np.float32(1.0) / d                              # correctly rounded reciprocal
            q = (vv * rd).astype(np.float32)
            q = ((q.view(np.uint32) + np.uint32(8)) & np.uint32(0xFFFFFFF0)).view(np.float32)
            mismatches += int((formats.e2m1_encode(qd) != formats.e2m1_encode(q)).sum())
            checked += vv.size
    assert checked > 4_000_000
    assert mismatches == 0
