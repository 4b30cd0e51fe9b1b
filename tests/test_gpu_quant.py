"""GPU block16 quantizer vs the oracle: codes and scales must be bit-identical
(FourTune §3.2, §4.3 16x16 blocks; E2M1 codes, E4M3 scales, nearest-even)."""
import numpy as np
import pytest

from bit_lora_fine_b200 import synth
from oracle import block16, formats
from tests.helpers import tie_tensor, to_dev_bf16

pytestmark = pytest.mark.gpu


def _gpu_quant(cuda_lib, x, transposed=True):
    codes, scales, codes_t = cuda_lib.quantize_block16(to_dev_bf16(x), transposed=transposed)
    return codes.cpu().numpy(), scales.cpu().numpy(), None if codes_t is None else codes_t.cpu().numpy()


def _check(cuda_lib, x):
    c, s, ct = _gpu_quant(cuda_lib, x)
    rc, rs = block16.quantize(x)
    np.testing.assert_array_equal(s, rs)
    np.testing.assert_array_equal(c, rc)
    np.testing.assert_array_equal(ct, block16.transpose_pack(rc))


def test_worked_ties_probe(cuda_lib):
    # block amax 6 -> scale 1.0: the element codes are the E2M1 rounding ties,
    # including the sign of small negatives and saturation; second block row: scale midpoints
    b = np.zeros((32, 32), np.float32)
    b[0, 0] = 6.0
    b[1, :16] = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -0.25, -0.1, -0.0, 0.2500001, 2.9, -5.5, 4.5, 1.0, -6.0]
    b[16, 0] = 6.375                        # s = 1.0625 -> scale 1.0, element saturates
    b[16, 16] = 6 * 3 * 2.0 ** -9           # subnormal scale 0x03
    b[0, 16] = 6 * 1000.0                   # scale saturates at 448
    b[16:32, 16] = np.float32(1e-3)         # tiny block: after rounding to bf16 still small
    b = synth.to_bf16(b)
    _check(cuda_lib, b)


def test_every_e2m1_tie(cuda_lib):
    """All seven E2M1 ties, both signs, one bf16 ulp either side, under normal and
    subnormal scales: the codes must be the oracle's nearest-even table search."""
    x = tie_tensor(176, 224, seed=1)
    _check(cuda_lib, x)


@pytest.mark.parametrize("shape,std,seed", [((16, 16), 1.0, 0), ((32, 48), 0.02, 1), ((48, 80), 5.0, 2),
                                            ((64, 96), 1e-4, 3), ((256, 512), 1.0, 4), ((144, 208), 0.3, 5)])
def test_random_shapes(cuda_lib, shape, std, seed):
    rng = np.random.default_rng(seed)
    x = (rng.standard_normal(shape) * std).astype(np.float32)
    x[:, rng.integers(shape[1])] *= 40
    _check(cuda_lib, synth.to_bf16(x))            # both sides see the same bf16 values


def test_zero_and_negative_zero_blocks(cuda_lib):
    x = np.zeros((32, 32), np.float32)
    x[0:16, 16:32] = -0.0
    x[16, 16] = 3.0
    _check(cuda_lib, synth.to_bf16(x))


def test_flux_weight_full(cuda_lib):
    """The FLUX-width residual weight R [3072, 3072] ~ N(0, 0.02), bit-exact in full."""
    spec = synth.WORKLOADS["flux-linear-3072"].layers[0]
    R = synth.layer_params(spec)["R"]
    _check(cuda_lib, R)


def test_row_stride(cuda_lib):
    """A strided view (row stride 96 elements, 64 columns) through the C ABI."""
    import ctypes
    import torch
    rng = np.random.default_rng(7)
    big = synth.to_bf16(rng.standard_normal((48, 96)).astype(np.float32))
    xd = to_dev_bf16(big)[:, 16:80]
    c = torch.empty((48, 32), dtype=torch.uint8, device="cuda")
    s = torch.empty((3, 4), dtype=torch.uint8, device="cuda")
    rc = cuda_lib.load().fourtune_quantize_block16(
        ctypes.c_void_p(xd.data_ptr()), 48, 64, 96, ctypes.c_void_p(c.data_ptr()), ctypes.c_void_p(s.data_ptr()),
        None, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0
    rc_, rs_ = block16.quantize(np.ascontiguousarray(big[:, 16:80]))
    np.testing.assert_array_equal(s.cpu().numpy(), rs_)
    np.testing.assert_array_equal(c.cpu().numpy(), rc_)


def _mma_layout(scales, rows, cols, transposed):
    """The MMA-ready scale order written out from its definition (the 512-byte
    block of 128-row chunk c and 64-column step t holds the scale of row
    128 c + 32 q + l and group 4 t + j at byte 16 l + 4 q + j; zero elsewhere)."""
    ks = (cols + 63) // 64
    out = np.zeros(((rows + 127) // 128) * ks * 512, np.uint8)
    r = np.arange(rows)[:, None]
    g = np.arange(cols // 16)[None, :]
    off = ((r // 128) * ks + g // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + g % 4
    src = scales.T if transposed else scales
    out[off.ravel()] = src[np.arange(rows) // 16][:, np.arange(cols // 16)].ravel()
    return out


@pytest.mark.parametrize("rows,cols", [(16, 32), (144, 96), (400, 320), (3072, 3072)])
def test_mma_scale_layout(cuda_lib, rows, cols):
    """fourtune_mma_scales on the oracle's scales of R [rows, cols] (forward operand)
    and of R^T (backward operand, transposed read of the same bytes)."""
    import torch
    rng = np.random.default_rng(rows + cols)
    R = synth.to_bf16((rng.standard_normal((rows, cols)) * 0.02).astype(np.float32))
    _, rs = block16.quantize(R)
    sd = torch.from_numpy(rs).to("cuda")
    got = cuda_lib.mma_scales(sd, rows, cols).cpu().numpy()
    np.testing.assert_array_equal(got, _mma_layout(rs, rows, cols, False))
    got_t = cuda_lib.mma_scales(sd, cols, rows, transposed=True).cpu().numpy()
    np.testing.assert_array_equal(got_t, _mma_layout(rs, cols, rows, True))


def _near_tie_f32(rows, cols, seed):
    """float32 blocks for the fp32-input quantizer: each 16x16 block gets a chosen
    E4M3 scale d (one element is +-6 d, so amax / 6 = d exactly) and elements on,
    and a few float32 ulps either side of, every E2M1 rounding threshold times d,
    both signs -- the cases where the float32 rounding of the quotient decides the
    code -- plus random values.  Scales run over subnormal, normal and near-448 codes."""
    rng = np.random.default_rng(seed)
    ties = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
    codes = np.concatenate([np.arange(1, 8), rng.integers(8, 0x7F, size=64)])
    x = np.zeros((rows, cols), np.float64)
    for rb in range(rows // 16):
        for cb in range(cols // 16):
            d = float(formats.e4m3_decode(np.array([codes[(rb * 7 + cb) % len(codes)]], np.uint8))[0])
            t = rng.choice(ties, size=(16, 16)) * rng.choice([-1.0, 1.0], size=(16, 16))
            k = rng.integers(-6, 7, size=(16, 16))
            blk = (t * d * (1.0 + k * 2.0 ** -24)).astype(np.float32).astype(np.float64)
            rnd = rng.random((16, 16)) < 0.25
            blk[rnd] = (rng.uniform(-6, 6, size=int(rnd.sum())) * d).astype(np.float32)
            blk[0, 0] = 6.0 * d * rng.choice([-1.0, 1.0])
            x[rb * 16:(rb + 1) * 16, cb * 16:(cb + 1) * 16] = blk
    return x.astype(np.float32)


@pytest.mark.parametrize("rows,cols,seed", [(64, 256, 0), (160, 96, 1), (512, 1024, 2)])
def test_fp32_quantizer_near_ties(cuda_lib, rows, cols, seed):
    """fourtune_quantize_block16_f32 (the division-free IEEE-quotient quantizer used
    for the MLP's fp32 GELU output) bit for bit against the oracle at the E2M1
    rounding thresholds."""
    import torch
    x = _near_tie_f32(rows, cols, seed)
    c, s = cuda_lib.quantize_block16_f32(torch.from_numpy(x).to("cuda"))
    rc, rs = block16.quantize(x)
    np.testing.assert_array_equal(s.cpu().numpy(), rs)
    np.testing.assert_array_equal(c.cpu().numpy(), rc)


def test_every_bf16_block_maximum(cuda_lib):
    """One 16x16 block per positive finite bf16 value as its maximum (32640 blocks,
    normal and subnormal, up to the largest finite): the block scales (E4M3 of
    fp32(amax / 6)) and codes match the oracle's IEEE division bit for bit."""
    rng = np.random.default_rng(11)
    bits = np.arange(1, 0x7F80, dtype=np.uint32)
    amax = (bits << 16).view(np.float32)                                  # 32639 values
    amax = np.concatenate([amax, np.float32([0.0])])                      # + an all-zero block
    nb = len(amax)                                                        # 32640 = 255 x 128
    frac = rng.uniform(-1.0, 1.0, size=(nb, 16, 16)).astype(np.float32)
    blocks = synth.to_bf16(frac * amax[:, None, None])
    blocks = np.minimum(np.abs(blocks), amax[:, None, None]) * np.sign(blocks)
    blocks[:, 0, 0] = amax                                                # the exact maximum
    x = blocks.reshape(255, 128, 16, 16).transpose(0, 2, 1, 3).reshape(255 * 16, 128 * 16)
    _check(cuda_lib, synth.to_bf16(x))
