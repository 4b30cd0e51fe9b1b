"""The stabilizer split on the GPU (FourTune §3.1) against the oracle.

fourtune_stabilizer_residual is fed the oracle's bf16 factors and must give the
oracle's residual R = bf16(W - (S_dn S_up)^T) within one bf16 ulp plus the fp32
bound of the rank-r_s sum; R's block16 codes are bit-identical to the oracle's
quantizer applied to the GPU's R.  The whole split (library SVD in float32,
this library's residual and quantizer) reproduces the oracle's low-rank part and
residual to the precision of a float32 SVD."""
import numpy as np
import pytest

from oracle import block16, formats, stabilizer
from tests.helpers import check_bf16_rounded, normwise, to_dev_bf16, to_host

pytestmark = pytest.mark.gpu


def _weight(N, K, seed):
    rng = np.random.default_rng(seed)
    W = rng.standard_normal((N, K)) * 0.02
    for _ in range(3):        # a few large directions: what the stabilizer is for
        W += 2.0 * np.outer(rng.standard_normal(N), rng.standard_normal(K)) / np.sqrt(K)
    return formats.bf16_round(W).astype(np.float32)


@pytest.mark.parametrize("N,K,r_s", [(256, 512, 16), (512, 384, 32), (3072, 3072, 32)])
def test_residual_kernel_matches_oracle(cuda_lib, N, K, r_s):
    ft = cuda_lib
    W = _weight(N, K, N + K)
    o = stabilizer.split(W, r_s)
    R = ft.stabilizer_residual(to_dev_bf16(W), to_dev_bf16(o["S_dn"]), to_dev_bf16(o["S_up"]))
    Rg = to_host(R)
    absdot = (np.abs(o["S_dn"]) @ np.abs(o["S_up"])).T
    check_bf16_rounded(Rg, W.astype(np.float64) - (o["S_dn"] @ o["S_up"]).T,
                       r_s * 2.0 ** -23 * absdot + 2.0 ** -24 * np.abs(W), name="R")
    codes, scales, _ = ft.quantize_block16(R)
    rc, rs = block16.quantize(Rg.astype(np.float32))
    np.testing.assert_array_equal(codes.cpu().numpy(), rc)
    np.testing.assert_array_equal(scales.cpu().numpy(), rs)


def test_full_split_matches_oracle(cuda_lib):
    from bit_lora_fine_b200 import prepare
    N, K, r_s = 768, 512, 32
    W = _weight(N, K, 7)
    S_dn, S_up, R = prepare.stabilizer_split(to_dev_bf16(W), r_s)
    o = stabilizer.split(W, r_s)
    S_g = to_host(S_dn) @ to_host(S_up)
    assert normwise(S_g, o["S_dn"] @ o["S_up"]) <= 5e-3          # float32 SVD, bf16 factors
    assert normwise(to_host(R), o["R"]) <= 5e-2                    # the residual is the small part
    # the split moved the large directions out of the quantized weight
    assert np.abs(to_host(R)).max() < 0.5 * np.abs(W).max()
