"""The 4-bit product alone (fourtune_gemm_block16) against the oracle: out =
deq(A) deq(B)^T (+ bias), elementwise within the fp32 accumulation bound, on
ragged shapes, bf16 output = nearest-even rounding of the fp32 output."""
import numpy as np
import pytest

from oracle import block16
from tests.helpers import check_fp32_dot, nan_dev, to_dev_bf16, to_host

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("M,N,K,bias", [(16, 32, 32, False), (144, 288, 96, True), (400, 544, 320, False),
                                        (1024, 768, 1536, True)])
def test_gemm_block16_matches_oracle(cuda_lib, M, N, K, bias):
    import torch
    ft = cuda_lib
    rng = np.random.default_rng(M + N + K)
    a = (rng.standard_normal((M, K)) * 2).astype(np.float32)
    b = (rng.standard_normal((N, K)) * 0.05).astype(np.float32)
    bvec = (rng.standard_normal(N) * 0.1).astype(np.float32) if bias else None
    ac, asc, _ = ft.quantize_block16(to_dev_bf16(a))
    bc, bsc, _ = ft.quantize_block16(to_dev_bf16(b))
    a_sf, b_sf = ft.mma_scales(asc, M, K), ft.mma_scales(bsc, N, K)
    bias_d = to_dev_bf16(bvec) if bias else None
    out, ws = ft.gemm_block16(ac, a_sf, bc, b_sf, M, N, K, bias=bias_d, out=nan_dev((M, N)))
    ft.device_status(ws)
    Aq = block16.dequantize(ac.cpu().numpy(), asc.cpu().numpy())
    Bq = block16.dequantize(bc.cpu().numpy(), bsc.cpu().numpy())
    bias_h = to_host(bias_d) if bias else 0.0
    ref = Aq @ Bq.T + bias_h
    absdot = np.abs(Aq) @ np.abs(Bq).T + np.abs(bias_h)
    check_fp32_dot(to_host(out), ref, absdot, K, name="deq(A) deq(B)^T")
    outb, _ = ft.gemm_block16(ac, a_sf, bc, b_sf, M, N, K, bias=bias_d, out=nan_dev((M, N), torch.bfloat16), ws=ws)
    torch.cuda.synchronize()
    assert torch.equal(outb, out.to(torch.bfloat16))
