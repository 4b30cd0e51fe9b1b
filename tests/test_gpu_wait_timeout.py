"""Failure detection without a GPU fault: every wait in the kernels is bounded, and
an expired wait is recorded in the call's status word and reported to the host.

The test makes the failure on the host side of the kernel's protocol: through the
library's test hook, the first CTA's TMA producer leaves its first stage unloaded
(nothing faults, nothing traps; the data simply never arrives), with every wait
limited to 5 ms.  The waits for that stage expire, the CTA stops, drains the
copies it started and frees its tensor memory, and fourtune_device_status
returns FT_ERR_TIMEOUT.  The same GPU then runs a normal call that must match
the oracle bit for bit.
"""
import numpy as np
import pytest

from oracle import block16
from tests.helpers import check_bf16_dot, to_dev_bf16, to_host

pytestmark = pytest.mark.gpu


def test_expired_wait_is_reported_and_the_gpu_stays_usable(cuda_lib):
    import torch
    ft = cuda_lib
    M, K, R = 148 * 128, 1024, 64          # one 128-row tile per SM, 16 stages each (more than the ring)
    rng = np.random.default_rng(3)
    Xh = rng.standard_normal((M, K)).astype(np.float32)
    Wh = (rng.standard_normal((R, K)) * 0.02).astype(np.float32)
    X, W = to_dev_bf16(Xh), to_dev_bf16(Wh)
    Xh, Wh = to_host(X), to_host(W)        # the bf16 values both sides use
    ws = torch.zeros(64 << 20, dtype=torch.uint8, device="cuda")

    ft.fault_wait_timeout(X, W, ws, wait_ns=5_000_000)
    with pytest.raises(ft.FourtuneError) as err:
        ft.device_status(ws)
    assert err.value.code == -6            # FT_ERR_TIMEOUT
    torch.cuda.synchronize()               # no CUDA error was left behind

    # the same GPU, a normal call: the rows of the CTA that stopped are correct again
    codes, scales, L = ft.quant_down_static(X, W)
    ft.quant_down_static_status()
    rows = np.arange(256)
    rc, rs = block16.quantize(Xh[rows])
    np.testing.assert_array_equal(codes.cpu().numpy()[rows], rc)
    np.testing.assert_array_equal(scales.cpu().numpy()[:16], rs)
    check_bf16_dot(to_host(L)[rows], np.asarray(Xh[rows], np.float64) @ Wh.T.astype(np.float64),
                   np.abs(Xh[rows]) @ np.abs(Wh).T, K)
