"""The precision variants of the layer on the GPU (FourTune §4.3, Table 4: W4A16G4,
W4A4G16, W4A16G16 beside W4A4G4) and the standard bf16 LoRA layer (§4.2) against
the oracle.

A 16-bit activation or gradient enters its product unquantized; the 4-bit weight
enters as its dequantized values, which fourtune_dequantize_block16 produces
exactly (checked bit for bit, both orientations).  y, dX, dA, dB are checked
elementwise within the fp32 accumulation bound on the GPU's own bf16
intermediates (L, P), and normwise within 2e-3; L and P within the bf16-dot
bound; the 16-bit paths' L equals the 4-bit forward's L bit for bit (the same
row pass, without the quantizer).  Outputs start poisoned (NaN).
"""
import numpy as np
import pytest

from oracle import block16, layer as olayer
from tests.helpers import (TOL, check_bf16_dot, check_fp32_dot, nan_dev, normwise, random_layer, to_dev_bf16,
                           to_host)

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("rows,cols", [(16, 16), (48, 80), (256, 512), (144, 208)])
def test_dequantize_is_exact_both_orientations(cuda_lib, rows, cols):
    ft = cuda_lib
    rng = np.random.default_rng(rows + cols)
    x = (rng.standard_normal((rows, cols)) * 0.3).astype(np.float32)
    x[:, rng.integers(cols)] *= 30
    codes, scales, _ = ft.quantize_block16(to_dev_bf16(x))
    ref = block16.dequantize(codes.cpu().numpy(), scales.cpu().numpy())
    np.testing.assert_array_equal(to_host(ft.dequantize_block16(codes, scales, rows, cols)), ref)
    np.testing.assert_array_equal(to_host(ft.dequantize_block16(codes, scales, rows, cols, transposed=True)), ref.T)


def _check_fwd16(ft, lay16, p, Wq, M, bias=None):
    import torch
    X = p["X"]
    Y, L, _ = ft.linear_fwd_a16(lay16, to_dev_bf16(X), Y=nan_dev((M, lay16.N)),
                                L=nan_dev((M, lay16.R_all), torch.bfloat16))
    ref = olayer.linear_fwd_a16(X, Wq, p["S_dn"], p["S_up"], p["A"], p["B"], bias)
    D = np.concatenate([p["S_dn"], p["A"]], 1).astype(np.float64)
    U = np.concatenate([p["S_up"], p["B"]], 0).astype(np.float64)
    Lg, Yg = to_host(L), to_host(Y)
    check_bf16_dot(Lg, ref["L"], np.abs(X) @ np.abs(D), lay16.K)
    y_ex = ref["y"] + (Lg - ref["L"]) @ U
    absdot = np.abs(X) @ np.abs(Wq).T + np.abs(Lg) @ np.abs(U) + (0 if bias is None else np.abs(bias)[None, :])
    assert normwise(Yg, ref["y"]) <= TOL
    check_fp32_dot(Yg, y_ex, absdot, lay16.K + lay16.R_all, name="y (16-bit activation)")
    return L


def _check_bwd16(ft, lay16, p, Wq, L, M):
    import torch
    X, dY = p["X"], p["dY"]
    dX, dA, dB, ws = ft.linear_bwd_g16(lay16, to_dev_bf16(dY), to_dev_bf16(X), L, dX=nan_dev((M, lay16.K)),
                                       dA=nan_dev((lay16.K, lay16.r)), dB=nan_dev((lay16.r, lay16.N)))
    ft.device_status(ws)
    Lg = to_host(L)
    b = olayer.linear_bwd_g16(dY, X, Lg, Wq, p["S_dn"], p["S_up"], p["A"], p["B"])
    D = np.concatenate([p["S_dn"], p["A"]], 1).astype(np.float64)
    # the GPU's P is not exposed here: its one-ulp rounding flips (2^-7 relative) enter dX's bound
    pd = np.abs(b["P"]) @ np.abs(D).T
    dXg = to_host(dX)
    assert normwise(dXg, b["dX"]) <= TOL
    check_fp32_dot(dXg, b["dX"], np.abs(dY) @ np.abs(Wq) + pd, lay16.N + lay16.R_all, extra=2.0 ** -7 * pd,
                   name="dX (16-bit gradient)")
    r_s = lay16.r_s
    Xf = X.astype(np.float64)
    absA = np.abs(Xf).T @ np.abs(b["P"][:, r_s:])
    assert normwise(to_host(dA), b["dA"]) <= TOL
    check_fp32_dot(to_host(dA), b["dA"], absA, M, extra=2.0 ** -7 * absA, name="dA")
    check_fp32_dot(to_host(dB), b["dB"], np.abs(Lg[:, r_s:]).T @ np.abs(dY), M, name="dB")


@pytest.mark.parametrize("M,K,N,r_s,r,bias", [
    (16, 32, 32, 0, 16, False),
    (144, 96, 288, 16, 32, False),
    (400, 320, 544, 32, 64, True),
    (1024, 768, 768, 32, 32, False),
])
def test_precision_variants_match_oracle(cuda_lib, M, K, N, r_s, r, bias):
    """W4A16 forward and G16 backward; with the 4-bit forward / backward already
    checked elsewhere these make W4A16G4, W4A4G16 and W4A16G16."""
    import torch
    ft = cuda_lib
    p = random_layer(K, N, r_s, r, seed=3 * M + K, bias=bias, M=M)
    dev = {k: to_dev_bf16(p[k]) for k in ("R", "S_dn", "S_up", "A", "B")}
    lay = ft.Linear.from_weights(dev["R"], dev["S_dn"], dev["S_up"], dev["A"], dev["B"],
                                 to_dev_bf16(p["bias"]) if bias else None)
    lay16 = ft.Linear16.from_linear(lay)
    Rc, Rs = block16.quantize(p["R"])
    Wq = block16.dequantize(Rc, Rs)
    L16 = _check_fwd16(ft, lay16, p, Wq, M, p["bias"] if bias else None)
    _, L4, _ = ft.linear_fwd(lay, to_dev_bf16(p["X"]))
    torch.cuda.synchronize()
    assert torch.equal(L16, L4)                      # the same row pass, quantizer off
    _check_bwd16(ft, lay16, p, Wq, L16, M)


def test_bf16_lora_layer_matches_oracle(cuda_lib):
    """The standard bf16 LoRA layer (bf16 weight, rank-32 adapter, no stabilizer):
    the 16-bit calls given W itself."""
    ft = cuda_lib
    M, K, N, r = 512, 768, 1024, 32
    p = random_layer(K, N, 0, r, seed=11, M=M)
    W = p["R"]
    lay16 = ft.Linear16.from_bf16_lora(to_dev_bf16(W), to_dev_bf16(p["A"]), to_dev_bf16(p["B"]))
    L = _check_fwd16(ft, lay16, p, W.astype(np.float64), M)
    _check_bwd16(ft, lay16, p, W.astype(np.float64), L, M)
