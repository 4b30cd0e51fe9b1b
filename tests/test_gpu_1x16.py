"""GPU 1x16 group-wise layer (the granularity comparator of FourTune §4.3,
Table 5) vs the oracle (oracle/group16.py, oracle/layer.py).

Bar: the quantizer's codes, scales and per-tensor maximum bit-identical to the
oracle's on the same input (the weight in both orientations; X and G inside the
fused passes); y, dX, dA, dB within the normwise 2e-3 tolerance and the
elementwise fp32 accumulation bound of tests/helpers.py, L and P within one
bf16 ulp plus that bound.
"""
import numpy as np
import pytest

from bit_lora_fine_b200 import synth
from oracle import group16, layer as olayer
from tests.helpers import (TOL, check_bf16_dot, check_fp32_dot, nan_dev, normwise, poisoned_ws, random_layer,
                           to_dev_bf16, to_host)

pytestmark = pytest.mark.gpu


def _mma_ready(scales, rows, cols):
    """The MMA-ready byte layout of per-row group scales [rows, cols/16]:
    128-row chunks x 64-column k-steps of 512 bytes; row r = 32 q + l of a chunk
    and group j of the step at byte 16 l + 4 q + j; padding 0."""
    KS = (cols + 63) // 64
    out = np.zeros(((rows + 127) // 128) * KS * 512, np.uint8)
    r = np.arange(rows)[:, None]
    g = np.arange(cols // 16)[None, :]
    off = ((r // 128) * KS + g // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + g % 4
    out[off] = scales
    return out


def _amax_bits(t):
    return int(np.float32(np.abs(t).max()).view(np.uint32))


@pytest.mark.parametrize("rows,cols", [(32, 32), (96, 160), (160, 416)])
def test_quantize_1x16_both_orientations(cuda_lib, rows, cols):
    ft = cuda_lib
    rng = np.random.default_rng(rows + cols)
    W = synth.to_bf16((rng.standard_normal((rows, cols)) * rng.uniform(0.01, 3.0, (rows, 1))).astype(np.float32))
    W[rng.integers(rows), rng.integers(cols)] = 37.5                 # a tensor maximum away from the rest
    Wd = to_dev_bf16(W)
    for transposed in (False, True):
        codes, scales, sf, amax = ft.quantize_1x16(Wd, transposed=transposed)
        T = W.T if transposed else W
        rc, rs, e = group16.quantize(T)
        np.testing.assert_array_equal(scales.cpu().numpy(), rs)
        np.testing.assert_array_equal(codes.cpu().numpy(), rc)
        assert int(amax[0].item()) & 0xFFFFFFFF == _amax_bits(W)
        np.testing.assert_array_equal(sf.cpu().numpy(), _mma_ready(rs, *T.shape))


def test_quantize_1x16_extremes(cuda_lib):
    """Tiny tensors (the per-tensor exponent at its floor of -126), a huge one, a
    zero one, and exact E2M1 ties of the scaled values."""
    ft = cuda_lib
    rng = np.random.default_rng(5)
    base = synth.to_bf16(rng.standard_normal((64, 64)).astype(np.float32))
    cases = [base * np.float32(2.0 ** -120), base * np.float32(2.0 ** -130), base * np.float32(2.0 ** 100),
             np.zeros((64, 64), np.float32)]
    ties = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0], np.float32)
    t = rng.choice(np.concatenate([ties, -ties]), size=(64, 64)).astype(np.float32)
    t[:, ::16] = 6.0                                               # each group's scale is exactly 1 * 2^e
    cases.append(t * np.float32(2.0 ** -11))
    for W in cases:
        W = synth.to_bf16(W)
        codes, scales, sf, amax = ft.quantize_1x16(to_dev_bf16(W))
        rc, rs, e = group16.quantize(W)
        np.testing.assert_array_equal(scales.cpu().numpy(), rs)
        np.testing.assert_array_equal(codes.cpu().numpy(), rc)


def _device_layer(ft, p):
    import torch
    dev = {k: (to_dev_bf16(v) if v is not None else None) for k, v in p.items() if k in
           ("R", "S_dn", "S_up", "A", "B", "bias")}
    lay = ft.Linear1x16.from_weights(dev["R"], dev["S_dn"], dev["S_up"], dev["A"], dev["B"], dev["bias"])
    torch.cuda.synchronize()
    return lay


def run_and_check(ft, p, rows=None):
    """Forward and backward against the oracle on every row (rows=None) or on the
    sampled 16-row blocks `rows` (the per-tensor exponents from the full X, G)."""
    import torch
    X, dY = p["X"], p["dY"]
    M, K = X.shape
    lay = _device_layer(ft, p)
    N, R_all, r_s = lay.N, lay.R_all, lay.r_s
    Rc, Rs, eR = group16.quantize(p["R"])
    Rtc, Rts, _ = group16.quantize(p["R"].T)
    np.testing.assert_array_equal(lay.t["R_codes"].cpu().numpy(), Rc)
    np.testing.assert_array_equal(lay.t["Rt_codes"].cpu().numpy(), Rtc)
    Rq = group16.dequantize(Rc, Rs, eR)
    Rtq = group16.dequantize(Rtc, Rts, eR)
    bias = p.get("bias")
    D = np.concatenate([p["S_dn"], p["A"]], axis=1).astype(np.float64)
    U = np.concatenate([p["S_up"], p["B"]], axis=0).astype(np.float64)
    sel = np.arange(M) if rows is None else rows

    Xd, dYd = to_dev_bf16(X), to_dev_bf16(dY)
    ws = poisoned_ws(lay.fwd_workspace(M).numel())
    Y, L, ws = ft.linear_fwd_1x16(lay, Xd, torch.float32, ws=ws, Y=nan_dev((M, N)),
                                  L=nan_dev((M, R_all), torch.bfloat16))
    ft.device_status(ws)
    co, so, ao, _ = lay.ws_offsets(M, backward=False)
    qx = ws[co:co + M * K // 2].view(M, K // 2).cpu().numpy()[sel]
    qxs = ws[so:so + M * (K // 16)].view(M, K // 16).cpu().numpy()[sel]
    assert int(ws[ao:ao + 4].view(torch.int32).item()) & 0xFFFFFFFF == _amax_bits(X)
    eX = group16.tensor_exponent(np.abs(X).max())
    ref = olayer.linear_fwd_1x16(X[sel], Rq, p["S_dn"], p["S_up"], p["A"], p["B"], bias,
                                 Qx=group16.quantize(X[sel], e=eX))
    np.testing.assert_array_equal(qxs, ref["qx_scales"])
    np.testing.assert_array_equal(qx, ref["qx_codes"])
    Lg = to_host(L)[sel]
    check_bf16_dot(Lg, ref["L"], np.abs(X[sel]) @ np.abs(D), K)
    Yg = to_host(Y)[sel]
    assert normwise(Yg, ref["y"]) <= TOL, normwise(Yg, ref["y"])
    y_ex = ref["y"] + (Lg - ref["L"]) @ U
    absdot = np.abs(group16.dequantize(qx, qxs, eX)) @ np.abs(Rq).T + np.abs(Lg) @ np.abs(U)
    if bias is not None:
        absdot = absdot + np.abs(bias)[None, :]
    check_fp32_dot(Yg, y_ex, absdot, K + R_all, name="y")

    wsb = poisoned_ws(lay.bwd_workspace(M).numel())
    dX, dA, dB, wsb = ft.linear_bwd_1x16(lay, dYd, Xd, L, torch.float32, ws=wsb, dX=nan_dev((M, K)),
                                         dA=nan_dev((K, lay.r)), dB=nan_dev((lay.r, N)))
    ft.device_status(wsb)
    gc, gs, ga, po = lay.ws_offsets(M, backward=True)
    qg = wsb[gc:gc + M * N // 2].view(M, N // 2).cpu().numpy()[sel]
    qgs = wsb[gs:gs + M * (N // 16)].view(M, N // 16).cpu().numpy()[sel]
    assert int(wsb[ga:ga + 4].view(torch.int32).item()) & 0xFFFFFFFF == _amax_bits(dY)
    Pg = to_host(wsb[po:po + M * R_all * 2].view(torch.bfloat16).view(M, R_all))
    eG = group16.tensor_exponent(np.abs(dY).max())
    Lh = to_host(L)
    b = olayer.linear_bwd_1x16(dY[sel], X[sel], Lh[sel], Rtq, p["S_dn"], p["S_up"], p["A"], p["B"],
                               Qg=group16.quantize(dY[sel], e=eG))
    np.testing.assert_array_equal(qgs, b["qg_scales"])
    np.testing.assert_array_equal(qg, b["qg_codes"])
    check_bf16_dot(Pg[sel], b["P"], np.abs(dY[sel]) @ np.abs(U).T, N)
    dXg = to_host(dX)[sel]
    assert normwise(dXg, b["dX"]) <= TOL, normwise(dXg, b["dX"])
    # exact dX given the GPU's own P, and the fp32 bound of its products
    dx_ex = b["dX"] + (Pg[sel] - b["P"]) @ D.T
    absdot_dx = np.abs(group16.dequantize(qg, qgs, eG)) @ np.abs(Rtq).T + np.abs(Pg[sel]) @ np.abs(D).T
    check_fp32_dot(dXg, dx_ex, absdot_dx, N + R_all, name="dX")
    # dA, dB in full from the GPU's own L and P (the whole-M reductions)
    Xf = X.astype(np.float64)
    dAg, dBg = to_host(dA), to_host(dB)
    check_fp32_dot(dAg, Xf.T @ Pg[:, r_s:], np.abs(Xf).T @ np.abs(Pg[:, r_s:]), M, name="dA")
    check_fp32_dot(dBg, Lh[:, r_s:].T @ dY.astype(np.float64), np.abs(Lh[:, r_s:]).T @ np.abs(dY), M, name="dB")
    assert normwise(dAg, Xf.T @ Pg[:, r_s:]) <= TOL
    return dict(Y=Y, dX=dX, lay=lay)


@pytest.mark.parametrize("M,K,N,r_s,r,bias", [
    (32, 32, 32, 0, 16, False),        # smallest
    (144, 96, 288, 16, 32, True),      # ragged M tile, K block and N tile
    (256, 320, 544, 32, 64, False),    # ragged K and N, rank 96
])
def test_linear_1x16_edge_shapes(cuda_lib, M, K, N, r_s, r, bias):
    p = random_layer(K, N, r_s, r, seed=M + K + N + 1, bias=bias, M=M)
    run_and_check(cuda_lib, p)


def test_linear_1x16_flux_3072_sampled(cuda_lib):
    """FLUX-width layer at its full size (M=4608, K=N=3072, ranks 32/32): every
    output of 256 sampled rows (16 blocks of 16) against the oracle."""
    wl = synth.WORKLOADS["flux-linear-3072"]
    p = synth.layer_params(wl.layers[0])
    p["X"] = synth.layer_input(wl)
    p["dY"] = synth.upstream_grad(wl)
    rng = np.random.default_rng(0)
    blocks = np.sort(rng.choice(wl.M // 16, size=16, replace=False))
    rows = (blocks[:, None] * 16 + np.arange(16)[None, :]).reshape(-1)
    run_and_check(cuda_lib, p, rows)
