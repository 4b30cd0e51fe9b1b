"""GPU triple-branch linear (fwd + bwd) vs the oracle.

FourTune §3.1 (three branches), §3.2 (4-bit backward on transposed blocks, no
gradient for frozen parts), §3.3 (LoRA fusion).  Bar: Q(X) and Q(G) codes and
scales bit-identical; y, dX, dA, dB, L, P within the normwise 2e-3 tolerance of
tests/helpers.py; the bf16 intermediates L and P within one bf16 ulp plus the
fp32 accumulation bound of the oracle's (both round once after accumulating);
bf16 outputs equal to the rounding of the fp32 outputs.
"""
import numpy as np
import pytest

from bit_lora_fine_b200 import synth
from oracle import block16, formats, layer as olayer
from tests.helpers import (TOL, check_bf16_dot, check_fp32_dot, nan_dev, normwise, poisoned_ws, random_layer,
                           tie_tensor, to_dev_bf16, to_host)

pytestmark = pytest.mark.gpu


def _device_layer(ft, p):
    import torch
    dev = {k: (to_dev_bf16(v) if v is not None else None) for k, v in p.items() if k in
           ("R", "S_dn", "S_up", "A", "B", "bias")}
    lay = ft.Linear.from_weights(dev["R"], dev["S_dn"], dev["S_up"], dev["A"], dev["B"], dev["bias"])
    torch.cuda.synchronize()
    return lay


def _fwd_ref_on_gpu_L(ref, Lg, U, bias, Xq, Rq):
    """Exact forward given the GPU's own bf16 L (the GPU's y used it): the oracle's y
    with its L U replaced by Lg U, and the elementwise |.| sums of the products."""
    y = ref["y"] + (Lg - ref["L"]) @ U
    absdot = np.abs(Xq) @ np.abs(Rq).T + np.abs(Lg) @ np.abs(U)
    if bias is not None:
        absdot = absdot + np.abs(bias)[None, :]
    return y, absdot


def _bwd_ref_on_gpu_P(b, Pg, D, Gq, Rq):
    """Exact dX given the GPU's own bf16 P, and its elementwise |.| sums."""
    dX = b["dX"] + (Pg - b["P"]) @ D.T
    absdot = np.abs(Gq) @ np.abs(Rq) + np.abs(Pg) @ np.abs(D).T
    return dX, absdot


def run_and_check(ft, p, M, check_bf16=True):
    """Forward and backward at full size against the oracle, every element.  Outputs
    and workspaces start poisoned (NaN / 0xFF), so an element that no kernel
    writes, or a header the call does not clear, fails the comparison."""
    import torch
    X, dY = p["X"], p["dY"]
    lay = _device_layer(ft, p)
    R_codes, R_scales = block16.quantize(p["R"])
    np.testing.assert_array_equal(lay.t["R_codes"].cpu().numpy(), R_codes)
    np.testing.assert_array_equal(lay.t["R_scales"].cpu().numpy(), R_scales)
    np.testing.assert_array_equal(lay.t["R_codes_t"].cpu().numpy(), block16.transpose_pack(R_codes))
    K, N, R_all, r_s = lay.K, lay.N, lay.R_all, lay.r_s
    bias = p.get("bias")
    D = np.concatenate([p["S_dn"], p["A"]], axis=1).astype(np.float64)
    U = np.concatenate([p["S_up"], p["B"]], axis=0).astype(np.float64)
    Rq = block16.dequantize(R_codes, R_scales)

    Xd, dYd = to_dev_bf16(X), to_dev_bf16(dY)
    ws = poisoned_ws(lay.fwd_workspace(M).numel())
    Y, L, ws = ft.linear_fwd(lay, Xd, torch.float32, ws=ws, Y=nan_dev((M, N)),
                             L=nan_dev((M, R_all), torch.bfloat16))
    ft.device_status(ws)
    co, so = lay.fwd_ws_offsets(M)
    qx_codes = ws[co:co + M * K // 2].view(M, K // 2).cpu().numpy()
    qx_scales = ws[so:so + (M // 16) * (K // 16)].view(M // 16, K // 16).cpu().numpy()

    ref = olayer.linear_fwd(X, R_codes, R_scales, p["S_dn"], p["S_up"], p["A"], p["B"], bias)
    np.testing.assert_array_equal(qx_scales, ref["qx_scales"])
    np.testing.assert_array_equal(qx_codes, ref["qx_codes"])
    Lg = to_host(L)
    check_bf16_dot(Lg, ref["L"], np.abs(X) @ np.abs(D), K)
    Yg = to_host(Y)
    assert normwise(Yg, ref["y"]) <= TOL, normwise(Yg, ref["y"])
    y_ex, absdot_y = _fwd_ref_on_gpu_L(ref, Lg, U, bias, block16.dequantize(qx_codes, qx_scales), Rq)
    check_fp32_dot(Yg, y_ex, absdot_y, K + R_all, name="y")

    if check_bf16:
        Yb, _, _ = ft.linear_fwd(lay, Xd, torch.bfloat16, ws=ws, Y=nan_dev((M, N), torch.bfloat16))
        torch.cuda.synchronize()
        np.testing.assert_array_equal(to_host(Yb), to_host(Y.to(torch.bfloat16)))

    wsb = poisoned_ws(lay.bwd_workspace(M).numel())
    dX, dA, dB, wsb = ft.linear_bwd(lay, dYd, Xd, L, torch.float32, ws=wsb, dX=nan_dev((M, K)),
                                    dA=nan_dev((K, lay.r)), dB=nan_dev((lay.r, N)))
    ft.device_status(wsb)
    gc, gs, po = lay.bwd_ws_offsets(M)
    qg_codes = wsb[gc:gc + M * N // 2].view(M, N // 2).cpu().numpy()
    qg_scales = wsb[gs:gs + (M // 16) * (N // 16)].view(M // 16, N // 16).cpu().numpy()
    Pg = to_host(wsb[po:po + M * R_all * 2].view(torch.bfloat16).view(M, R_all))

    # backward reference on the GPU's own saved L (the saved tensor is the interface)
    b = olayer.linear_bwd(dY, X, Lg, R_codes, R_scales, p["S_dn"], p["S_up"], p["A"], p["B"])
    np.testing.assert_array_equal(qg_scales, b["qg_scales"])
    np.testing.assert_array_equal(qg_codes, b["qg_codes"])
    check_bf16_dot(Pg, b["P"], np.abs(dY) @ np.abs(U).T, N)
    dXg, dAg, dBg = to_host(dX), to_host(dA), to_host(dB)
    assert normwise(dXg, b["dX"]) <= TOL, normwise(dXg, b["dX"])
    assert normwise(dAg, b["dA"]) <= TOL, normwise(dAg, b["dA"])
    assert normwise(dBg, b["dB"]) <= TOL, normwise(dBg, b["dB"])
    dx_ex, absdot_dx = _bwd_ref_on_gpu_P(b, Pg, D, block16.dequantize(qg_codes, qg_scales), Rq)
    check_fp32_dot(dXg, dx_ex, absdot_dx, N + R_all, name="dX")
    Xf = X.astype(np.float64)
    check_fp32_dot(dAg, Xf.T @ Pg[:, r_s:], np.abs(Xf).T @ np.abs(Pg[:, r_s:]), M, name="dA")
    check_fp32_dot(dBg, Lg[:, r_s:].T @ dY.astype(np.float64), np.abs(Lg[:, r_s:]).T @ np.abs(dY), M, name="dB")

    if check_bf16:
        dXb, _, _, _ = ft.linear_bwd(lay, dYd, Xd, L, torch.bfloat16, ws=wsb, dX=nan_dev((M, K), torch.bfloat16))
        torch.cuda.synchronize()
        np.testing.assert_array_equal(to_host(dXb), to_host(dX.to(torch.bfloat16)))

    # accumulate = 1 adds into dA, dB
    dX2, dA2, dB2, _ = ft.linear_bwd(lay, dYd, Xd, L, torch.float32, dA=dA.clone(), dB=dB.clone(),
                                     accumulate=True, ws=wsb)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(to_host(dA2), 2 * to_host(dA))
    np.testing.assert_array_equal(to_host(dB2), 2 * to_host(dB))
    np.testing.assert_array_equal(to_host(dX2), to_host(dX))       # deterministic
    return dict(Y=Y, dX=dX, dA=dA, dB=dB, lay=lay)


@pytest.mark.parametrize("M,K,N,r_s,r,bias", [
    (16, 32, 32, 0, 16, False),        # smallest: one 16-row block, one K group pair
    (144, 96, 288, 16, 32, False),     # ragged M tile (128+16), K block (96 of 256), N tile (256+32)
    (400, 320, 544, 32, 64, True),     # ragged everything, rank 96, bias
    (128, 256, 256, 16, 16, False),    # exactly one tile
])
def test_edge_shapes(cuda_lib, M, K, N, r_s, r, bias):
    p = random_layer(K, N, r_s, r, seed=M + K + N, bias=bias, M=M)
    run_and_check(cuda_lib, p, M)


def test_tie_inputs_through_fused_passes(cuda_lib):
    """Inputs and gradients made of exact E2M1 ties (both signs, all scales): the fused
    X and G passes must produce the oracle's codes bit for bit."""
    M, K, N = 256, 512, 256
    p = random_layer(K, N, 16, 16, seed=11)
    p["X"] = tie_tensor(M, K, seed=2)
    p["dY"] = tie_tensor(M, N, seed=3)
    run_and_check(cuda_lib, p, M, check_bf16=False)


def test_config_linear_256x512x512(cuda_lib):
    wl = synth.WORKLOADS["linear-256x512x512"]
    spec = wl.layers[0]
    p = synth.layer_params(spec)
    p["X"] = synth.layer_input(wl)
    p["dY"] = synth.upstream_grad(wl)
    run_and_check(cuda_lib, p, wl.M)


def test_special_case_zero_adapter(cuda_lib):
    """B = 0: the LoRA branch adds nothing and dA is exactly 0 (§3.2)."""
    p = random_layer(256, 256, 16, 16, seed=3, M=128)
    p["B"] = np.zeros_like(p["B"])
    out = run_and_check(cuda_lib, p, 128, check_bf16=False)
    assert np.all(to_host(out["dA"]) == 0)


def test_config_flux_linear_3072(cuda_lib):
    """FLUX-width linear at its full size (M=4608, K=N=3072, ranks 32/32)."""
    wl = synth.WORKLOADS["flux-linear-3072"]
    p = synth.layer_params(wl.layers[0])
    p["X"] = synth.layer_input(wl)
    p["dY"] = synth.upstream_grad(wl)
    run_and_check(cuda_lib, p, wl.M, check_bf16=True)


def test_repeated_calls_are_bit_identical(cuda_lib):
    """Split reductions sum in a fixed order: repeated calls give identical bits."""
    import torch
    ft = cuda_lib
    wl = synth.WORKLOADS["flux-linear-3072"]
    p = synth.layer_params(wl.layers[0])
    lay = _device_layer(ft, p)
    X, dY = to_dev_bf16(synth.layer_input(wl)), to_dev_bf16(synth.upstream_grad(wl))
    outs = []
    for _ in range(3):
        Y, L, ws = ft.linear_fwd(lay, X, torch.bfloat16)
        dX, dA, dB, wsb = ft.linear_bwd(lay, dY, X, L, torch.bfloat16)
        torch.cuda.synchronize()
        outs.append([t.clone() for t in (Y, L, dX, dA, dB)])
    for other in outs[1:]:
        for a, b in zip(outs[0], other):
            assert torch.equal(a, b)


def run_sampled(ft, p, X, dY, rows):
    """Full-size linear fwd+bwd; y, Q(X), Q(G), dX, L, P on sampled 16-row blocks
    against the oracle; dA and dB in full from the GPU's own L and P; bf16 y and
    dX equal to the rounding of the fp32 outputs everywhere."""
    import torch
    M = X.shape[0]
    lay = _device_layer(ft, p)
    K, N, r_s, R_all = lay.K, lay.N, lay.r_s, lay.R_all
    Rc, Rs = block16.quantize(p["R"])
    Rq = block16.dequantize(Rc, Rs)
    Xd, dYd = to_dev_bf16(X), to_dev_bf16(dY)
    ws = poisoned_ws(lay.fwd_workspace(M).numel())
    wsb = poisoned_ws(lay.bwd_workspace(M).numel())
    Y, L, ws = ft.linear_fwd(lay, Xd, torch.float32, ws=ws, Y=nan_dev((M, N)), L=nan_dev((M, R_all), torch.bfloat16))
    dX, dA, dB, wsb = ft.linear_bwd(lay, dYd, Xd, L, torch.float32, ws=wsb, dX=nan_dev((M, K)),
                                    dA=nan_dev((K, lay.r)), dB=nan_dev((lay.r, N)))
    ft.device_status(ws)
    ft.device_status(wsb)
    co, so = lay.fwd_ws_offsets(M)
    gc, gs, po = lay.bwd_ws_offsets(M)
    blocks = np.unique(rows // 16)
    qx = ws[co:co + M * K // 2].view(M, K // 2).cpu().numpy()[rows]
    qxs = ws[so:so + (M // 16) * (K // 16)].view(M // 16, K // 16).cpu().numpy()[blocks]
    qg = wsb[gc:gc + M * N // 2].view(M, N // 2).cpu().numpy()[rows]
    qgs = wsb[gs:gs + (M // 16) * (N // 16)].view(M // 16, N // 16).cpu().numpy()[blocks]
    Lh = to_host(L)
    P = to_host(wsb[po:po + M * R_all * 2].view(torch.bfloat16).view(M, R_all))
    Yg, dXg = to_host(Y), to_host(dX)
    assert not np.isnan(Yg).any() and not np.isnan(dXg).any()

    D = np.concatenate([p["S_dn"], p["A"]], axis=1).astype(np.float64)
    U = np.concatenate([p["S_up"], p["B"]], axis=0).astype(np.float64)
    ref = olayer.linear_fwd(X[rows], Rc, Rs, p["S_dn"], p["S_up"], p["A"], p["B"], p.get("bias"))
    np.testing.assert_array_equal(qxs, ref["qx_scales"])
    np.testing.assert_array_equal(qx, ref["qx_codes"])
    check_bf16_dot(Lh[rows], ref["L"], np.abs(X[rows]) @ np.abs(D), K)
    assert normwise(Yg[rows], ref["y"]) <= TOL
    y_ex, absdot_y = _fwd_ref_on_gpu_L(ref, Lh[rows], U, p.get("bias"), block16.dequantize(qx, qxs), Rq)
    check_fp32_dot(Yg[rows], y_ex, absdot_y, K + R_all, name="y")
    b = olayer.linear_bwd(dY[rows], X[rows], Lh[rows], Rc, Rs, p["S_dn"], p["S_up"], p["A"], p["B"])
    np.testing.assert_array_equal(qgs, b["qg_scales"])
    np.testing.assert_array_equal(qg, b["qg_codes"])
    check_bf16_dot(P[rows], b["P"], np.abs(dY[rows]) @ np.abs(U).T, N)
    assert normwise(dXg[rows], b["dX"]) <= TOL
    dx_ex, absdot_dx = _bwd_ref_on_gpu_P(b, P[rows], D, block16.dequantize(qg, qgs), Rq)
    check_fp32_dot(dXg[rows], dx_ex, absdot_dx, N + R_all, name="dX")
    Xf, dYf = X.astype(np.float64), dY.astype(np.float64)
    dA_ex, dB_ex = Xf.T @ P[:, r_s:], Lh[:, r_s:].T @ dYf
    assert normwise(to_host(dA), dA_ex) <= TOL
    assert normwise(to_host(dB), dB_ex) <= TOL
    check_fp32_dot(to_host(dA), dA_ex, np.abs(Xf).T @ np.abs(P[:, r_s:]), M, name="dA")
    check_fp32_dot(to_host(dB), dB_ex, np.abs(Lh[:, r_s:]).T @ np.abs(dYf), M, name="dB")
    # the production (bf16) outputs: the rounding of the fp32 outputs, every element
    Yb, _, _ = ft.linear_fwd(lay, Xd, torch.bfloat16, ws=ws, Y=nan_dev((M, N), torch.bfloat16))
    dXb, _, _, _ = ft.linear_bwd(lay, dYd, Xd, L, torch.bfloat16, ws=wsb, dX=nan_dev((M, K), torch.bfloat16))
    torch.cuda.synchronize()
    assert torch.equal(Yb, Y.to(torch.bfloat16))
    assert torch.equal(dXb, dX.to(torch.bfloat16))


def _sample_rows(M, nblocks=16, seed=0):
    rng = np.random.default_rng(seed)
    blocks = np.sort(rng.choice(M // 16, size=nblocks, replace=False))
    return (blocks[:, None] * 16 + np.arange(16)[None, :]).reshape(-1)


@pytest.mark.parametrize("layer", [0, 1], ids=["in-proj-3072x21504", "out-proj-15360x3072"])
def test_config_flux_single_stream_linears(cuda_lib, layer):
    """FLUX single-stream block linears at full size (M=4608, ranks 64/64, log-normal
    channel scales sigma 1.5): fused in-proj 3072 -> 21504 and out-proj 15360 -> 3072."""
    wl = synth.WORKLOADS["flux-single-stream"]
    p = synth.layer_params(wl.layers[layer], layer=layer)
    X = synth.layer_input(wl, layer=layer)
    dY = synth.upstream_grad(wl, layer=layer)
    run_sampled(cuda_lib, p, X, dY, _sample_rows(wl.M, seed=layer))


def test_timed_and_untimed_backward_agree(cuda_lib):
    """The plain backward runs dA/dB beside the dX GEMM (other M splits, the GEMM
    on fewer SMs); the timed one runs them one after the other on all SMs.  dX
    is the same product tile by tile: bit-identical.  dA and dB are the same fp32
    sums grouped differently over M: equal to fp32 rounding, and both match the
    oracle."""
    import torch
    M, K, N = 1024, 768, 768
    p = random_layer(K, N, 32, 32, seed=7, bias=False, M=M)
    lay = _device_layer(cuda_lib, p)
    Xd, dYd = to_dev_bf16(p["X"]), to_dev_bf16(p["dY"])
    Y, L, _ = cuda_lib.linear_fwd(lay, Xd, torch.float32)
    dX1, dA1, dB1, ws1 = cuda_lib.linear_bwd(lay, dYd, Xd, L, torch.float32)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(6)]
    dX2, dA2, dB2, ws2 = cuda_lib.linear_bwd(lay, dYd, Xd, L, torch.float32, events=ev)
    torch.cuda.synchronize()
    cuda_lib.device_status(ws1)
    cuda_lib.device_status(ws2)
    np.testing.assert_array_equal(to_host(dX1), to_host(dX2))
    for a, b in ((dA1, dA2), (dB1, dB2)):
        a, b = to_host(a), to_host(b)
        np.testing.assert_allclose(a, b, rtol=0, atol=1e-5 * np.abs(b).max())
    R_codes, R_scales = block16.quantize(p["R"])
    ref = olayer.linear_bwd(p["dY"], p["X"], to_host(L), R_codes, R_scales, p["S_dn"], p["S_up"], p["A"], p["B"])
    assert normwise(to_host(dA1), ref["dA"]) <= TOL
    assert normwise(to_host(dB1), ref["dB"]) <= TOL
