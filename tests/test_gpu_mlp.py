"""GPU MLP pair (FC1 -> GELU(tanh) -> FC2, FourTune §3.3 "MLP Fusion") vs the oracle.

Forward: h = bf16(FC1 output) within one bf16 ulp of the exact value plus the
fp32 accumulation bound; L1 and L2 within the bf16-dot bound; a = GELU(h) (the
fp32 values from the debug output) within the fp32 GELU bound of the float64
GELU of the GPU's h; Q(bf16(a)) codes and scales bit-identical to the oracle's
quantizer applied to the bf16 rounding of the GPU's own a (floating point
decides the codes, so both sides quantize the same values); y elementwise
within the fp32 accumulation bound.  Backward: d_h = bf16(d_a GELU'(h)) -- the
gradient FC1's three branches take, rounded to bf16 like any layer's incoming
gradient -- within one bf16 ulp of the exact value plus the bounds of d_a's
fp32 sum and GELU's fp32 evaluation; Q(d_h) bit-identical to the oracle's
quantizer on the GPU's d_h; P1 within the bf16-dot bound (through dX and dA1);
dX and all four adapter gradients within the normwise tolerance and the
elementwise fp32 bound; bf16(GELU(h)) is not stored (FC2's dA2 recomputes it).  bf16 y and dX equal the
rounding of the fp32 outputs.  Outputs and workspaces start poisoned.
"""
import numpy as np
import pytest

from bit_lora_fine_b200 import synth
from oracle import block16, formats, layer as olayer
from tests.helpers import (TOL, check_bf16_dot, check_bf16_rounded, check_fp32_dot, fp32_dot_bound, nan_dev,
                           normwise, poisoned_ws, to_dev_bf16, to_host)

pytestmark = pytest.mark.gpu


def _layer_dict(p):
    Rc, Rs = block16.quantize(p["R"])
    return dict(R_codes=Rc, R_scales=Rs, S_dn=p["S_dn"], S_up=p["S_up"], A=p["A"], B=p["B"], bias=p.get("bias"))


def _device_mlp(ft, p1, p2):
    dev = lambda p: {k: (to_dev_bf16(v) if v is not None else None) for k, v in p.items()}
    d1, d2 = dev(p1), dev(p2)
    l1 = ft.Linear.from_weights(d1["R"], d1["S_dn"], d1["S_up"], d1["A"], d1["B"], d1["bias"])
    l2 = ft.Linear.from_weights(d2["R"], d2["S_dn"], d2["S_up"], d2["A"], d2["B"], d2["bias"])
    return ft.MLP(l1, l2)


def _gelu_terms(h):
    """The two terms of GELU'(h) = 0.5 (1 + t) + 0.5 h (1 - t^2) c (1 + 3 k h^2): the
    GPU's fp32 evaluation (hardware exponential) errs by at most 4e-5 of their
    magnitudes, the bound used below."""
    h = np.asarray(h, dtype=np.float64)
    t = np.tanh(np.sqrt(2 / np.pi) * (h + 0.044715 * h ** 3))
    return np.abs(0.5 * (1 + t)) + np.abs(0.5 * h * (1 - t * t) * np.sqrt(2 / np.pi) * (1 + 3 * 0.044715 * h * h))


GELU_REL = 4e-5      # fp32 GELU / GELU' (hardware exponential) vs float64, relative
GELU_FLOOR = 1e-30   # absolute: beyond |u| = 40 the kernel returns the limits (0 or h, 0 or 1); the true
                     # GELU and GELU' there are below 1e-32 (h < -9.1) or within fp32 rounding of the limit


def run_mlp(ft, p1, p2, X, dY, rows=None):
    """Run fwd+bwd on the GPU (outputs and workspaces poisoned first); compare against
    the oracle on `rows` (16-row blocks), adapter gradients at full size from the
    GPU's own intermediates, bf16 outputs as the rounding of the fp32 ones."""
    import torch
    bf = torch.bfloat16
    M = X.shape[0]
    mlp = _device_mlp(ft, p1, p2)
    fc1, fc2 = _layer_dict(p1), _layer_dict(p2)
    H, K1, N2 = mlp.H, mlp.fc1.K, mlp.fc2.N
    R1, R2 = mlp.fc1.R_all, mlp.fc2.R_all
    rs1, rs2 = fc1["S_dn"].shape[1], fc2["S_dn"].shape[1]
    Xd, dYd = to_dev_bf16(X), to_dev_bf16(dY)
    wsf = poisoned_ws(mlp.fwd_workspace(M).numel())
    out = (nan_dev((M, N2)), nan_dev((M, H), bf), nan_dev((M, R1), bf), nan_dev((M, R2), bf))
    Y, h, L1, L2, wsf, a = ft.mlp_fwd(mlp, Xd, ws=wsf, dbg_a=True, out=out)
    ft.device_status(wsf)
    qc, qs = mlp.fwd_ws_offsets(M)
    qa_codes = wsf[qc:qc + M * H // 2].view(M, H // 2).cpu().numpy()
    qa_scales = wsf[qs:qs + (M // 16) * (H // 16)].view(M // 16, H // 16).cpu().numpy()
    wsb = poisoned_ws(mlp.bwd_workspace(M).numel())
    grads = (nan_dev((K1, mlp.fc1.r)), nan_dev((mlp.fc1.r, H)), nan_dev((H, mlp.fc2.r)), nan_dev((mlp.fc2.r, N2)))
    dX, dA1, dB1, dA2, dB2, wsb = ft.mlp_bwd(mlp, dYd, Xd, h, L1, L2, ws=wsb, dX=nan_dev((M, K1)), grads=grads)
    ft.device_status(wsb)
    dho, ao, qdc, qds = mlp.bwd_ws_offsets(M)
    assert ao == 2 ** 64 - 1                                        # bf16(GELU(h)) is not stored
    dh = wsb[dho:dho + M * H * 2].view(bf).view(M, H)
    qdh_codes = wsb[qdc:qdc + M * H // 2].view(M, H // 2).cpu().numpy()
    qdh_scales = wsb[qds:qds + (M // 16) * (H // 16)].view(M // 16, H // 16).cpu().numpy()

    h_g, L1_g, L2_g, a_g = to_host(h), to_host(L1), to_host(L2), to_host(a).astype(np.float32)
    dh_g = to_host(dh)
    # bf16(GELU(h)) as FC2's dA2 uses it (the GPU recomputes it from h in fp32;
    # one bf16 rounding step apart at most, covered by dA2's bound below)
    abf_g = formats.bf16_round(olayer.gelu_tanh(h_g).astype(np.float32).astype(np.float64))
    Y_g, dX_g = to_host(Y), to_host(dX)
    assert not np.isnan(Y_g).any() and not np.isnan(dX_g).any()
    rows = np.arange(M) if rows is None else rows
    blocks = np.unique(rows // 16)
    U1 = np.concatenate([fc1["S_up"], fc1["B"]], 0).astype(np.float64)
    U2 = np.concatenate([fc2["S_up"], fc2["B"]], 0).astype(np.float64)
    D1 = np.concatenate([fc1["S_dn"], fc1["A"]], 1).astype(np.float64)
    D2 = np.concatenate([fc2["S_dn"], fc2["A"]], 1).astype(np.float64)
    Rq1 = block16.dequantize(fc1["R_codes"], fc1["R_scales"])
    Rq2 = block16.dequantize(fc2["R_codes"], fc2["R_scales"])

    # ---- forward on the sampled rows
    Xs, a_s = X[rows], a_g[rows]
    o1 = olayer.linear_fwd(Xs, fc1["R_codes"], fc1["R_scales"], fc1["S_dn"], fc1["S_up"], fc1["A"], fc1["B"],
                           fc1["bias"])
    D1 = np.concatenate([fc1["S_dn"], fc1["A"]], 1)
    check_bf16_dot(L1_g[rows], o1["L"], np.abs(Xs) @ np.abs(D1), K1)
    # h = bf16(FC1 output): one bf16 ulp of the exact value (given the GPU's own L1)
    # plus the fp32 accumulation bound
    h_ex = o1["y"] + (L1_g[rows] - o1["L"]) @ U1
    absdot_h = (np.abs(block16.dequantize(o1["qx_codes"], o1["qx_scales"])) @ np.abs(Rq1).T
                + np.abs(L1_g[rows]) @ np.abs(U1) + np.abs(fc1["bias"])[None, :])
    check_bf16_rounded(h_g[rows], h_ex, fp32_dot_bound(absdot_h, K1 + R1) + 2.0 ** -24 * np.abs(h_ex), name="h")
    g_ref = olayer.gelu_tanh(h_g[rows])
    assert np.all(np.abs(a_s - g_ref) <= GELU_REL * np.abs(g_ref) + GELU_FLOOR), "GELU(h) beyond its fp32 bound"
    a_bf = formats.bf16_round(a_s.astype(np.float64))                   # FC2's input, all three branches
    rc, rs_ = block16.quantize(a_bf.astype(np.float32))                  # oracle quantizer on the GPU's bf16(a)
    np.testing.assert_array_equal(qa_scales[blocks], rs_)
    np.testing.assert_array_equal(qa_codes[rows], rc)
    o2 = olayer.linear_fwd(a_bf, fc2["R_codes"], fc2["R_scales"], fc2["S_dn"], fc2["S_up"], fc2["A"], fc2["B"],
                           fc2["bias"], Qx=(rc, rs_))
    check_bf16_dot(L2_g[rows], o2["L"], np.abs(a_bf) @ np.abs(D2), H)
    assert normwise(Y_g[rows], o2["y"]) <= TOL
    y_ex = o2["y"] + (L2_g[rows] - o2["L"]) @ U2
    absdot_y = (np.abs(block16.dequantize(rc, rs_)) @ np.abs(Rq2).T + np.abs(L2_g[rows]) @ np.abs(U2)
                + np.abs(fc2["bias"])[None, :])
    check_fp32_dot(Y_g[rows], y_ex, absdot_y, H + R2, name="y")

    # ---- backward on the sampled rows (oracle fed the GPU's h, L, d_h)
    b = olayer.mlp_bwd(dY[rows], Xs, h_g[rows], L1_g[rows], L2_g[rows], fc1, fc2, dh_bf=dh_g[rows])
    # d_h = bf16(d_a GELU'(h)): d_a is an fp32 sum on the GPU's own P2 (one bf16 ulp,
    # at most 2^-7 relative, from the oracle's), GELU' an fp32 evaluation
    Gq = block16.dequantize(b["qg_codes"], b["qg_scales"])
    pd2 = np.abs(b["P2"]) @ np.abs(D2).T
    err_da = fp32_dot_bound(np.abs(Gq) @ np.abs(Rq2) + pd2, N2 + R2) + 2.0 ** -7 * pd2
    gp = olayer.gelu_tanh_grad(h_g[rows])
    err_dh = (np.abs(gp) * err_da + np.abs(b["d_a"]) * (GELU_REL * _gelu_terms(h_g[rows]) + GELU_FLOOR)
              + 2.0 ** -24 * np.abs(b["d_h"]))
    check_bf16_rounded(dh_g[rows], b["d_h"], err_dh, name="d_h")
    np.testing.assert_array_equal(qdh_scales[blocks], b["qdh_scales"])
    np.testing.assert_array_equal(qdh_codes[rows], b["qdh_codes"])
    assert normwise(dX_g[rows], b["dX"]) <= TOL
    pd1 = np.abs(b["P1"]) @ np.abs(D1).T
    check_fp32_dot(dX_g[rows], b["dX"], np.abs(block16.dequantize(b["qdh_codes"], b["qdh_scales"])) @ np.abs(Rq1) + pd1,
                   H + R1, extra=2.0 ** -7 * pd1, name="dX")

    # ---- adapter gradients at full size, from the GPU's intermediates
    P2 = formats.bf16_round(dY.astype(np.float64) @ U2.T)
    P1 = formats.bf16_round(dh_g @ U1.T)
    Xf, dYf = X.astype(np.float64), dY.astype(np.float64)
    for got, ex, absd, extra, name in (
            (dA2, abf_g.T @ P2[:, rs2:], np.abs(abf_g).T @ np.abs(P2[:, rs2:]), True, "dA2"),
            (dB2, L2_g[:, rs2:].T @ dYf, np.abs(L2_g[:, rs2:]).T @ np.abs(dYf), False, "dB2"),
            (dA1, Xf.T @ P1[:, rs1:], np.abs(Xf).T @ np.abs(P1[:, rs1:]), True, "dA1"),
            (dB1, L1_g[:, rs1:].T @ dh_g, np.abs(L1_g[:, rs1:]).T @ np.abs(dh_g), False, "dB1")):
        g = to_host(got)
        assert normwise(g, ex) <= TOL, name
        # P (and, for dA2, bf16(GELU(h))) recomputed here may differ from the GPU's by
        # one bf16 ulp each (2^-7 relative)
        check_fp32_dot(g, ex, absd, M, extra=2.0 ** -6 * absd if extra else 0.0, name=name)

    # ---- production outputs: bf16 y and dX are the rounding of the fp32 ones
    outb = (nan_dev((M, N2), bf),) + out[1:]
    Yb = ft.mlp_fwd(mlp, Xd, ws=wsf, out=outb)[0]
    dXb = ft.mlp_bwd(mlp, dYd, Xd, h, L1, L2, ws=wsb, dX=nan_dev((M, K1), bf))[0]
    torch.cuda.synchronize()
    assert torch.equal(Yb, Y.to(bf))
    assert torch.equal(dXb, dX.to(bf))
    return dict(Y=Y, dX=dX)


def _small(seed, K1, H, N2, r_s, r, M):
    rng = np.random.default_rng(seed)
    f = lambda shape, s: synth.to_bf16((rng.standard_normal(shape) * s).astype(np.float32))
    mk = lambda K, N: dict(R=f((N, K), 0.05), S_dn=f((K, r_s), 0.05), S_up=f((r_s, N), 0.05), A=f((K, r), 0.05),
                           B=f((r, N), 0.01), bias=f((N,), 0.05))
    X = (rng.standard_normal((M, K1)) * 1.0).astype(np.float32)
    X[:, rng.integers(K1)] *= 20
    return mk(K1, H), mk(H, N2), synth.to_bf16(X), f((M, N2), 1.0)


@pytest.mark.parametrize("K1,H,N2,r_s,r,M", [(96, 288, 160, 16, 32, 144), (256, 512, 256, 32, 32, 256)])
def test_small_mlp_full_oracle(cuda_lib, K1, H, N2, r_s, r, M):
    p1, p2, X, dY = _small(K1 + H, K1, H, N2, r_s, r, M)
    run_mlp(cuda_lib, p1, p2, X, dY)


def test_flux_mlp_3072_sampled_rows(cuda_lib):
    """FLUX-width MLP at full size (M=4608, 3072 -> 12288 -> 3072, ranks 32/32, biases):
    row-local outputs on 16 sampled 16-row blocks (256 rows), adapter gradients in full."""
    wl = synth.WORKLOADS["flux-mlp-3072"]
    p1 = synth.layer_params(wl.layers[0], layer=0)
    p2 = synth.layer_params(wl.layers[1], layer=1)
    X = synth.layer_input(wl)
    dY = synth.upstream_grad(wl, layer=1)
    rng = np.random.default_rng(0)
    blocks = np.sort(rng.choice(wl.M // 16, size=16, replace=False))
    rows = (blocks[:, None] * 16 + np.arange(16)[None, :]).reshape(-1)
    run_mlp(cuda_lib, p1, p2, X, dY, rows=rows)


def test_video_mlp_5120_sampled_rows(cuda_lib):
    """Video-DiT-width MLP at full size (M=32768, 5120 -> 13824 -> 5120, ranks 64/64,
    2% outlier channels x30, weights N(0, 0.015)): 256 sampled rows, gradients in full."""
    wl = synth.WORKLOADS["video-mlp-5120"]
    p1 = synth.layer_params(wl.layers[0], layer=0)
    p2 = synth.layer_params(wl.layers[1], layer=1)
    X = synth.layer_input(wl)
    dY = synth.upstream_grad(wl, layer=1)
    rng = np.random.default_rng(1)
    blocks = np.sort(rng.choice(wl.M // 16, size=16, replace=False))
    rows = (blocks[:, None] * 16 + np.arange(16)[None, :]).reshape(-1)
    run_mlp(cuda_lib, p1, p2, X, dY, rows=rows)
