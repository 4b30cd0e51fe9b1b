"""GPU MLP pair (FC1 -> GELU(tanh) -> FC2, FourTune §3.3 "MLP Fusion") vs the oracle.

Forward: h (bf16) and L1 against the oracle; a = GELU(h) (the fp32 values the
GPU quantized, from the debug output) against the float64 GELU of the GPU's h;
Q(a) codes and scales bit-identical to the oracle's quantizer applied to the
GPU's own fp32 a (floating point decides the codes, so both sides quantize the
same a); L2 and y against the oracle on those operands.  Backward: d_h and
bf16(GELU(h)) against the oracle, Q(d_h) bit-identical to the oracle's
quantizer on the GPU's d_h, dX and all four adapter gradients within the
normwise tolerance.
"""
import numpy as np
import pytest

from bit_lora_fine_b200 import synth
from oracle import block16, formats, layer as olayer
from tests.helpers import TOL, check_bf16_dot, normwise, to_dev_bf16, to_host

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


def run_mlp(ft, p1, p2, X, dY, rows=None):
    """Run fwd+bwd on the GPU; compare against the oracle on `rows` (16-row blocks),
    and check the adapter gradients at full size from the GPU's own intermediates."""
    import torch
    M = X.shape[0]
    mlp = _device_mlp(ft, p1, p2)
    fc1, fc2 = _layer_dict(p1), _layer_dict(p2)
    H = mlp.H
    Xd, dYd = to_dev_bf16(X), to_dev_bf16(dY)
    Y, h, L1, L2, wsf, a = ft.mlp_fwd(mlp, Xd, torch.float32, dbg_a=True)
    ft.device_status(wsf)
    qc, qs = mlp.fwd_ws_offsets(M)
    qa_codes = wsf[qc:qc + M * H // 2].view(M, H // 2).cpu().numpy()
    qa_scales = wsf[qs:qs + (M // 16) * (H // 16)].view(M // 16, H // 16).cpu().numpy()
    dX, dA1, dB1, dA2, dB2, wsb = ft.mlp_bwd(mlp, dYd, Xd, h, L1, L2, torch.float32)
    ft.device_status(wsb)
    dho, ao, qdc, qds = mlp.bwd_ws_offsets(M)
    dh = wsb[dho:dho + M * H * 2].view(torch.bfloat16).view(M, H)
    abf = wsb[ao:ao + M * H * 2].view(torch.bfloat16).view(M, H)
    qdh_codes = wsb[qdc:qdc + M * H // 2].view(M, H // 2).cpu().numpy()
    qdh_scales = wsb[qds:qds + (M // 16) * (H // 16)].view(M // 16, H // 16).cpu().numpy()

    h_g, L1_g, L2_g, a_g = to_host(h), to_host(L1), to_host(L2), to_host(a).astype(np.float32)
    dh_g, abf_g = to_host(dh), to_host(abf)
    rows = np.arange(M) if rows is None else rows
    blocks = np.unique(rows // 16)

    # ---- forward on the sampled rows
    Xs, a_s = X[rows], a_g[rows]
    o1 = olayer.linear_fwd(Xs, fc1["R_codes"], fc1["R_scales"], fc1["S_dn"], fc1["S_up"], fc1["A"], fc1["B"],
                           fc1["bias"])
    assert normwise(h_g[rows], o1["y"]) <= 2.0 ** -8 + TOL               # h = bf16(FC1 output)
    D1 = np.concatenate([fc1["S_dn"], fc1["A"]], 1)
    check_bf16_dot(L1_g[rows], o1["L"], np.abs(Xs) @ np.abs(D1), X.shape[1])
    assert normwise(a_s, olayer.gelu_tanh(h_g[rows])) <= 1e-5            # fp32 tanhf vs float64
    rc, rs_ = block16.quantize(a_s)                                      # oracle quantizer on the GPU's a
    np.testing.assert_array_equal(qa_scales[blocks], rs_)
    np.testing.assert_array_equal(qa_codes[rows], rc)
    a_bf = formats.bf16_round(a_s.astype(np.float64))
    D2 = np.concatenate([fc2["S_dn"], fc2["A"]], 1)
    o2 = olayer.linear_fwd(a_bf, fc2["R_codes"], fc2["R_scales"], fc2["S_dn"], fc2["S_up"], fc2["A"], fc2["B"],
                           fc2["bias"], Qx=(rc, rs_))
    check_bf16_dot(L2_g[rows], o2["L"], np.abs(a_bf) @ np.abs(D2), H)
    assert normwise(to_host(Y)[rows], o2["y"]) <= TOL

    # ---- backward on the sampled rows (oracle fed the GPU's h, L, d_h, bf16(GELU(h)))
    # bf16(GELU(h)) from fp32 tanh: tiny outputs for very negative h carry the
    # cancellation in (1 + tanh) -- small in absolute terms, so normwise
    assert normwise(abf_g[rows], olayer.gelu_tanh(h_g[rows])) <= 2.0 ** -8
    b = olayer.mlp_bwd(dY[rows], Xs, h_g[rows], L1_g[rows], L2_g[rows], fc1, fc2, dh_bf=dh_g[rows],
                       a_bf=abf_g[rows])
    assert normwise(dh_g[rows], b["d_h"]) <= 2.0 ** -8 + TOL             # d_h = bf16(d_a GELU'(h))
    np.testing.assert_array_equal(qdh_scales[blocks], b["qdh_scales"])
    np.testing.assert_array_equal(qdh_codes[rows], b["qdh_codes"])
    assert normwise(to_host(dX)[rows], b["dX"]) <= TOL

    # ---- adapter gradients at full size, from the GPU's intermediates
    U2 = np.concatenate([fc2["S_up"], fc2["B"]], 0)
    U1 = np.concatenate([fc1["S_up"], fc1["B"]], 0)
    P2 = formats.bf16_round(dY.astype(np.float64) @ U2.T)
    P1 = formats.bf16_round(dh_g @ U1.T)
    rs1, rs2 = fc1["S_dn"].shape[1], fc2["S_dn"].shape[1]
    assert normwise(to_host(dA2), abf_g.T @ P2[:, rs2:]) <= TOL
    assert normwise(to_host(dB2), L2_g[:, rs2:].T @ dY.astype(np.float64)) <= TOL
    assert normwise(to_host(dA1), X.astype(np.float64).T @ P1[:, rs1:]) <= TOL
    assert normwise(to_host(dB1), L1_g[:, rs1:].T @ dh_g) <= TOL
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
    row-local outputs on 8 sampled 16-row blocks, adapter gradients in full."""
    wl = synth.WORKLOADS["flux-mlp-3072"]
    p1 = synth.layer_params(wl.layers[0], layer=0)
    p2 = synth.layer_params(wl.layers[1], layer=1)
    X = synth.layer_input(wl)
    dY = synth.upstream_grad(wl, layer=1)
    rng = np.random.default_rng(0)
    blocks = np.sort(rng.choice(wl.M // 16, size=8, replace=False))
    rows = (blocks[:, None] * 16 + np.arange(16)[None, :]).reshape(-1)
    run_mlp(cuda_lib, p1, p2, X, dY, rows=rows)


def test_video_mlp_5120_sampled_rows(cuda_lib):
    """Video-DiT-width MLP at full size (M=32768, 5120 -> 13824 -> 5120, ranks 64/64,
    2% outlier channels x30, weights N(0, 0.015)): sampled rows, gradients in full."""
    wl = synth.WORKLOADS["video-mlp-5120"]
    p1 = synth.layer_params(wl.layers[0], layer=0)
    p2 = synth.layer_params(wl.layers[1], layer=1)
    X = synth.layer_input(wl)
    dY = synth.upstream_grad(wl, layer=1)
    rng = np.random.default_rng(1)
    blocks = np.sort(rng.choice(wl.M // 16, size=6, replace=False))
    rows = (blocks[:, None] * 16 + np.arange(16)[None, :]).reshape(-1)
    run_mlp(cuda_lib, p1, p2, X, dY, rows=rows)
