"""Pins of the 1x16 group-wise quantizer (oracle/group16.py) and of the 1x16
layer functions (oracle/layer.py).

Checked against: hand-worked values (tests/golden/group16_worked.txt), the
reduction to the pinned 16x16 block quantizer when every 16-row block repeats
one row, the power-of-two equivariance of the per-tensor scale, the format's
invariants, and triple-loop / adjoint forms of the layer on lossless operands.
"""
import os

import numpy as np
import pytest

from oracle import block16, formats, group16, layer

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "group16_worked.txt")


def _lines(tag):
    out = []
    with open(GOLDEN) as f:
        for line in f:
            parts = line.split()
            if parts and parts[0] == tag:
                out.append(parts[1:])
    return out


def test_tensor_exponent_golden():
    rows = _lines("exponent")
    assert len(rows) == 9
    for amax, e in rows:
        assert group16.tensor_exponent(float(amax)) == int(e), amax


def test_worked_tensor_golden():
    t = np.zeros((3, 16), np.float32)
    t[0] = 0.5 * np.arange(16)
    t[1] = -1.0
    codes, scales, e = group16.quantize(t)
    assert e == int(_lines("tensor_e")[0][0])
    for r, sc, *cb in _lines("row"):
        r = int(r)
        assert scales[r, 0] == int(sc, 16), r
        np.testing.assert_array_equal(codes[r], [int(x, 16) for x in cb])


def test_reduces_to_block16_when_rows_repeat():
    # every 16-row block repeats one row: 1x16 groups with e = 0 are the 16x16
    # blocks, row by row
    rng = np.random.default_rng(7)
    base = (rng.standard_normal((4, 96)) * 10.0 ** rng.integers(-3, 3, (4, 1))).astype(np.float32)
    t = np.repeat(base, 16, axis=0)
    c16, s16 = block16.quantize(t)
    cg, sg, e = group16.quantize(t, e=0)
    assert e == 0
    np.testing.assert_array_equal(cg, c16)
    np.testing.assert_array_equal(sg, np.repeat(s16, 16, axis=0))


def test_power_of_two_equivariance():
    # scaling the tensor by 2^k moves only the per-tensor exponent
    rng = np.random.default_rng(8)
    t = (rng.standard_normal((32, 64)) * 3.0).astype(np.float32)
    c0, s0, e0 = group16.quantize(t)
    for k in (-20, -3, 5, 30):
        ck, sk, ek = group16.quantize((t * np.float32(2.0 ** k)).astype(np.float32))
        assert ek == e0 + k
        np.testing.assert_array_equal(ck, c0)
        np.testing.assert_array_equal(sk, s0)


def test_format_invariants():
    rng = np.random.default_rng(9)
    t = (rng.standard_normal((64, 128)) * rng.uniform(0.5, 2.0, (64, 1))).astype(np.float32)
    codes, scales, e = group16.quantize(t)
    # the tensor maximum maps at or below the E4M3 maximum, within a factor 2 of it
    amax = np.abs(t).max()
    assert amax / (6 * 2.0 ** e) <= 448 < 2 * amax / (6 * 2.0 ** e)
    assert np.all(scales <= 0x7E)
    # each group's largest element takes a top code (4 or 6): its scale is within
    # 1/16 (relative) of amax / 6
    c4 = block16.unpack_codes(codes) & 0x7
    top = c4.reshape(64, 8, 16).max(axis=2)
    assert np.all((top == 7) | (top == 6))
    # dequantized error within half the largest E2M1 gap (1.0) times the group scale
    deq = group16.dequantize(codes, scales, e)
    step = np.repeat(formats.e4m3_decode(scales), 16, axis=1) * 2.0 ** e
    assert np.all(np.abs(deq - t) <= step * 1.0 + 1e-30)


def test_rejects_ragged_columns():
    with pytest.raises(ValueError):
        group16.quantize(np.zeros((4, 24), np.float32))


def _lossless(rng, rows, cols, e):
    """A tensor whose 1x16 quantization is exact: E2M1 values times a per-group
    E4M3 scale times 2^e, with a 6 in every group so the scale is recovered and
    one group scaled by 448 so that the tensor maximum gives back e."""
    c = rng.choice([-6, -4, -3, -2, -1.5, -1, -0.5, 0, 0.5, 1, 1.5, 2, 3, 4, 6], size=(rows, cols))
    c[:, ::16] = 6.0
    sc = formats.e4m3_decode(rng.integers(0x30, 0x48, (rows, cols // 16)))
    sc[0, 0] = 448.0
    return c * np.repeat(sc, 16, axis=1) * 2.0 ** e


def test_layer_forward_lossless_triple_loop():
    rng = np.random.default_rng(10)
    M, K, N, r_s, r = 16, 32, 16, 2, 3
    X = _lossless(rng, M, K, -8)
    assert group16.tensor_exponent(np.abs(X).max()) == -8
    assert np.array_equal(group16.dequantize(*group16.quantize(X.astype(np.float32))), X)
    Rq = rng.standard_normal((N, K))
    f = lambda *s: formats.bf16_round(rng.standard_normal(s) * 0.1)
    S_dn, S_up, A, B, bias = f(K, r_s), f(r_s, N), f(K, r), f(r, N), f(N)
    out = layer.linear_fwd_1x16(X, Rq, S_dn, S_up, A, B, bias)
    Dm = np.concatenate([S_dn, A], 1)
    Um = np.concatenate([S_up, B], 0)
    L = np.zeros((M, r_s + r))
    for m in range(M):
        for j in range(r_s + r):
            L[m, j] = sum(X[m, k] * Dm[k, j] for k in range(K))
    L = formats.bf16_round(L)
    y = np.zeros((M, N))
    for m in range(M):
        for n in range(N):
            y[m, n] = (sum(X[m, k] * Rq[n, k] for k in range(K)) + sum(L[m, j] * Um[j, n] for j in range(r_s + r))
                       + bias[n])
    np.testing.assert_array_equal(out["L"], L)
    np.testing.assert_allclose(out["y"], y, rtol=1e-12, atol=1e-12)


def test_layer_backward_adjoint_on_lossless_operands():
    # with lossless G and R, dX's 4-bit part is the adjoint of the forward's:
    # <X R^T, G> = <X, G R> (R^T's groups run along N, so Q16(R^T) = R^T exactly)
    rng = np.random.default_rng(11)
    M, K, N, r_s, r = 16, 32, 48, 2, 2
    G = _lossless(rng, M, N, 3)
    Rt = _lossless(rng, K, N, -2)                             # R^T [K, N], groups along N
    X = formats.bf16_round(rng.standard_normal((M, K)))
    f = lambda *s: formats.bf16_round(rng.standard_normal(s) * 0.1)
    S_dn, S_up, A, B = f(K, r_s), f(r_s, N), f(K, r), f(r, N)
    L = formats.bf16_round(X @ np.concatenate([S_dn, A], 1))
    out = layer.linear_bwd_1x16(G, X, L, Rt, S_dn, S_up, A, B)
    P = out["P"]
    dX4 = out["dX"] - P @ np.concatenate([S_dn, A], 1).T
    np.testing.assert_allclose(np.sum((X @ Rt) * G), np.sum(X * dX4), rtol=1e-12)
    np.testing.assert_allclose(dX4, G @ Rt.T, rtol=1e-12, atol=1e-12)
    np.testing.assert_array_equal(out["dA"], X.T @ P[:, r_s:])
    np.testing.assert_array_equal(out["dB"], L[:, r_s:].T @ G)
