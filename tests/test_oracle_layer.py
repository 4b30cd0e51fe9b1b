"""Pins for oracle/layer.py (FourTune §3.1 triple branch, §3.2 backward, §3.3 MLP).

Operands are built so that quantization and the bf16 roundings are lossless
(every 16x16 block holds E2M1-grid multiples of an E4M3 value d with one
element at 6d; the low-rank factors are sparse dyadics).  Then the layer must
equal the plain matrix definition exactly, which a triple loop checks; the
backward must satisfy the adjoint identity and exact finite differences.  The
MLP's chain rule is checked against torch autograd with quantization and
rounding replaced by the identity.
"""
import numpy as np
import pytest
import torch

from oracle import block16, formats, layer


def lossless(rows, cols, d, rng):
    grid = np.concatenate([formats.E2M1_MAGNITUDES, -formats.E2M1_MAGNITUDES])
    t = rng.choice(grid, size=(rows, cols)) * d
    for bi in range(rows // 16):
        for bj in range(cols // 16):
            t[bi * 16 + rng.integers(16), bj * 16 + rng.integers(16)] = 6 * d * rng.choice([-1, 1])
    return t.astype(np.float32).astype(np.float64)


def sparse_dyadic(rows, cols, rng, per_col=2, axis=0):
    """Each column (axis=0) or row (axis=1) has at most `per_col` entries of +-1/16."""
    t = np.zeros((rows, cols))
    if axis == 0:
        for j in range(cols):
            idx = rng.choice(rows, size=per_col, replace=False)
            t[idx, j] = rng.choice([-1, 1], size=per_col) / 16
    else:
        for i in range(rows):
            idx = rng.choice(cols, size=per_col, replace=False)
            t[i, idx] = rng.choice([-1, 1], size=per_col) / 16
    return t


def make_case(M=32, K=48, N=32, r_s=2, r=3, seed=0):
    rng = np.random.default_rng(seed)
    X = lossless(M, K, 0.25, rng)
    R = lossless(N, K, 0.125, rng)
    G = lossless(M, N, 0.5, rng)
    S_dn = sparse_dyadic(K, r_s, rng)
    A = sparse_dyadic(K, r, rng)
    S_up = sparse_dyadic(r_s, N, rng, axis=1)
    B = sparse_dyadic(r, N, rng, axis=1)
    Rc, Rs = block16.quantize(R.astype(np.float32))
    return dict(X=X, R=R, G=G, S_dn=S_dn, A=A, S_up=S_up, B=B, Rc=Rc, Rs=Rs, r_s=r_s, r=r)


def fwd(c, **kw):
    p = dict(S_dn=c["S_dn"], S_up=c["S_up"], A=c["A"], B=c["B"])
    p.update(kw)
    return layer.linear_fwd(c["X"], c["Rc"], c["Rs"], p["S_dn"], p["S_up"], p["A"], p["B"], p.get("bias"))


def bwd(c, L, **kw):
    p = dict(S_dn=c["S_dn"], S_up=c["S_up"], A=c["A"], B=c["B"])
    p.update(kw)
    return layer.linear_bwd(c["G"], c["X"], L, c["Rc"], c["Rs"], p["S_dn"], p["S_up"], p["A"], p["B"])


def test_lossless_construction():
    c = make_case()
    np.testing.assert_array_equal(block16.dequantize(c["Rc"], c["Rs"]), c["R"])
    o = fwd(c)
    np.testing.assert_array_equal(block16.dequantize(o["qx_codes"], o["qx_scales"]), c["X"])


def test_forward_equals_triple_loop():
    c = make_case(M=16, K=32, N=32, r_s=2, r=2, seed=1)
    X, R, S_dn, A, S_up, B = (c[k] for k in ("X", "R", "S_dn", "A", "S_up", "B"))
    bias = np.arange(32) / 64.0
    M, K = X.shape
    N = R.shape[0]
    D = [[(S_dn[k][j] if j < 2 else A[k][j - 2]) for j in range(4)] for k in range(K)]
    U = [[(S_up[j][n] if j < 2 else B[j - 2][n]) for n in range(N)] for j in range(4)]
    want = np.zeros((M, N))
    for m in range(M):
        Lrow = [sum(X[m][k] * D[k][j] for k in range(K)) for j in range(4)]
        for n in range(N):
            acc = sum(X[m][k] * R[n][k] for k in range(K))
            acc += sum(Lrow[j] * U[j][n] for j in range(4))
            want[m][n] = acc + bias[n]
    got = fwd(c, bias=bias)["y"]
    np.testing.assert_array_equal(got, want)


def test_backward_equals_triple_loop():
    c = make_case(M=16, K=32, N=32, r_s=2, r=2, seed=2)
    X, R, G, S_dn, A, S_up, B = (c[k] for k in ("X", "R", "G", "S_dn", "A", "S_up", "B"))
    M, K = X.shape
    N = R.shape[0]
    L = fwd(c)["L"]
    o = bwd(c, L)
    D = np.concatenate([S_dn, A], 1)
    U = np.concatenate([S_up, B], 0)
    dX = np.zeros((M, K))
    dA = np.zeros((K, 2))
    dB = np.zeros((2, N))
    for m in range(M):
        P = [sum(G[m][n] * U[j][n] for n in range(N)) for j in range(4)]
        for k in range(K):
            dX[m][k] = sum(G[m][n] * R[n][k] for n in range(N)) + sum(P[j] * D[k][j] for j in range(4))
            for j in range(2):
                dA[k][j] += X[m][k] * P[2 + j]
        for j in range(2):
            for n in range(N):
                dB[j][n] += L[m][2 + j] * G[m][n]
    np.testing.assert_array_equal(o["dX"], dX)
    np.testing.assert_array_equal(o["dA"], dA)
    np.testing.assert_array_equal(o["dB"], dB)


def test_adjoint_identity():
    c = make_case(seed=3)
    o = fwd(c)
    b = bwd(c, o["L"])
    lhs = np.sum(c["G"] * o["y"])
    rhs = np.sum(b["dX"] * c["X"])
    assert lhs == rhs


def test_dA_dB_exact_finite_differences():
    c = make_case(seed=4)
    base = fwd(c)
    b = bwd(c, base["L"])
    loss0 = np.sum(c["G"] * base["y"])
    delta = 1.0 / 16
    rng = np.random.default_rng(0)
    for _ in range(6):
        j, n = rng.integers(c["r"]), rng.integers(c["B"].shape[1])
        B2 = c["B"].copy()
        B2[j, n] += delta
        assert (np.sum(c["G"] * fwd(c, B=B2)["y"]) - loss0) / delta == b["dB"][j, n]
        k, j = rng.integers(c["A"].shape[0]), rng.integers(c["r"])
        A2 = c["A"].copy()
        A2[k, j] += delta
        assert (np.sum(c["G"] * fwd(c, A=A2)["y"]) - loss0) / delta == b["dA"][k, j]


def test_special_cases():
    c = make_case(seed=5)
    zB = np.zeros_like(c["B"])
    o = fwd(c, B=zB)
    b = bwd(c, o["L"], B=zB)
    assert np.all(b["dA"] == 0)                         # B = 0 -> no gradient reaches A
    # dB does not depend on B
    b2 = bwd(c, o["L"], B=c["B"] * 3)
    np.testing.assert_array_equal(b["dB"], b2["dB"])
    # S = A = B = 0 -> only the 4-bit branch remains
    z = dict(S_dn=np.zeros_like(c["S_dn"]), A=np.zeros_like(c["A"]),
             S_up=np.zeros_like(c["S_up"]), B=zB)
    o0 = fwd(c, **z)
    np.testing.assert_array_equal(o0["y"], c["X"] @ c["R"].T)
    b0 = bwd(c, o0["L"], **z)
    np.testing.assert_array_equal(b0["dX"], c["G"] @ c["R"])


def test_frozen_parts_get_no_gradient():
    c = make_case(seed=6)
    o = fwd(c)
    b = bwd(c, o["L"])
    assert set(b) >= {"dX", "dA", "dB"}
    assert not ({"dR", "dS_dn", "dS_up", "dbias"} & set(b))   # §3.2: only the adapter updates


def test_16bit_variants_equal_triple_loops():
    """W4A16 forward and G16 backward (§4.3, Table 4) on unquantized bf16-like
    operands against triple loops (the activation / gradient is not quantized)."""
    rng = np.random.default_rng(5)
    M, K, N, r_s, r = 16, 32, 16, 2, 3
    f = lambda *s: formats.bf16_round(rng.standard_normal(s))
    X, G, Rq = f(M, K), f(M, N), f(N, K)
    S_dn, A, S_up, B = f(K, r_s), f(K, r), f(r_s, N), f(r, N)
    D, U = np.concatenate([S_dn, A], 1), np.concatenate([S_up, B], 0)
    o = layer.linear_fwd_a16(X, Rq, S_dn, S_up, A, B)
    L = np.zeros((M, r_s + r))
    for m in range(M):
        for j in range(r_s + r):
            L[m, j] = sum(X[m, k] * D[k, j] for k in range(K))
    L = formats.bf16_round(L)
    np.testing.assert_array_equal(o["L"], L)
    y = np.zeros((M, N))
    for m in range(M):
        for n in range(N):
            y[m, n] = sum(X[m, k] * Rq[n, k] for k in range(K)) + sum(L[m, j] * U[j, n] for j in range(r_s + r))
    np.testing.assert_allclose(o["y"], y, rtol=1e-13, atol=1e-13)
    b = layer.linear_bwd_g16(G, X, L, Rq, S_dn, S_up, A, B)
    P = np.zeros((M, r_s + r))
    for m in range(M):
        for j in range(r_s + r):
            P[m, j] = sum(G[m, n] * U[j, n] for n in range(N))
    P = formats.bf16_round(P)
    np.testing.assert_array_equal(b["P"], P)
    dX = np.zeros((M, K))
    for m in range(M):
        for k in range(K):
            dX[m, k] = sum(G[m, n] * Rq[n, k] for n in range(N)) + sum(P[m, j] * D[k, j] for j in range(r_s + r))
    np.testing.assert_allclose(b["dX"], dX, rtol=1e-13, atol=1e-13)
    dA = np.array([[sum(X[m, k] * P[m, r_s + j] for m in range(M)) for j in range(r)] for k in range(K)])
    dB = np.array([[sum(L[m, r_s + j] * G[m, n] for m in range(M)) for n in range(N)] for j in range(r)])
    np.testing.assert_allclose(b["dA"], dA, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(b["dB"], dB, rtol=1e-13, atol=1e-13)


def test_16bit_variants_coincide_with_4bit_on_lossless_operands():
    """When X and G are exactly representable in block16 FP4 (quantization is the
    identity), every precision variant is the W4A4G4 layer, exactly."""
    c = make_case(seed=4)
    Rq = block16.dequantize(c["Rc"], c["Rs"])
    o4, o16 = fwd(c), layer.linear_fwd_a16(c["X"], Rq, c["S_dn"], c["S_up"], c["A"], c["B"])
    np.testing.assert_array_equal(o16["y"], o4["y"])
    np.testing.assert_array_equal(o16["L"], o4["L"])
    b4 = bwd(c, o4["L"])
    b16 = layer.linear_bwd_g16(c["G"], c["X"], o4["L"], Rq, c["S_dn"], c["S_up"], c["A"], c["B"])
    for k in ("dX", "dA", "dB", "P"):
        np.testing.assert_array_equal(b16[k], b4[k])


def test_16bit_variants_differ_from_4bit_on_generic_operands():
    """On operands that are not on the FP4 grid, the 16-bit activation path does not
    see the quantization error: its difference from W4A4 is the 4-bit branch's
    (Q(X) - X) R^T, exactly."""
    rng = np.random.default_rng(6)
    c = make_case(seed=6)
    X = formats.bf16_round(rng.standard_normal(c["X"].shape))
    Rq = block16.dequantize(c["Rc"], c["Rs"])
    o4 = layer.linear_fwd(X, c["Rc"], c["Rs"], c["S_dn"], c["S_up"], c["A"], c["B"])
    o16 = layer.linear_fwd_a16(X, Rq, c["S_dn"], c["S_up"], c["A"], c["B"])
    Xq = block16.dequantize(o4["qx_codes"], o4["qx_scales"])
    assert np.abs(Xq - X).max() > 0
    np.testing.assert_allclose(o4["y"] - o16["y"], (Xq - X) @ Rq.T, rtol=1e-12, atol=1e-12)


def test_gelu_matches_torch():
    h = np.linspace(-9, 9, 20001)
    th = torch.tensor(h, requires_grad=True)
    g = torch.nn.functional.gelu(th, approximate="tanh")
    g.sum().backward()
    np.testing.assert_allclose(layer.gelu_tanh(h), g.detach().numpy(), rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(layer.gelu_tanh_grad(h), th.grad.numpy(), rtol=1e-12, atol=1e-14)


_PI = "3.14159265358979323846264338327950288419716939937510582097494459"


def _gelu_exact(x):
    """The textbook tanh form 0.5 x (1 + tanh u), u = sqrt(2/pi) (x + 0.044715 x^3),
    in the current decimal context (tanh from exp), with enough digits that
    1 + tanh u keeps its own significant digits where float64 has none left."""
    import decimal
    D = decimal.Decimal
    u = (D(2) / D(_PI)).sqrt() * (x + D("0.044715") * x ** 3)
    e2 = (2 * u).exp()
    return D("0.5") * x * (1 + (e2 - 1) / (e2 + 1))


def test_gelu_against_high_precision_textbook_form():
    """Relative agreement with the 120-digit evaluation of 0.5 h (1 + tanh u) from
    h = -12 (GELU ~ -1e-61, where float64's 1 + tanh u has lost every digit; 120
    digits keep ~50 of them there) to 12."""
    import decimal
    hs = np.concatenate([np.linspace(-12, 12, 241), [-1e-3, 1e-3, -0.75]])
    for h in hs[hs != 0]:
        with decimal.localcontext() as ctx:
            ctx.prec = 120
            ref = _gelu_exact(decimal.Decimal(float(h)))
            got = layer.gelu_tanh(np.float64(h))
            rel = abs((decimal.Decimal(float(got)) - ref) / ref)
        assert rel < 1e-13, (h, got, ref)
    assert layer.gelu_tanh(np.float64(0.0)) == 0.0
    assert layer.gelu_tanh(np.float64(-1e30)) == 0.0 and layer.gelu_tanh(np.float64(1e30)) == 1e30


def test_gelu_grad_against_high_precision_difference_quotient():
    """The closed-form derivative against a central difference of the 120-digit
    textbook form (step 1e-25, truncation error ~1e-50), absolute error relative
    to 1 + |h|^3 (the size of the derivative's terms; it crosses zero near -0.75)."""
    import decimal
    for h in np.linspace(-10, 10, 101):
        with decimal.localcontext() as ctx:
            ctx.prec = 120
            d = decimal.Decimal("1e-25")
            x = decimal.Decimal(float(h))
            ref = float((_gelu_exact(x + d) - _gelu_exact(x - d)) / (2 * d))
        got = layer.gelu_tanh_grad(np.float64(h))
        assert abs(got - ref) <= 1e-13 * (1.0 + abs(h) ** 3), (h, got, ref)


def test_mlp_chain_rule_vs_autograd(monkeypatch):
    """With Q and the bf16 roundings replaced by the identity, mlp_fwd/mlp_bwd must be
    the float64 function FC2(GELU(FC1(X))) and its exact gradient."""
    monkeypatch.setattr(block16, "quantize", lambda t: (np.asarray(t, np.float64), "id"))
    monkeypatch.setattr(block16, "dequantize", lambda c, s: np.asarray(c, np.float64))
    monkeypatch.setattr(formats, "bf16_round", lambda x: np.asarray(x, np.float64))
    rng = np.random.default_rng(8)
    M, K, H, N, r_s, r = 8, 12, 20, 10, 2, 3

    def lin(K_, N_):
        return dict(R_codes=rng.standard_normal((N_, K_)) * 0.3, R_scales=None,
                    S_dn=rng.standard_normal((K_, r_s)) * 0.3, S_up=rng.standard_normal((r_s, N_)) * 0.3,
                    A=rng.standard_normal((K_, r)) * 0.3, B=rng.standard_normal((r, N_)) * 0.3,
                    bias=rng.standard_normal(N_) * 0.1)
    fc1, fc2 = lin(K, H), lin(H, N)
    X = rng.standard_normal((M, K))
    G = rng.standard_normal((M, N))
    f = layer.mlp_fwd(X, fc1, fc2)
    b = layer.mlp_bwd(G, X, f["h"], f["L1"], f["L2"], fc1, fc2, a_bf=f["a32"].astype(np.float64))

    T = lambda a: torch.tensor(a, dtype=torch.float64, requires_grad=True)
    tX = T(X)
    t1 = {k: T(v) for k, v in fc1.items() if v is not None}
    t2 = {k: T(v) for k, v in fc2.items() if v is not None}

    def tl(x, p):
        return x @ p["R_codes"].T + (x @ p["S_dn"]) @ p["S_up"] + (x @ p["A"]) @ p["B"] + p["bias"]
    hh = tl(tX, t1)
    y = tl(torch.nn.functional.gelu(hh, approximate="tanh"), t2)
    (y * torch.tensor(G)).sum().backward()
    # float32 casts inside the oracle (a, d_h) limit agreement to ~1e-7 relative
    np.testing.assert_allclose(f["y"], y.detach().numpy(), rtol=2e-6, atol=2e-6)
    np.testing.assert_allclose(b["dX"], tX.grad.numpy(), rtol=2e-6, atol=2e-6)
    np.testing.assert_allclose(b["dA1"], t1["A"].grad.numpy(), rtol=2e-6, atol=2e-6)
    np.testing.assert_allclose(b["dB1"], t1["B"].grad.numpy(), rtol=2e-6, atol=2e-6)
    np.testing.assert_allclose(b["dA2"], t2["A"].grad.numpy(), rtol=2e-6, atol=2e-6)
    np.testing.assert_allclose(b["dB2"], t2["B"].grad.numpy(), rtol=2e-6, atol=2e-6)
