"""Pins for oracle/stabilizer.py (FourTune §3.1: a frozen low-rank stabilizer is
isolated from each weight and the rest is quantized; read as a truncated SVD).

The SVD is pinned by weights built from known orthogonal factors (a normalized
Hadamard matrix and a rotation): the truncated product must equal the known
rank-r_s part, and the residual the known remainder, whatever signs or order the
library returns.  The residual's rounding and the quantizer hand-off are pinned
by exact identities."""
import numpy as np

from oracle import block16, formats, stabilizer


def _hadamard(n):
    H = np.array([[1.0]])
    while H.shape[0] < n:
        H = np.block([[H, H], [H, -H]])
    return H / np.sqrt(n)


def _known(N=64, K=64, seed=0):
    rng = np.random.default_rng(seed)
    U = _hadamard(K)                                  # W^T = U diag(s) V^T
    theta = rng.uniform(0, np.pi)
    c, s_ = np.cos(theta), np.sin(theta)
    V = _hadamard(N) @ np.kron(np.eye(N // 2), np.array([[c, -s_], [s_, c]]))   # orthogonal
    s = np.sort(rng.uniform(0.5, 3.0, size=min(N, K)))[::-1] * np.geomspace(1, 1e-3, min(N, K))
    return U, s, V, (U * s[None, :]) @ V.T            # W^T


def test_truncated_product_equals_the_known_rank_r_part():
    U, s, V, Wt = _known()
    for r_s in (1, 8, 16):
        S_dn, S_up = stabilizer.truncated_factors(Wt.T, r_s)
        np.testing.assert_allclose(S_dn @ S_up, (U[:, :r_s] * s[None, :r_s]) @ V[:, :r_s].T, atol=1e-12)
        # the factors carry sqrt(s) each: column norms of S_dn are sqrt(s)
        np.testing.assert_allclose(np.linalg.norm(S_dn, axis=0), np.sqrt(s[:r_s]), rtol=1e-12)


def test_residual_is_the_known_remainder_and_eckart_young():
    U, s, V, Wt = _known(seed=1)
    r_s = 8
    S_dn, S_up = stabilizer.truncated_factors(Wt.T, r_s)
    rest = Wt - S_dn @ S_up
    np.testing.assert_allclose(rest, (U[:, r_s:] * s[None, r_s:]) @ V[:, r_s:].T, atol=1e-12)
    assert abs(np.linalg.norm(rest) ** 2 - np.sum(s[r_s:] ** 2)) < 1e-10


def test_low_rank_weight_leaves_only_the_factor_rounding():
    """A weight of rank r_s (or a full-rank split): the stabilizer takes all of it,
    and the residual is only what the factors' bf16 rounding leaves, at most a
    few bf16 ulps of the weight's largest entry."""
    rng = np.random.default_rng(2)
    K, N, r_s = 32, 48, 2
    P = rng.integers(-3, 4, size=(K, r_s)) / 4.0
    Q = rng.integers(-3, 4, size=(r_s, N)) / 4.0
    W = (P @ Q).T
    out = stabilizer.split(W, r_s)
    # the rounded product differs from W only by the factors' bf16 rounding
    assert np.abs(out["R"]).max() <= 2.0 ** -6 * np.abs(W).max()
    Wq = np.round(W * 4) / 4
    out2 = stabilizer.split(Wq, K)       # full rank: the residual is the factors' rounding alone
    assert np.abs(out2["R"]).max() <= 2.0 ** -6 * np.abs(Wq).max()


def test_residual_rounds_once_against_the_rounded_factors():
    rng = np.random.default_rng(3)
    W = formats.bf16_round(rng.standard_normal((32, 48)) * 0.02)
    out = stabilizer.split(W, 4)
    exact = W - (out["S_dn"] @ out["S_up"]).T
    np.testing.assert_array_equal(out["R"], formats.bf16_round(exact))
    np.testing.assert_array_equal(out["S_dn"], formats.bf16_round(out["S_dn"]))
    c, sc = block16.quantize(out["R"].astype(np.float32))
    np.testing.assert_array_equal(out["R_codes"], c)
    np.testing.assert_array_equal(out["R_scales"], sc)


def test_stabilizer_takes_the_outlier_directions():
    """§3.1's purpose: with a few large outlier directions in W, the stabilizer
    captures them and the residual's block scales shrink."""
    rng = np.random.default_rng(4)
    K = N = 128
    W = rng.standard_normal((N, K)) * 0.02
    W += 3.0 * np.outer(rng.standard_normal(N), rng.standard_normal(K)) / np.sqrt(K)
    W = formats.bf16_round(W)
    _, sc_full = block16.quantize(W.astype(np.float32))
    out = stabilizer.split(W, 4)
    dec = lambda s: formats.e4m3_decode(s)
    assert dec(out["R_scales"]).mean() < 0.5 * dec(sc_full).mean()
