"""Triple-branch W4A4G4 linear layer and its MLP pair, forward and backward.

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).

Follows FourTune:
  §3.1  y = (4-bit residual branch) + (frozen low-rank stabilizer) + (LoRA):
        y = deq(Q(X)) deq(Q(R))^T + (X S_dn) S_up + (X A) B  (+ bias)
  §3.2  backward: the gradient flows through all three branches; only the
        adapter (A, B) receives parameter gradients -- no gradient for R, S or
        bias.  The 4-bit branch uses Q(G) against the same blocks of Q(R) read
        transposed: dX = deq(Q(G)) deq(Q(R)) in this file's orientation
        (R is stored [N, K], so the pages' Q(G) Q(R)^T is the same product).
  §3.3  LoRA fusion: all three branches share the same input (X forward, G
        backward); MLP fusion: FC1 -> GELU -> FC2 quantization.

Readings of what the pages leave open (each is also listed in the design notes):
  * The low-rank branches take the full-precision bf16 input (X, G), not Q(X).
  * The down-projections L = X [S_dn | A] and P = G [S_up ; B]^T are rounded to
    bf16 (ties-to-even) once, after exact accumulation: they feed bf16 products.
  * dA = X^T P[:, r_s:]   and   dB = L[:, r_s:]^T G   (straight-through: Q has
    no derivative of its own).
  * MLP: h = bf16(FC1(X) + b1) is the saved hidden; a = GELU_tanh(h) (float32);
    FC2's three branches share one input, bf16(a) -- Q(bf16(a)) for the 4-bit
    branch, bf16(a) for the low-rank ones -- as every layer's input is a bf16
    tensor (§3.3 "LoRA Fusion").  Backward: d_a from FC2, d_h =
    bf16(d_a * GELU'(h)) -- the gradient reaching FC1 is a bf16 tensor like any
    layer's incoming gradient, and all three of FC1's branches take it (Q(d_h)
    for the 4-bit branch).

All GEMMs run in float64 on the exactly dequantized operands; a library matmul
is the only primitive used.
"""
import numpy as np

from . import block16, formats, group16


def _f64(a):
    return np.asarray(a, dtype=np.float64)


def _D(S_dn, A):
    return np.concatenate([_f64(S_dn), _f64(A)], axis=1)      # [K, r_s + r]


def _U(S_up, B):
    return np.concatenate([_f64(S_up), _f64(B)], axis=0)      # [r_s + r, N]


def linear_fwd(X, R_codes, R_scales, S_dn, S_up, A, B, bias=None, Qx=None):
    """Forward.  X [M, K] (bf16 values), R codes [N, K/2] / scales [N/16, K/16].

    Returns dict(y [M, N] float64, L [M, r_s+r] bf16 values, qx_codes, qx_scales).
    `Qx` may pass precomputed (codes, scales) of the 4-bit input (used for the
    MLP's FC2 whose 4-bit input is Q(a) of a float32 a).
    """
    X = _f64(X)
    if Qx is None:
        Qx = block16.quantize(X.astype(np.float32))
    qx_codes, qx_scales = Qx
    Xq = block16.dequantize(qx_codes, qx_scales)
    Rq = block16.dequantize(R_codes, R_scales)
    L = formats.bf16_round(X @ _D(S_dn, A))
    y = Xq @ Rq.T + L @ _U(S_up, B)
    if bias is not None:
        y = y + _f64(bias)[None, :]
    return dict(y=y, L=L, qx_codes=qx_codes, qx_scales=qx_scales)


def linear_bwd(G, X, L, R_codes, R_scales, S_dn, S_up, A, B, Qg=None):
    """Backward.  G = dL/dy [M, N] (bf16 values), X [M, K] (bf16 values),
    L [M, r_s+r] saved by the forward.

    Returns dict(dX [M, K], dA [K, r], dB [r, N], P [M, r_s+r] bf16 values,
    qg_codes, qg_scales).  `Qg` may pass a precomputed 4-bit gradient (MLP).
    """
    G = _f64(G)
    X = _f64(X)
    L = _f64(L)
    r_s = np.asarray(S_dn).shape[1]
    if Qg is None:
        Qg = block16.quantize(G.astype(np.float32))
    qg_codes, qg_scales = Qg
    Gq = block16.dequantize(qg_codes, qg_scales)
    Rq = block16.dequantize(R_codes, R_scales)
    D = _D(S_dn, A)
    U = _U(S_up, B)
    P = formats.bf16_round(G @ U.T)
    dX = Gq @ Rq + P @ D.T
    dA = X.T @ P[:, r_s:]
    dB = L[:, r_s:].T @ G
    return dict(dX=dX, dA=dA, dB=dB, P=P, qg_codes=qg_codes, qg_scales=qg_scales)


# -------------------------------------------------------------- precision variants
# §4.3 (Table 4) ablates which tensors are 4-bit: W4A16G4, W4A4G16, W4A16G16 next
# to W4A4G4.  A 16-bit activation or gradient enters its GEMM unquantized (bf16);
# the weight is always the 4-bit one, seen by the GEMM as Rq = deq(Q(R)).  The
# low-rank branches are the same as in linear_fwd / linear_bwd.  With a bf16
# weight in place of Rq and no stabilizer (r_s = 0), the 16-bit forward and
# backward are the standard bf16 LoRA layer the pages compare against (§4.2).

def linear_fwd_a16(X, Rq, S_dn, S_up, A, B, bias=None):
    """Forward with a 16-bit activation: y = X Rq^T + L [S_up ; B] (+ bias),
    L = bf16(X [S_dn | A]).  Rq [N, K] in float64 (exact values).
    Returns dict(y, L)."""
    X = _f64(X)
    L = formats.bf16_round(X @ _D(S_dn, A))
    y = X @ _f64(Rq).T + L @ _U(S_up, B)
    if bias is not None:
        y = y + _f64(bias)[None, :]
    return dict(y=y, L=L)


def linear_bwd_g16(G, X, L, Rq, S_dn, S_up, A, B):
    """Backward with a 16-bit gradient: dX = G Rq + P [S_dn | A]^T with
    P = bf16(G [S_up ; B]^T); dA = X^T P[:, r_s:], dB = L[:, r_s:]^T G as in
    linear_bwd.  Returns dict(dX, dA, dB, P)."""
    G = _f64(G)
    X = _f64(X)
    L = _f64(L)
    r_s = np.asarray(S_dn).shape[1]
    P = formats.bf16_round(G @ _U(S_up, B).T)
    dX = G @ _f64(Rq) + P @ _D(S_dn, A).T
    return dict(dX=dX, dA=X.T @ P[:, r_s:], dB=L[:, r_s:].T @ G, P=P)


# ------------------------------------------------------- 1x16 group-wise variant
# §4.3 (Table 5) compares the 16x16 blocks with 1x16 groups (group16.py): the
# same triple-branch layer with X, G and the weight quantized in 1x16 groups
# along each GEMM's reduction dimension, plus a per-tensor scale.  The weight
# has two quantized forms: Q16(R) [N, K] (groups along K) for the forward, and
# Q16(R^T) [K, N] (groups along N) for dX -- the transposed operand is
# quantized again, which the block layout avoids (§3.2).

def linear_fwd_1x16(X, Rq, S_dn, S_up, A, B, bias=None, Qx=None):
    """Forward: y = deq(Q16(X)) Rq^T + L [S_up ; B] (+ bias), L = bf16(X [S_dn | A]).
    Rq = deq(Q16(R)) [N, K] in float64.  Returns dict(y, L, qx_codes, qx_scales, qx_e)."""
    X = _f64(X)
    if Qx is None:
        Qx = group16.quantize(X.astype(np.float32))
    codes, scales, e = Qx
    L = formats.bf16_round(X @ _D(S_dn, A))
    y = group16.dequantize(codes, scales, e) @ _f64(Rq).T + L @ _U(S_up, B)
    if bias is not None:
        y = y + _f64(bias)[None, :]
    return dict(y=y, L=L, qx_codes=codes, qx_scales=scales, qx_e=e)


def linear_bwd_1x16(G, X, L, Rtq, S_dn, S_up, A, B, Qg=None):
    """Backward: dX = deq(Q16(G)) Rtq^T + P [S_dn | A]^T with Rtq = deq(Q16(R^T))
    [K, N] and P = bf16(G [S_up ; B]^T); dA, dB as in linear_bwd.
    Returns dict(dX, dA, dB, P, qg_codes, qg_scales, qg_e)."""
    G = _f64(G)
    X = _f64(X)
    L = _f64(L)
    r_s = np.asarray(S_dn).shape[1]
    if Qg is None:
        Qg = group16.quantize(G.astype(np.float32))
    codes, scales, e = Qg
    P = formats.bf16_round(G @ _U(S_up, B).T)
    dX = group16.dequantize(codes, scales, e) @ _f64(Rtq).T + P @ _D(S_dn, A).T
    return dict(dX=dX, dA=X.T @ P[:, r_s:], dB=L[:, r_s:].T @ G, P=P, qg_codes=codes, qg_scales=scales, qg_e=e)


# ------------------------------------------------------------------------- MLP
_GELU_C = np.sqrt(2.0 / np.pi)
_GELU_K = 0.044715


def gelu_tanh(h):
    """GELU, tanh form: 0.5 h (1 + tanh(sqrt(2/pi) (h + 0.044715 h^3))).

    Evaluated through the identity 0.5 (1 + tanh u) = 1 / (1 + e^{-2u}): the same
    function, without the cancellation of 1 + tanh u for very negative u (which
    in float64 loses every digit below u ~ -18)."""
    h = _f64(h)
    u = _GELU_C * (h + _GELU_K * h ** 3)
    with np.errstate(over="ignore"):
        return h / (1.0 + np.exp(-2.0 * u))


def gelu_tanh_grad(h):
    """d/dh of gelu_tanh, closed form: with s = 0.5 (1 + tanh u) = 1 / (1 + e^{-2u}),
    1 - tanh(u)^2 = 4 s (1 - s) and 1 - s = 1 / (1 + e^{2u}), so
    GELU'(h) = s + 2 h s (1 - s) sqrt(2/pi) (1 + 3 * 0.044715 h^2)."""
    h = _f64(h)
    u = _GELU_C * (h + _GELU_K * h ** 3)
    with np.errstate(over="ignore"):
        s = 1.0 / (1.0 + np.exp(-2.0 * u))
        sc = 1.0 / (1.0 + np.exp(2.0 * u))
    return s + 2.0 * h * s * sc * _GELU_C * (1.0 + 3.0 * _GELU_K * h * h)


def mlp_fwd(X, fc1, fc2, a_f32=None):
    """FC1 -> GELU(tanh) -> FC2, both triple-branch layers.

    fc1/fc2: dict(R_codes, R_scales, S_dn, S_up, A, B, bias).
    `a_f32` optionally overrides the float32 activation a (the GPU's own, so
    that downstream results compare on identical operands); FC2's input is
    bf16(a) for all three of its branches.
    Returns dict(y, h, a, L1, L2, qa_codes, qa_scales, ...).
    """
    o1 = linear_fwd(X, fc1["R_codes"], fc1["R_scales"], fc1["S_dn"], fc1["S_up"],
                    fc1["A"], fc1["B"], fc1.get("bias"))
    h = formats.bf16_round(o1["y"])
    a = gelu_tanh(h)
    a32 = a.astype(np.float32) if a_f32 is None else np.asarray(a_f32, dtype=np.float32)
    a_bf = formats.bf16_round(a32.astype(np.float64))
    Qa = block16.quantize(a_bf.astype(np.float32))
    o2 = linear_fwd(a_bf, fc2["R_codes"], fc2["R_scales"], fc2["S_dn"], fc2["S_up"],
                    fc2["A"], fc2["B"], fc2.get("bias"), Qx=Qa)
    return dict(y=o2["y"], h=h, a=a, a32=a32, a_bf=a_bf, L1=o1["L"], L2=o2["L"],
                qx_codes=o1["qx_codes"], qx_scales=o1["qx_scales"],
                qa_codes=Qa[0], qa_scales=Qa[1])


def mlp_bwd(G, X, h, L1, L2, fc1, fc2, dh_bf=None, a_bf=None):
    """Backward of mlp_fwd.  G = dL/dy [M, N2].  h, L1, L2 as saved by the forward.

    `dh_bf` optionally overrides the bf16 d_h that FC1's backward consumes (the
    GPU's own, so that FC1's results compare on identical operands).
    `a_bf` optionally overrides FC2's low-rank input bf16(a) (else recomputed
    from h as in the forward).
    Returns dict(dX, dA1, dB1, dA2, dB2, d_a, d_h, ...).
    """
    h = _f64(h)
    if a_bf is None:
        a_bf = formats.bf16_round(gelu_tanh(h).astype(np.float32).astype(np.float64))
    b2 = linear_bwd(G, a_bf, L2, fc2["R_codes"], fc2["R_scales"], fc2["S_dn"], fc2["S_up"],
                    fc2["A"], fc2["B"])
    d_a = b2["dX"]
    d_h = d_a * gelu_tanh_grad(h)
    dh = formats.bf16_round(d_h) if dh_bf is None else np.asarray(dh_bf, dtype=np.float64)
    Qdh = block16.quantize(dh.astype(np.float32))
    b1 = linear_bwd(dh, X, L1, fc1["R_codes"], fc1["R_scales"], fc1["S_dn"], fc1["S_up"],
                    fc1["A"], fc1["B"], Qg=Qdh)
    return dict(dX=b1["dX"], dA1=b1["dA"], dB1=b1["dB"], dA2=b2["dA"], dB2=b2["dB"],
                d_a=d_a, d_h=d_h, dh_bf=dh, a_bf=a_bf, P1=b1["P"], P2=b2["P"],
                qdh_codes=Qdh[0], qdh_scales=Qdh[1], qg_codes=b2["qg_codes"],
                qg_scales=b2["qg_scales"])
