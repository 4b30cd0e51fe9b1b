"""Python binding of libfourtune.so: argument marshalling only.

Every step of the layer runs in the library's CUDA kernels; PyTorch supplies
device memory and the current stream.  There is no fallback: if the library is
missing or the device is not sm_100, calls raise.

Names follow the C ABI in include/fourtune/fourtune.h (FourTune §3.1-§3.3):
quantize_block16, transpose_codes, linear_fwd, linear_bwd.
"""
import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfourtune.so")

FT_DTYPE_F32 = 0
FT_DTYPE_BF16 = 1
ERRORS = {0: "FT_OK", -1: "FT_ERR_INVALID_ARG", -2: "FT_ERR_SHAPE", -3: "FT_ERR_ALIGN",
          -4: "FT_ERR_WORKSPACE", -5: "FT_ERR_CUDA", -6: "FT_ERR_TIMEOUT", -7: "FT_ERR_UNSUPPORTED"}

EXPORTED = ("fourtune_quantize_block16", "fourtune_transpose_codes", "fourtune_linear_fwd_workspace_size",
            "fourtune_linear_bwd_workspace_size", "fourtune_linear_fwd", "fourtune_linear_bwd",
            "fourtune_linear_fwd_ws_offsets", "fourtune_linear_bwd_ws_offsets", "fourtune_device_status",
            "fourtune_error_string", "fourtune_linear_fwd_timed", "fourtune_linear_bwd_timed",
            "fourtune_quant_down_static", "fourtune_mlp_fwd_workspace_size", "fourtune_mlp_fwd",
            "fourtune_mlp_bwd_workspace_size", "fourtune_mlp_bwd", "fourtune_mlp_fwd_ws_offsets",
            "fourtune_mlp_bwd_ws_offsets", "fourtune_mma_scales_size", "fourtune_mma_scales",
            "fourtune_mlp_fwd_timed", "fourtune_mlp_bwd_timed", "fourtune_quantize_block16_f32",
            "fourtune_quant_down_static_status", "fourtune_test_wait_timeout", "fourtune_dequantize_block16",
            "fourtune_linear_fwd_a16", "fourtune_linear_bwd_g16", "fourtune_linear_fwd_a16_workspace_size",
            "fourtune_linear_bwd_g16_workspace_size", "fourtune_stabilizer_residual", "fourtune_gemm_block16",
            "fourtune_quantize_1x16", "fourtune_linear_fwd_1x16_workspace_size",
            "fourtune_linear_bwd_1x16_workspace_size", "fourtune_linear_fwd_1x16", "fourtune_linear_bwd_1x16",
            "fourtune_linear_fwd_1x16_timed", "fourtune_linear_bwd_1x16_timed", "fourtune_linear_1x16_ws_offsets")
SIZE_FUNCS = ("fourtune_linear_fwd_workspace_size", "fourtune_linear_bwd_workspace_size", "fourtune_mma_scales_size",
              "fourtune_mlp_fwd_workspace_size", "fourtune_mlp_bwd_workspace_size",
              "fourtune_linear_fwd_a16_workspace_size", "fourtune_linear_bwd_g16_workspace_size",
              "fourtune_linear_fwd_1x16_workspace_size", "fourtune_linear_bwd_1x16_workspace_size")

# kernels each call launches, in order (the *_timed entry points bracket each with events)
FWD_KERNELS = ("xpass_quant_down", "gemm_fp4_fwd")
BWD_KERNELS = ("gpass_quant_down", "tgrad_dA_dB", "gemm_fp4_dx")
FWD_1X16_KERNELS = ("amax_x", "xpass_quant_down_1x16", "scale_u", "gemm_fp4_fwd_1x16")
BWD_1X16_KERNELS = ("amax_g", "gpass_quant_down_1x16", "scale_d", "tgrad_dA_dB", "gemm_fp4_dx_1x16")
MLP_FWD_KERNELS = ("xpass_quant_down", "gemm_fp4_fc1_gelu_quant_proj", "proj_reduce_l2", "gemm_fp4_fc2")
MLP_BWD_KERNELS = ("gpass_quant_down_fc2", "gemm_fp4_dx_fc2_gelu_bwd_quant_proj", "proj_reduce_p1", "tgrad_fc2",
                   "tgrad_fc1",
                   "gemm_fp4_dx_fc1")


class FourtuneError(RuntimeError):
    def __init__(self, code, where):
        super().__init__(f"{where}: {ERRORS.get(code, code)} ({code})")
        self.code = code


class ft_linear_t(ctypes.Structure):
    _fields_ = [("K", ctypes.c_int64), ("N", ctypes.c_int64), ("r_s", ctypes.c_int64), ("r", ctypes.c_int64),
                ("R_codes", ctypes.c_void_p), ("R_scales", ctypes.c_void_p), ("R_codes_t", ctypes.c_void_p),
                ("D", ctypes.c_void_p), ("U", ctypes.c_void_p), ("bias", ctypes.c_void_p),
                ("R_sf", ctypes.c_void_p), ("R_sf_t", ctypes.c_void_p)]


class ft_linear_1x16_t(ctypes.Structure):
    _fields_ = [("K", ctypes.c_int64), ("N", ctypes.c_int64), ("r_s", ctypes.c_int64), ("r", ctypes.c_int64),
                ("R_codes", ctypes.c_void_p), ("R_sf", ctypes.c_void_p), ("Rt_codes", ctypes.c_void_p),
                ("Rt_sf", ctypes.c_void_p), ("R_amax", ctypes.c_void_p), ("D", ctypes.c_void_p),
                ("U", ctypes.c_void_p), ("bias", ctypes.c_void_p)]


_lib = None


def load():
    """Load libfourtune.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m bit_lora_fine_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    vp, i64, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t
    P = ctypes.POINTER
    L.fourtune_quantize_block16.argtypes = [vp, i64, i64, i64, vp, vp, vp, vp]
    L.fourtune_transpose_codes.argtypes = [vp, i64, i64, vp, vp]
    L.fourtune_quantize_block16_f32.argtypes = [vp, i64, i64, i64, vp, vp, vp]
    L.fourtune_mma_scales_size.argtypes = [i64, i64]
    L.fourtune_mma_scales_size.restype = sz
    L.fourtune_mma_scales.argtypes = [vp, i64, i64, ctypes.c_int, vp, vp]
    L.fourtune_linear_fwd_workspace_size.argtypes = [P(ft_linear_t), i64]
    L.fourtune_linear_fwd_workspace_size.restype = sz
    L.fourtune_linear_bwd_workspace_size.argtypes = [P(ft_linear_t), i64]
    L.fourtune_linear_bwd_workspace_size.restype = sz
    L.fourtune_linear_fwd.argtypes = [P(ft_linear_t), vp, i64, vp, ctypes.c_int, vp, vp, sz, vp]
    L.fourtune_linear_bwd.argtypes = [P(ft_linear_t), vp, vp, vp, i64, vp, ctypes.c_int, vp, vp, ctypes.c_int,
                                      vp, sz, vp]
    L.fourtune_linear_fwd_timed.argtypes = list(L.fourtune_linear_fwd.argtypes) + [P(vp), ctypes.c_int]
    L.fourtune_linear_bwd_timed.argtypes = list(L.fourtune_linear_bwd.argtypes) + [P(vp), ctypes.c_int]
    L.fourtune_linear_fwd_ws_offsets.argtypes = [P(ft_linear_t), i64, P(sz), P(sz)]
    L.fourtune_linear_bwd_ws_offsets.argtypes = [P(ft_linear_t), i64, P(sz), P(sz), P(sz)]
    L.fourtune_quant_down_static.argtypes = [vp, i64, i64, vp, i64, vp, vp, vp, vp]
    L.fourtune_quant_down_static_status.argtypes = [vp]
    L.fourtune_test_wait_timeout.argtypes = [vp, i64, i64, vp, i64, vp, vp, vp, vp, sz, i64, vp]
    L.fourtune_device_status.argtypes = [vp, vp]
    L.fourtune_error_string.argtypes = [ctypes.c_int]
    L.fourtune_error_string.restype = ctypes.c_char_p
    PL = P(ft_linear_t)
    L.fourtune_mlp_fwd_workspace_size.argtypes = [PL, PL, i64]
    L.fourtune_mlp_fwd_workspace_size.restype = sz
    L.fourtune_mlp_bwd_workspace_size.argtypes = [PL, PL, i64]
    L.fourtune_mlp_bwd_workspace_size.restype = sz
    L.fourtune_mlp_fwd.argtypes = [PL, PL, vp, i64, vp, ctypes.c_int, vp, vp, vp, vp, vp, sz, vp]
    L.fourtune_mlp_bwd.argtypes = [PL, PL, vp, vp, vp, vp, vp, i64, vp, ctypes.c_int, vp, vp, vp, vp,
                                   ctypes.c_int, vp, sz, vp]
    L.fourtune_mlp_fwd_timed.argtypes = list(L.fourtune_mlp_fwd.argtypes) + [P(vp), ctypes.c_int]
    L.fourtune_mlp_bwd_timed.argtypes = list(L.fourtune_mlp_bwd.argtypes) + [P(vp), ctypes.c_int]
    L.fourtune_mlp_fwd_ws_offsets.argtypes = [PL, PL, i64, P(sz), P(sz)]
    L.fourtune_mlp_bwd_ws_offsets.argtypes = [PL, PL, i64, P(sz), P(sz), P(sz), P(sz)]
    L.fourtune_dequantize_block16.argtypes = [vp, vp, i64, i64, ctypes.c_int, vp, vp]
    L.fourtune_stabilizer_residual.argtypes = [vp, i64, i64, vp, vp, i64, vp, vp]
    L.fourtune_gemm_block16.argtypes = [vp, vp, vp, vp, i64, i64, i64, vp, vp, ctypes.c_int, vp, sz, vp]
    L.fourtune_linear_fwd_a16.argtypes = [P(ft_linear_t), vp, vp, i64, vp, ctypes.c_int, vp, vp, sz, vp]
    L.fourtune_linear_bwd_g16.argtypes = [P(ft_linear_t), vp, vp, vp, vp, i64, vp, ctypes.c_int, vp, vp, ctypes.c_int,
                                          vp, sz, vp]
    L.fourtune_linear_fwd_a16_workspace_size.argtypes = [P(ft_linear_t), i64]
    L.fourtune_linear_bwd_g16_workspace_size.argtypes = [P(ft_linear_t), i64]
    P16 = P(ft_linear_1x16_t)
    L.fourtune_quantize_1x16.argtypes = [vp, i64, i64, ctypes.c_int, vp, vp, vp, vp, vp]
    L.fourtune_linear_fwd_1x16_workspace_size.argtypes = [P16, i64]
    L.fourtune_linear_bwd_1x16_workspace_size.argtypes = [P16, i64]
    L.fourtune_linear_fwd_1x16.argtypes = [P16, vp, i64, vp, ctypes.c_int, vp, vp, sz, vp]
    L.fourtune_linear_bwd_1x16.argtypes = [P16, vp, vp, vp, i64, vp, ctypes.c_int, vp, vp, ctypes.c_int, vp, sz, vp]
    L.fourtune_linear_fwd_1x16_timed.argtypes = list(L.fourtune_linear_fwd_1x16.argtypes) + [P(vp), ctypes.c_int]
    L.fourtune_linear_bwd_1x16_timed.argtypes = list(L.fourtune_linear_bwd_1x16.argtypes) + [P(vp), ctypes.c_int]
    L.fourtune_linear_1x16_ws_offsets.argtypes = [P16, i64, ctypes.c_int, P(sz), P(sz), P(sz), P(sz)]
    for f in SIZE_FUNCS:
        getattr(L, f).restype = sz
    for f in EXPORTED:
        if f not in SIZE_FUNCS and f != "fourtune_error_string":
            getattr(L, f).restype = ctypes.c_int
    _lib = L
    return L


def _check(code, where):
    if code != 0:
        raise FourtuneError(code, where)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _need(t, dtype, name):
    if t is None:
        return
    if not t.is_cuda or t.dtype != dtype or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous CUDA {dtype} tensor")


def _shape(t, shape, name):
    """Raise ValueError unless tensor t (if given) has exactly `shape`."""
    if t is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def _out_dtype(t, name):
    if t is not None and t.dtype not in (torch.float32, torch.bfloat16):
        raise ValueError(f"{name} must be float32 or bfloat16, got {t.dtype}")


def _ndim2(t, name):
    if t.dim() != 2:
        raise ValueError(f"{name} must be a 2-D tensor, got {t.dim()} dimensions")


def _same_device(*named):
    """All given tensors on one device (None entries skipped)."""
    devs = {(n, t.device) for n, t in named if t is not None}
    if len({d for _, d in devs}) > 1:
        raise ValueError("tensors on different devices: " + ", ".join(f"{n}:{d}" for n, d in sorted(devs, key=str)))


def quantize_block16(x, transposed=False):
    """x: bf16 [rows, cols] -> (codes u8 [rows, cols/2], scales u8 [rows/16, cols/16], codes_t or None)."""
    _need(x, torch.bfloat16, "x")
    rows, cols = x.shape
    codes = torch.empty((rows, cols // 2), dtype=torch.uint8, device=x.device)
    scales = torch.empty((rows // 16, cols // 16), dtype=torch.uint8, device=x.device)
    codes_t = torch.empty((cols, rows // 2), dtype=torch.uint8, device=x.device) if transposed else None
    _check(load().fourtune_quantize_block16(_ptr(x), rows, cols, x.stride(0), _ptr(codes), _ptr(scales),
                                            _ptr(codes_t), _stream()), "fourtune_quantize_block16")
    return codes, scales, codes_t


def quantize_block16_f32(x):
    """x: float32 [rows, cols] -> (codes u8 [rows, cols/2], scales u8 [rows/16, cols/16])."""
    _need(x, torch.float32, "x")
    rows, cols = x.shape
    codes = torch.empty((rows, cols // 2), dtype=torch.uint8, device=x.device)
    scales = torch.empty((rows // 16, cols // 16), dtype=torch.uint8, device=x.device)
    _check(load().fourtune_quantize_block16_f32(_ptr(x), rows, cols, x.stride(0), _ptr(codes), _ptr(scales),
                                                _stream()), "fourtune_quantize_block16_f32")
    return codes, scales


def mma_scales(scales, rows, cols, transposed=False):
    """Block16 scales of an operand [rows, cols] rearranged for the block-scaled MMA (u8 tensor).
    transposed: the operand is the transpose of the matrix whose scales are given
    ([cols/16, rows/16]); otherwise scales is [rows/16, cols/16]."""
    _need(scales, torch.uint8, "scales")
    n = load().fourtune_mma_scales_size(rows, cols)
    if n == 0:
        raise FourtuneError(-2, "fourtune_mma_scales_size")
    out = torch.empty(n, dtype=torch.uint8, device=scales.device)
    _check(load().fourtune_mma_scales(_ptr(scales), rows, cols, int(transposed), _ptr(out), _stream()),
           "fourtune_mma_scales")
    return out


def transpose_codes(codes, rows, cols):
    out = torch.empty((cols, rows // 2), dtype=torch.uint8, device=codes.device)
    _check(load().fourtune_transpose_codes(_ptr(codes), rows, cols, _ptr(out), _stream()),
           "fourtune_transpose_codes")
    return out


class Linear:
    """Device tensors of one triple-branch layer: frozen R codes/scales/codes_t and bias,
    D = [S_dn | A] [K, r_s + r] and U = [S_up ; B] [r_s + r, N] (bf16), and R's scales
    in the MMA-ready layouts of R and R^T (prepared here once).  The LoRA factors
    are views: A = D[:, r_s:], B = U[r_s:, :].  Holds references so pointers stay valid."""

    def __init__(self, R_codes, R_scales, R_codes_t, D, U, r_s, bias=None):
        N, half_k = R_codes.shape
        self.K, self.N = half_k * 2, N
        self.r_s = r_s
        self.r = D.shape[1] - r_s
        for t, n in ((R_codes, "R_codes"), (R_scales, "R_scales"), (R_codes_t, "R_codes_t")):
            _need(t, torch.uint8, n)
        for t, n in ((D, "D"), (U, "U"), (bias, "bias")):
            _need(t, torch.bfloat16, n)
        R_sf = mma_scales(R_scales, self.N, self.K)
        R_sf_t = mma_scales(R_scales, self.K, self.N, transposed=True)
        self.t = dict(R_codes=R_codes, R_scales=R_scales, R_codes_t=R_codes_t, D=D, U=U, bias=bias,
                      R_sf=R_sf, R_sf_t=R_sf_t)
        self.c = ft_linear_t(self.K, self.N, self.r_s, self.r, *[
            _ptr(self.t[k]) for k in ("R_codes", "R_scales", "R_codes_t", "D", "U", "bias", "R_sf", "R_sf_t")])

    @classmethod
    def from_weights(cls, R, S_dn, S_up, A, B, bias=None):
        """Quantize the frozen residual weight R [N, K] (bf16) on the device and
        concatenate the stabilizer and LoRA factors along the rank."""
        codes, scales, codes_t = quantize_block16(R, transposed=True)
        D = torch.cat([S_dn, A], dim=1).contiguous()
        U = torch.cat([S_up, B], dim=0).contiguous()
        return cls(codes, scales, codes_t, D, U, S_dn.shape[1], bias)

    @property
    def A(self):
        return self.t["D"][:, self.r_s:]

    @property
    def B(self):
        return self.t["U"][self.r_s:, :]

    @property
    def R_all(self):
        return self.r_s + self.r

    def fwd_workspace(self, M):
        n = load().fourtune_linear_fwd_workspace_size(ctypes.byref(self.c), M)
        if n == 0:
            raise FourtuneError(-2, "fourtune_linear_fwd_workspace_size")
        return torch.empty(n, dtype=torch.uint8, device="cuda")

    def bwd_workspace(self, M):
        n = load().fourtune_linear_bwd_workspace_size(ctypes.byref(self.c), M)
        if n == 0:
            raise FourtuneError(-2, "fourtune_linear_bwd_workspace_size")
        return torch.empty(n, dtype=torch.uint8, device="cuda")

    def fwd_ws_offsets(self, M):
        c, s = ctypes.c_size_t(), ctypes.c_size_t()
        _check(load().fourtune_linear_fwd_ws_offsets(ctypes.byref(self.c), M, ctypes.byref(c), ctypes.byref(s)),
               "fourtune_linear_fwd_ws_offsets")
        return c.value, s.value

    def bwd_ws_offsets(self, M):
        c, s, p = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
        _check(load().fourtune_linear_bwd_ws_offsets(ctypes.byref(self.c), M, ctypes.byref(c), ctypes.byref(s),
                                                     ctypes.byref(p)), "fourtune_linear_bwd_ws_offsets")
        return c.value, s.value, p.value


def _events(events):
    """List of torch.cuda.Event (already recorded once, so they exist) -> void*[]."""
    arr = (ctypes.c_void_p * len(events))(*[ctypes.c_void_p(e.cuda_event) for e in events])
    return arr, len(events)


def linear_fwd(layer, X, y_dtype=torch.float32, ws=None, Y=None, L=None, events=None):
    """Y = deq(Q(X) Q(R)^T) + L [S_up ; B] + bias, L = bf16(X [S_dn | A]).  Returns (Y, L, ws).
    `events`: optional 2*len(FWD_KERNELS) torch.cuda.Events recorded around each kernel."""
    _ndim2(X, "X")
    M = X.shape[0]
    _shape(X, (M, layer.K), "X")
    _shape(Y, (M, layer.N), "Y")
    _shape(L, (M, layer.R_all), "L")
    _same_device(("X", X), ("Y", Y), ("L", L), ("ws", ws))
    _out_dtype(Y, "Y")
    _need(X, torch.bfloat16, "X")
    Y = torch.empty((M, layer.N), dtype=y_dtype, device=X.device) if Y is None else Y
    L = torch.empty((M, layer.R_all), dtype=torch.bfloat16, device=X.device) if L is None else L
    ws = layer.fwd_workspace(M) if ws is None else ws
    code = FT_DTYPE_F32 if Y.dtype == torch.float32 else FT_DTYPE_BF16
    args = (ctypes.byref(layer.c), _ptr(X), M, _ptr(Y), code, _ptr(L), _ptr(ws), ws.numel(), _stream())
    if events is None:
        _check(load().fourtune_linear_fwd(*args), "fourtune_linear_fwd")
    else:
        arr, n = _events(events)
        _check(load().fourtune_linear_fwd_timed(*args, arr, n), "fourtune_linear_fwd_timed")
    return Y, L, ws


def linear_bwd(layer, dY, X, L, dx_dtype=torch.float32, dA=None, dB=None, accumulate=False, ws=None, dX=None,
               events=None):
    """dX = deq(Q(dY)) deq(Q(R)) + P [S_dn | A]^T, dA = X^T P_B, dB = L_B^T dY.  Returns (dX, dA, dB, ws)."""
    _ndim2(dY, "dY")
    M = dY.shape[0]
    _shape(dY, (M, layer.N), "dY")
    _shape(X, (M, layer.K), "X")
    _shape(L, (M, layer.R_all), "L")
    _shape(dX, (M, layer.K), "dX")
    _shape(dA, (layer.K, layer.r), "dA")
    _shape(dB, (layer.r, layer.N), "dB")
    _same_device(("dY", dY), ("X", X), ("L", L), ("dX", dX), ("dA", dA), ("dB", dB), ("ws", ws))
    _out_dtype(dX, "dX")
    _need(dY, torch.bfloat16, "dY")
    _need(X, torch.bfloat16, "X")
    _need(L, torch.bfloat16, "L")
    dX = torch.empty((M, layer.K), dtype=dx_dtype, device=dY.device) if dX is None else dX
    dA = torch.zeros((layer.K, layer.r), dtype=torch.float32, device=dY.device) if dA is None else dA
    dB = torch.zeros((layer.r, layer.N), dtype=torch.float32, device=dY.device) if dB is None else dB
    ws = layer.bwd_workspace(M) if ws is None else ws
    code = FT_DTYPE_F32 if dX.dtype == torch.float32 else FT_DTYPE_BF16
    args = (ctypes.byref(layer.c), _ptr(dY), _ptr(X), _ptr(L), M, _ptr(dX), code, _ptr(dA), _ptr(dB),
            int(accumulate), _ptr(ws), ws.numel(), _stream())
    if events is None:
        _check(load().fourtune_linear_bwd(*args), "fourtune_linear_bwd")
    else:
        arr, n = _events(events)
        _check(load().fourtune_linear_bwd_timed(*args, arr, n), "fourtune_linear_bwd_timed")
    return dX, dA, dB, ws


class MLP:
    """FC1 -> GELU(tanh) -> FC2, two Linear layers with fc1.N == fc2.K (FourTune §3.3)."""

    def __init__(self, fc1, fc2):
        if fc1.N != fc2.K:
            raise ValueError("fc1.N must equal fc2.K")
        self.fc1, self.fc2 = fc1, fc2
        self.H = fc1.N

    def _ws(self, fn, M):
        n = fn(ctypes.byref(self.fc1.c), ctypes.byref(self.fc2.c), M)
        if n == 0:
            raise FourtuneError(-2, "fourtune_mlp_*_workspace_size")
        return torch.empty(n, dtype=torch.uint8, device="cuda")

    def fwd_workspace(self, M):
        return self._ws(load().fourtune_mlp_fwd_workspace_size, M)

    def bwd_workspace(self, M):
        return self._ws(load().fourtune_mlp_bwd_workspace_size, M)

    def fwd_ws_offsets(self, M):
        c, s = ctypes.c_size_t(), ctypes.c_size_t()
        _check(load().fourtune_mlp_fwd_ws_offsets(ctypes.byref(self.fc1.c), ctypes.byref(self.fc2.c), M,
                                                  ctypes.byref(c), ctypes.byref(s)), "fourtune_mlp_fwd_ws_offsets")
        return c.value, s.value

    def bwd_ws_offsets(self, M):
        o = [ctypes.c_size_t() for _ in range(4)]
        _check(load().fourtune_mlp_bwd_ws_offsets(ctypes.byref(self.fc1.c), ctypes.byref(self.fc2.c), M,
                                                  *[ctypes.byref(x) for x in o]), "fourtune_mlp_bwd_ws_offsets")
        return tuple(x.value for x in o)


def mlp_fwd(mlp, X, y_dtype=torch.float32, ws=None, dbg_a=False, out=None, events=None):
    """Returns (Y, h, L1, L2, ws, a) -- a is the fp32 activation when dbg_a, else None.
    out: optional preallocated (Y, h, L1, L2); events: 2*len(MLP_FWD_KERNELS) torch.cuda.Events."""
    _ndim2(X, "X")
    M = X.shape[0]
    _shape(X, (M, mlp.fc1.K), "X")
    if out is not None:
        for t, shp, n in zip(out, ((M, mlp.fc2.N), (M, mlp.H), (M, mlp.fc1.R_all), (M, mlp.fc2.R_all)),
                             ("Y", "h", "L1", "L2")):
            _shape(t, shp, n)
    _same_device(("X", X), ("ws", ws), *(() if out is None else zip(("Y", "h", "L1", "L2"), out)))
    _need(X, torch.bfloat16, "X")
    dev = X.device
    if out is None:
        Y = torch.empty((M, mlp.fc2.N), dtype=y_dtype, device=dev)
        h = torch.empty((M, mlp.H), dtype=torch.bfloat16, device=dev)
        L1 = torch.empty((M, mlp.fc1.R_all), dtype=torch.bfloat16, device=dev)
        L2 = torch.empty((M, mlp.fc2.R_all), dtype=torch.bfloat16, device=dev)
    else:
        Y, h, L1, L2 = out
    a = torch.empty((M, mlp.H), dtype=torch.float32, device=dev) if dbg_a else None
    ws = mlp.fwd_workspace(M) if ws is None else ws
    code = FT_DTYPE_F32 if Y.dtype == torch.float32 else FT_DTYPE_BF16
    args = (ctypes.byref(mlp.fc1.c), ctypes.byref(mlp.fc2.c), _ptr(X), M, _ptr(Y), code, _ptr(h), _ptr(L1),
            _ptr(L2), _ptr(a), _ptr(ws), ws.numel(), _stream())
    if events is None:
        _check(load().fourtune_mlp_fwd(*args), "fourtune_mlp_fwd")
    else:
        arr, n = _events(events)
        _check(load().fourtune_mlp_fwd_timed(*args, arr, n), "fourtune_mlp_fwd_timed")
    return Y, h, L1, L2, ws, a


def mlp_bwd(mlp, dY, X, h, L1, L2, dx_dtype=torch.float32, accumulate=False, grads=None, ws=None, dX=None,
            events=None):
    """Returns (dX, dA1, dB1, dA2, dB2, ws).  events: 2*len(MLP_BWD_KERNELS) torch.cuda.Events."""
    _ndim2(dY, "dY")
    M = dY.shape[0]
    _shape(dY, (M, mlp.fc2.N), "dY")
    _shape(X, (M, mlp.fc1.K), "X")
    _shape(h, (M, mlp.H), "h")
    _shape(L1, (M, mlp.fc1.R_all), "L1")
    _shape(L2, (M, mlp.fc2.R_all), "L2")
    _shape(dX, (M, mlp.fc1.K), "dX")
    if grads is not None:
        for t, shp, n in zip(grads, ((mlp.fc1.K, mlp.fc1.r), (mlp.fc1.r, mlp.fc1.N), (mlp.fc2.K, mlp.fc2.r),
                                     (mlp.fc2.r, mlp.fc2.N)), ("dA1", "dB1", "dA2", "dB2")):
            _shape(t, shp, n)
    _same_device(("dY", dY), ("X", X), ("h", h), ("L1", L1), ("L2", L2), ("dX", dX), ("ws", ws),
                 *(() if grads is None else zip(("dA1", "dB1", "dA2", "dB2"), grads)))
    _need(dY, torch.bfloat16, "dY")
    for t, n in ((X, "X"), (h, "h"), (L1, "L1"), (L2, "L2")):
        _need(t, torch.bfloat16, n)
    dev = dY.device
    dX = torch.empty((M, mlp.fc1.K), dtype=dx_dtype, device=dev) if dX is None else dX
    if grads is None:
        grads = (torch.zeros((mlp.fc1.K, mlp.fc1.r), dtype=torch.float32, device=dev),
                 torch.zeros((mlp.fc1.r, mlp.fc1.N), dtype=torch.float32, device=dev),
                 torch.zeros((mlp.fc2.K, mlp.fc2.r), dtype=torch.float32, device=dev),
                 torch.zeros((mlp.fc2.r, mlp.fc2.N), dtype=torch.float32, device=dev))
    dA1, dB1, dA2, dB2 = grads
    ws = mlp.bwd_workspace(M) if ws is None else ws
    code = FT_DTYPE_F32 if dX.dtype == torch.float32 else FT_DTYPE_BF16
    args = (ctypes.byref(mlp.fc1.c), ctypes.byref(mlp.fc2.c), _ptr(dY), _ptr(X), _ptr(h), _ptr(L1), _ptr(L2), M,
            _ptr(dX), code, _ptr(dA1), _ptr(dB1), _ptr(dA2), _ptr(dB2), int(accumulate), _ptr(ws), ws.numel(),
            _stream())
    if events is None:
        _check(load().fourtune_mlp_bwd(*args), "fourtune_mlp_bwd")
    else:
        arr, n = _events(events)
        _check(load().fourtune_mlp_bwd_timed(*args, arr, n), "fourtune_mlp_bwd_timed")
    return dX, dA1, dB1, dA2, dB2, ws


def quant_down_static(X, W, codes=None, scales=None, L=None):
    """Allocation-free fused row pass: block16(X) and L = bf16(X W^T), X [M, K], W [R, K] bf16.
    The library keeps this call's scratch in a fixed device array (no workspace);
    overlapping calls race.  Returns (codes, scales, L)."""
    M, K, R = _quant_down_shapes(X, W, codes, scales, L)
    codes = torch.empty((M, K // 2), dtype=torch.uint8, device=X.device) if codes is None else codes
    scales = torch.empty((M // 16, K // 16), dtype=torch.uint8, device=X.device) if scales is None else scales
    L = torch.empty((M, R), dtype=torch.bfloat16, device=X.device) if L is None else L
    _check(load().fourtune_quant_down_static(_ptr(X), M, K, _ptr(W), R, _ptr(codes), _ptr(scales), _ptr(L),
                                             _stream()), "fourtune_quant_down_static")
    return codes, scales, L


def gemm_block16(A_codes, A_sf, B_codes, B_sf, M, N, K, out_dtype=torch.float32, bias=None, out=None, ws=None):
    """out [M, N] = deq(A) deq(B)^T (+ bias); A, B block16 codes, scales in the MMA-ready
    layout (mma_scales).  Returns (out, ws)."""
    for t, n in ((A_codes, "A_codes"), (A_sf, "A_sf"), (B_codes, "B_codes"), (B_sf, "B_sf")):
        _need(t, torch.uint8, n)
    _shape(A_codes, (M, K // 2), "A_codes")
    _shape(B_codes, (N, K // 2), "B_codes")
    _shape(out, (M, N), "out")
    _out_dtype(out, "out")
    out = torch.empty((M, N), dtype=out_dtype, device=A_codes.device) if out is None else out
    ws = torch.empty(256, dtype=torch.uint8, device=A_codes.device) if ws is None else ws
    code = FT_DTYPE_F32 if out.dtype == torch.float32 else FT_DTYPE_BF16
    _check(load().fourtune_gemm_block16(_ptr(A_codes), _ptr(A_sf), _ptr(B_codes), _ptr(B_sf), M, N, K, _ptr(bias),
                                        _ptr(out), code, _ptr(ws), ws.numel(), _stream()), "fourtune_gemm_block16")
    return out, ws


def stabilizer_residual(W, S_dn, S_up):
    """R = bf16(W - (S_dn S_up)^T) for W [N, K], S_dn [K, r_s], S_up [r_s, N] (bf16)."""
    _ndim2(W, "W")
    N, K = W.shape
    r_s = S_dn.shape[1] if S_dn.dim() == 2 else -1
    _shape(S_dn, (K, r_s), "S_dn")
    _shape(S_up, (r_s, N), "S_up")
    _same_device(("W", W), ("S_dn", S_dn), ("S_up", S_up))
    for t, n in ((W, "W"), (S_dn, "S_dn"), (S_up, "S_up")):
        _need(t, torch.bfloat16, n)
    R = torch.empty_like(W)
    _check(load().fourtune_stabilizer_residual(_ptr(W), N, K, _ptr(S_dn), _ptr(S_up), r_s, _ptr(R), _stream()),
           "fourtune_stabilizer_residual")
    return R


def dequantize_block16(codes, scales, rows, cols, transposed=False):
    """bf16 values of a block16 matrix [rows, cols] (exact), or of its transpose [cols, rows]."""
    _need(codes, torch.uint8, "codes")
    _need(scales, torch.uint8, "scales")
    _shape(codes, (rows, cols // 2), "codes")
    _shape(scales, (rows // 16, cols // 16), "scales")
    out = torch.empty((cols, rows) if transposed else (rows, cols), dtype=torch.bfloat16, device=codes.device)
    _check(load().fourtune_dequantize_block16(_ptr(codes), _ptr(scales), rows, cols, int(transposed), _ptr(out),
                                              _stream()), "fourtune_dequantize_block16")
    return out


class Linear16:
    """The 16-bit precision variants' view of a layer (§4.3, Table 4): the low-rank
    factors D = [S_dn | A], U = [S_up ; B] (bf16), an optional bias, and the weight
    as bf16 -- W16 [N, K] and its transpose W16_t [K, N].  From a 4-bit Linear,
    W16 = deq(Q(R)) (from_linear); from a bf16 weight and r_s = 0 it is the
    standard bf16 LoRA layer (from_bf16_lora)."""

    def __init__(self, W16, W16_t, D, U, r_s, bias=None):
        self.N, self.K = W16.shape
        self.r_s, self.r = r_s, D.shape[1] - r_s
        for t, n in ((W16, "W16"), (W16_t, "W16_t"), (D, "D"), (U, "U"), (bias, "bias")):
            _need(t, torch.bfloat16, n)
        _shape(W16_t, (self.K, self.N), "W16_t")
        _shape(D, (self.K, self.r_s + self.r), "D")
        _shape(U, (self.r_s + self.r, self.N), "U")
        self.t = dict(W16=W16, W16_t=W16_t, D=D, U=U, bias=bias)
        self.c = ft_linear_t(self.K, self.N, self.r_s, self.r, None, None, None, _ptr(D), _ptr(U), _ptr(bias),
                             None, None)

    @classmethod
    def from_linear(cls, lay):
        """W16 = deq(Q(R)) of a 4-bit layer, same low-rank factors and bias."""
        W = dequantize_block16(lay.t["R_codes"], lay.t["R_scales"], lay.N, lay.K)
        Wt = dequantize_block16(lay.t["R_codes"], lay.t["R_scales"], lay.N, lay.K, transposed=True)
        return cls(W, Wt, lay.t["D"], lay.t["U"], lay.r_s, lay.t["bias"])

    @classmethod
    def from_bf16_lora(cls, W, A, B, bias=None):
        """Standard LoRA: bf16 weight W [N, K], adapter A [K, r], B [r, N], no stabilizer."""
        return cls(W.contiguous(), W.t().contiguous(), A.contiguous(), B.contiguous(), 0, bias)

    @property
    def R_all(self):
        return self.r_s + self.r

    def _ws(self, fn, M):
        n = fn(ctypes.byref(self.c), M)
        if n == 0:
            raise FourtuneError(-2, "fourtune_linear_*16_workspace_size")
        return torch.empty(n, dtype=torch.uint8, device="cuda")

    def fwd_workspace(self, M):
        return self._ws(load().fourtune_linear_fwd_a16_workspace_size, M)

    def bwd_workspace(self, M):
        return self._ws(load().fourtune_linear_bwd_g16_workspace_size, M)


def linear_fwd_a16(layer16, X, y_dtype=torch.float32, ws=None, Y=None, L=None):
    """16-bit-activation forward: Y = X W16^T + L U + bias, L = bf16(X D).  Returns (Y, L, ws)."""
    _ndim2(X, "X")
    M = X.shape[0]
    _shape(X, (M, layer16.K), "X")
    _shape(Y, (M, layer16.N), "Y")
    _shape(L, (M, layer16.R_all), "L")
    _out_dtype(Y, "Y")
    _need(X, torch.bfloat16, "X")
    Y = torch.empty((M, layer16.N), dtype=y_dtype, device=X.device) if Y is None else Y
    L = torch.empty((M, layer16.R_all), dtype=torch.bfloat16, device=X.device) if L is None else L
    ws = layer16.fwd_workspace(M) if ws is None else ws
    code = FT_DTYPE_F32 if Y.dtype == torch.float32 else FT_DTYPE_BF16
    _check(load().fourtune_linear_fwd_a16(ctypes.byref(layer16.c), _ptr(layer16.t["W16"]), _ptr(X), M, _ptr(Y), code,
                                          _ptr(L), _ptr(ws), ws.numel(), _stream()), "fourtune_linear_fwd_a16")
    return Y, L, ws


def linear_bwd_g16(layer16, dY, X, L, dx_dtype=torch.float32, dA=None, dB=None, accumulate=False, ws=None, dX=None):
    """16-bit-gradient backward: dX = dY W16 + P D^T, dA = X^T P_B, dB = L_B^T dY.  Returns (dX, dA, dB, ws)."""
    _ndim2(dY, "dY")
    M = dY.shape[0]
    _shape(dY, (M, layer16.N), "dY")
    _shape(X, (M, layer16.K), "X")
    _shape(L, (M, layer16.R_all), "L")
    _shape(dX, (M, layer16.K), "dX")
    _shape(dA, (layer16.K, layer16.r), "dA")
    _shape(dB, (layer16.r, layer16.N), "dB")
    _out_dtype(dX, "dX")
    for t, n in ((dY, "dY"), (X, "X"), (L, "L")):
        _need(t, torch.bfloat16, n)
    dev = dY.device
    dX = torch.empty((M, layer16.K), dtype=dx_dtype, device=dev) if dX is None else dX
    dA = torch.zeros((layer16.K, layer16.r), dtype=torch.float32, device=dev) if dA is None else dA
    dB = torch.zeros((layer16.r, layer16.N), dtype=torch.float32, device=dev) if dB is None else dB
    ws = layer16.bwd_workspace(M) if ws is None else ws
    code = FT_DTYPE_F32 if dX.dtype == torch.float32 else FT_DTYPE_BF16
    _check(load().fourtune_linear_bwd_g16(ctypes.byref(layer16.c), _ptr(layer16.t["W16_t"]), _ptr(dY), _ptr(X),
                                          _ptr(L), M, _ptr(dX), code, _ptr(dA), _ptr(dB), int(accumulate), _ptr(ws),
                                          ws.numel(), _stream()), "fourtune_linear_bwd_g16")
    return dX, dA, dB, ws


def _quant_down_shapes(X, W, codes, scales, L):
    """Shape, device and dtype checks of the fused row pass's arguments; returns (M, K, R)."""
    _ndim2(X, "X")
    _ndim2(W, "W")
    M, K = X.shape
    R = W.shape[0]
    _shape(W, (R, K), "W")
    _shape(codes, (M, K // 2), "codes")
    _shape(scales, (M // 16, K // 16), "scales")
    _shape(L, (M, R), "L")
    _same_device(("X", X), ("W", W), ("codes", codes), ("scales", scales), ("L", L))
    _need(X, torch.bfloat16, "X")
    _need(W, torch.bfloat16, "W")
    return M, K, R


def quant_down_static_status():
    """Synchronize and raise FourtuneError(FT_ERR_TIMEOUT) if a kernel wait of the last
    quant_down_static call on this device expired."""
    _check(load().fourtune_quant_down_static_status(_stream()), "fourtune_quant_down_static_status")


def fault_wait_timeout(X, W, ws, wait_ns=5_000_000):
    """Failure-path test hook: the fused row pass with one CTA's first stage left
    unloaded and every wait limited to wait_ns.  Returns (codes, scales, L); the
    expired wait is then reported by device_status(ws)."""
    M, K, R = _quant_down_shapes(X, W, None, None, None)
    _need(ws, torch.uint8, "ws")
    codes = torch.empty((M, K // 2), dtype=torch.uint8, device=X.device)
    scales = torch.empty((M // 16, K // 16), dtype=torch.uint8, device=X.device)
    L = torch.empty((M, R), dtype=torch.bfloat16, device=X.device)
    _check(load().fourtune_test_wait_timeout(_ptr(X), M, K, _ptr(W), R, _ptr(codes), _ptr(scales), _ptr(L),
                                             _ptr(ws), ws.numel(), int(wait_ns), _stream()),
           "fourtune_test_wait_timeout")
    return codes, scales, L


def device_status(ws):
    """Synchronize and raise FourtuneError(FT_ERR_TIMEOUT) if a kernel wait expired."""
    _check(load().fourtune_device_status(_ptr(ws), _stream()), "fourtune_device_status")


# ------------------------------------------------------- 1x16 group-wise variant
def quantize_1x16(W, transposed=False):
    """Q16(W) (or Q16(W^T)) of a bf16 W [rows, cols]: 1x16 groups along the
    output's rows below the per-tensor scale of max|W|.  Returns (codes
    [orows, ocols/2], scales [orows, ocols/16], sf (MMA-ready), amax word
    (int32 [4]: element 0 holds max|W|'s float32 bits))."""
    _need(W, torch.bfloat16, "W")
    _ndim2(W, "W")
    rows, cols = W.shape
    orows, ocols = (cols, rows) if transposed else (rows, cols)
    codes = torch.empty((orows, ocols // 2), dtype=torch.uint8, device=W.device)
    scales = torch.empty((orows, ocols // 16), dtype=torch.uint8, device=W.device)
    sf = torch.empty(load().fourtune_mma_scales_size(orows, ocols), dtype=torch.uint8, device=W.device)
    amax = torch.empty(4, dtype=torch.int32, device=W.device)
    _check(load().fourtune_quantize_1x16(_ptr(W), rows, cols, int(transposed), _ptr(amax), _ptr(codes), _ptr(scales),
                                          _ptr(sf), _stream()), "fourtune_quantize_1x16")
    return codes, scales, sf, amax


class Linear1x16:
    """Device tensors of the 1x16 layer: Q16(R) and Q16(R^T) (codes, MMA-ready
    scales) with the maximum word of R, D = [S_dn | A], U = [S_up ; B] and bias."""

    def __init__(self, R, D, U, r_s, bias=None):
        _need(R, torch.bfloat16, "R")
        for t, n in ((D, "D"), (U, "U"), (bias, "bias")):
            _need(t, torch.bfloat16, n)
        self.N, self.K = R.shape
        self.r_s = r_s
        self.r = D.shape[1] - r_s
        R_codes, R_scales, R_sf, R_amax = quantize_1x16(R)
        Rt_codes, Rt_scales, Rt_sf, _ = quantize_1x16(R, transposed=True)
        self.t = dict(R_codes=R_codes, R_scales=R_scales, R_sf=R_sf, Rt_codes=Rt_codes, Rt_scales=Rt_scales,
                      Rt_sf=Rt_sf, R_amax=R_amax, D=D, U=U, bias=bias)
        self.c = ft_linear_1x16_t(self.K, self.N, self.r_s, self.r, *[
            _ptr(self.t[k]) for k in ("R_codes", "R_sf", "Rt_codes", "Rt_sf", "R_amax", "D", "U", "bias")])

    @classmethod
    def from_weights(cls, R, S_dn, S_up, A, B, bias=None):
        D = torch.cat([S_dn, A], dim=1).contiguous()
        U = torch.cat([S_up, B], dim=0).contiguous()
        return cls(R, D, U, S_dn.shape[1], bias)

    @property
    def R_all(self):
        return self.r_s + self.r

    def _ws(self, fn, M):
        n = getattr(load(), fn)(ctypes.byref(self.c), M)
        if n == 0:
            raise FourtuneError(-2, fn)
        return torch.empty(n, dtype=torch.uint8, device="cuda")

    def fwd_workspace(self, M):
        return self._ws("fourtune_linear_fwd_1x16_workspace_size", M)

    def bwd_workspace(self, M):
        return self._ws("fourtune_linear_bwd_1x16_workspace_size", M)

    def ws_offsets(self, M, backward):
        """(codes, scales, maximum word, P) offsets in the forward (backward=False:
        P is 0) or backward workspace."""
        c, s, a, p = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
        _check(load().fourtune_linear_1x16_ws_offsets(ctypes.byref(self.c), M, int(backward), ctypes.byref(c),
                                                      ctypes.byref(s), ctypes.byref(a), ctypes.byref(p)),
               "fourtune_linear_1x16_ws_offsets")
        return c.value, s.value, a.value, p.value


def linear_fwd_1x16(layer, X, y_dtype=torch.float32, ws=None, Y=None, L=None, events=None):
    """The 1x16 forward: Y = deq(Q16(X)) deq(Q16(R))^T + L [S_up ; B] + bias.  Returns (Y, L, ws).
    `events`: optional 2*len(FWD_1X16_KERNELS) torch.cuda.Events."""
    _ndim2(X, "X")
    M = X.shape[0]
    _shape(X, (M, layer.K), "X")
    _shape(Y, (M, layer.N), "Y")
    _shape(L, (M, layer.R_all), "L")
    _same_device(("X", X), ("Y", Y), ("L", L), ("ws", ws))
    _out_dtype(Y, "Y")
    _need(X, torch.bfloat16, "X")
    Y = torch.empty((M, layer.N), dtype=y_dtype, device=X.device) if Y is None else Y
    L = torch.empty((M, layer.R_all), dtype=torch.bfloat16, device=X.device) if L is None else L
    ws = layer.fwd_workspace(M) if ws is None else ws
    code = FT_DTYPE_F32 if Y.dtype == torch.float32 else FT_DTYPE_BF16
    args = (ctypes.byref(layer.c), _ptr(X), M, _ptr(Y), code, _ptr(L), _ptr(ws), ws.numel(), _stream())
    if events is None:
        _check(load().fourtune_linear_fwd_1x16(*args), "fourtune_linear_fwd_1x16")
    else:
        arr, n = _events(events)
        _check(load().fourtune_linear_fwd_1x16_timed(*args, arr, n), "fourtune_linear_fwd_1x16_timed")
    return Y, L, ws


def linear_bwd_1x16(layer, dY, X, L, dx_dtype=torch.float32, dA=None, dB=None, accumulate=False, ws=None, dX=None,
                    events=None):
    """The 1x16 backward: dX = deq(Q16(dY)) deq(Q16(R^T))^T + P [S_dn | A]^T, dA, dB as linear_bwd.
    Returns (dX, dA, dB, ws)."""
    _ndim2(dY, "dY")
    M = dY.shape[0]
    _shape(dY, (M, layer.N), "dY")
    _shape(X, (M, layer.K), "X")
    _shape(L, (M, layer.R_all), "L")
    _shape(dX, (M, layer.K), "dX")
    _shape(dA, (layer.K, layer.r), "dA")
    _shape(dB, (layer.r, layer.N), "dB")
    _same_device(("dY", dY), ("X", X), ("L", L), ("dX", dX), ("dA", dA), ("dB", dB), ("ws", ws))
    _out_dtype(dX, "dX")
    for t, n in ((dY, "dY"), (X, "X"), (L, "L")):
        _need(t, torch.bfloat16, n)
    dX = torch.empty((M, layer.K), dtype=dx_dtype, device=dY.device) if dX is None else dX
    dA = torch.zeros((layer.K, layer.r), dtype=torch.float32, device=dY.device) if dA is None else dA
    dB = torch.zeros((layer.r, layer.N), dtype=torch.float32, device=dY.device) if dB is None else dB
    ws = layer.bwd_workspace(M) if ws is None else ws
    code = FT_DTYPE_F32 if dX.dtype == torch.float32 else FT_DTYPE_BF16
    args = (ctypes.byref(layer.c), _ptr(dY), _ptr(X), _ptr(L), M, _ptr(dX), code, _ptr(dA), _ptr(dB),
            int(accumulate), _ptr(ws), ws.numel(), _stream())
    if events is None:
        _check(load().fourtune_linear_bwd_1x16(*args), "fourtune_linear_bwd_1x16")
    else:
        arr, n = _events(events)
        _check(load().fourtune_linear_bwd_1x16_timed(*args, arr, n), "fourtune_linear_bwd_1x16_timed")
    return dX, dA, dB, ws
