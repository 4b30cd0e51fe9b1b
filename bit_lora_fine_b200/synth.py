"""Seeded synthetic inputs shaped like the DiT workloads FourTune trains.

This module holds only input generation -- none of the layer's arithmetic -- so
that the CUDA path and the CPU oracle can be fed the same tensors.

FourTune's experiments post-train FLUX.1-dev (12B, hidden 3072, LoRA rank 64)
and Qwen-Image DiTs (§4.1, §4.2); no weights or datasets exist here, so every
tensor is drawn from a fixed-seed PCG64 stream in float32 and rounded to
bfloat16 (ties-to-even).  Activations carry outlier channels, the property that
motivates the stabilizer branch (§3.1).

Workloads (M tokens, K in, N out, r_s stabilizer rank, r LoRA rank):
  linear-256x512x512      M=256   K=N=512      r_s=r=16  8 outlier columns x20
  flux-linear-3072        M=4608  K=N=3072     r_s=r=32  1% outlier columns x20
  flux-mlp-3072           M=4608  3072->12288->3072 (GELU tanh) r_s=r=32, biases
  flux-single-stream      M=4608  in 3072->21504, out 15360->3072, r_s=r=64,
                          log-normal per-channel activation scales (sigma 1.5)
  video-mlp-5120          M=32768 5120->13824->5120, r_s=r=64, 2% outliers x30,
                          weights N(0, 0.015)
M = 4608 is 4096 image tokens + 512 text tokens (a 1024^2 FLUX image).
"""
from dataclasses import dataclass, field

import numpy as np

BASE_SEED = 20260707

# fixed per-tensor stream offsets: every tensor has its own generator
_OFFSETS = {
    "X": 1, "dY": 2,
    "R": 10, "S_dn": 11, "S_up": 12, "A": 13, "B": 14, "bias": 15,
    "outlier_cols": 20, "lognormal": 21,
}


def _rng(name: str, layer: int = 0) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64([BASE_SEED, _OFFSETS[name], layer]))


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bfloat16 bit patterns (uint16), round-to-nearest-even."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def bf16_from_bits(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def to_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16, returned as float32 (exact values)."""
    return bf16_from_bits(bf16_bits(x))


def normal(name: str, shape, std: float, layer: int = 0) -> np.ndarray:
    g = _rng(name, layer).standard_normal(size=shape, dtype=np.float32)
    return to_bf16(g * np.float32(std))


def activations(name: str, M: int, K: int, outlier_frac=None, n_outliers=None,
                outlier_scale=20.0, lognormal_sigma=None, layer: int = 0) -> np.ndarray:
    """N(0,1) activations [M, K] with seeded outlier columns or per-channel log-normal scales."""
    z = _rng(name, layer).standard_normal(size=(M, K), dtype=np.float32)
    if lognormal_sigma is not None:
        g = _rng("lognormal", layer).standard_normal(size=K, dtype=np.float32)
        z = z * np.exp(np.float32(lognormal_sigma) * g)[None, :].astype(np.float32)
    else:
        if n_outliers is None:
            n_outliers = int(round((outlier_frac or 0.0) * K))
        if n_outliers:
            cols = _rng("outlier_cols", layer).choice(K, size=n_outliers, replace=False)
            z[:, cols] *= np.float32(outlier_scale)
    return to_bf16(z.astype(np.float32))


@dataclass
class LinearSpec:
    K: int
    N: int
    r_s: int
    r: int
    w_std: float = 0.02
    b_std: float = 1e-3          # LoRA B: "zeros plus N(0, 1e-3)" read as std 1e-3
    bias_std: float = 0.0        # 0 -> no bias


@dataclass
class Workload:
    name: str
    M: int
    kind: str                    # "linear" | "mlp"
    layers: list = field(default_factory=list)   # LinearSpec per layer
    x_outlier_frac: float = 0.0
    x_n_outliers: int = 0
    x_outlier_scale: float = 20.0
    x_lognormal_sigma: float = None


WORKLOADS = {
    "linear-256x512x512": Workload(
        "linear-256x512x512", 256, "linear", [LinearSpec(512, 512, 16, 16)],
        x_n_outliers=8, x_outlier_scale=20.0),
    "flux-linear-3072": Workload(
        "flux-linear-3072", 4608, "linear", [LinearSpec(3072, 3072, 32, 32)],
        x_outlier_frac=0.01, x_outlier_scale=20.0),
    "flux-mlp-3072": Workload(
        "flux-mlp-3072", 4608, "mlp",
        [LinearSpec(3072, 12288, 32, 32, bias_std=0.02), LinearSpec(12288, 3072, 32, 32, bias_std=0.02)],
        x_outlier_frac=0.01, x_outlier_scale=20.0),
    "flux-single-stream": Workload(
        "flux-single-stream", 4608, "linear",
        [LinearSpec(3072, 21504, 64, 64), LinearSpec(15360, 3072, 64, 64)],
        x_lognormal_sigma=1.5),
    "video-mlp-5120": Workload(
        "video-mlp-5120", 32768, "mlp",
        [LinearSpec(5120, 13824, 64, 64, w_std=0.015, bias_std=0.015),
         LinearSpec(13824, 5120, 64, 64, w_std=0.015, bias_std=0.015)],
        x_outlier_frac=0.02, x_outlier_scale=30.0),
}


def layer_params(spec: LinearSpec, layer: int = 0) -> dict:
    """Frozen residual weight R [N, K] (bf16, quantized later), stabilizer S_dn [K, r_s],
    S_up [r_s, N], LoRA A [K, r], B [r, N], optional bias [N] -- all bf16 values."""
    p = dict(
        R=normal("R", (spec.N, spec.K), spec.w_std, layer),
        S_dn=normal("S_dn", (spec.K, spec.r_s), spec.w_std, layer),
        S_up=normal("S_up", (spec.r_s, spec.N), spec.w_std, layer),
        A=normal("A", (spec.K, spec.r), spec.w_std, layer),
        B=normal("B", (spec.r, spec.N), spec.b_std, layer),
        bias=normal("bias", (spec.N,), spec.bias_std, layer) if spec.bias_std > 0 else None,
    )
    return p


def layer_input(wl: Workload, layer: int = 0, M: int = None) -> np.ndarray:
    """Input X of layer `layer` of a linear workload (or the MLP's FC1 input)."""
    M = wl.M if M is None else M
    K = wl.layers[layer].K
    return activations("X", M, K, outlier_frac=wl.x_outlier_frac or None,
                       n_outliers=wl.x_n_outliers or None, outlier_scale=wl.x_outlier_scale,
                       lognormal_sigma=wl.x_lognormal_sigma, layer=layer)


def upstream_grad(wl: Workload, layer: int = 0, M: int = None) -> np.ndarray:
    """dL/dy for layer `layer` (the MLP uses the last layer's), N(0, 1)."""
    M = wl.M if M is None else M
    N = wl.layers[layer].N
    return normal("dY", (M, N), 1.0, layer)
