"""The Python binding refuses mismatched shapes, devices and dtypes before anything
reaches the C ABI (a wrong extent would make a kernel's tensor map span memory the
caller does not own).  CPU only: the checks run before any device work."""
import types

import pytest
import torch

from bit_lora_fine_b200 import fourtune as ft


def _layer(K=64, N=32, r_s=16, r=16):
    return types.SimpleNamespace(K=K, N=N, r_s=r_s, r=r, R_all=r_s + r)


def bf(*shape):
    return torch.zeros(shape, dtype=torch.bfloat16)


def test_linear_fwd_refuses_wrong_input_width():
    with pytest.raises(ValueError, match="X has shape"):
        ft.linear_fwd(_layer(), bf(16, 48))


def test_linear_fwd_refuses_wrong_output_shapes():
    with pytest.raises(ValueError, match="Y has shape"):
        ft.linear_fwd(_layer(), bf(16, 64), Y=torch.zeros(16, 16))
    with pytest.raises(ValueError, match="L has shape"):
        ft.linear_fwd(_layer(), bf(16, 64), L=bf(16, 16))
    with pytest.raises(ValueError, match="float32 or bfloat16"):
        ft.linear_fwd(_layer(), bf(16, 64), Y=torch.zeros(16, 32, dtype=torch.float16))


def test_linear_fwd_refuses_non_2d_input():
    with pytest.raises(ValueError, match="2-D"):
        ft.linear_fwd(_layer(), bf(2, 16, 64))


def test_linear_fwd_on_cpu_tensors_is_refused_not_computed():
    # right shapes, wrong device: still a ValueError (no CPU path exists)
    with pytest.raises(ValueError, match="CUDA"):
        ft.linear_fwd(_layer(), bf(16, 64))


def test_linear_bwd_refuses_mismatches():
    lay = _layer()
    with pytest.raises(ValueError, match="dY has shape"):
        ft.linear_bwd(lay, bf(16, 48), bf(16, 64), bf(16, 32))
    with pytest.raises(ValueError, match="X has shape"):
        ft.linear_bwd(lay, bf(16, 32), bf(16, 48), bf(16, 32))
    with pytest.raises(ValueError, match="L has shape"):
        ft.linear_bwd(lay, bf(16, 32), bf(16, 64), bf(16, 16))
    with pytest.raises(ValueError, match="dA has shape"):
        ft.linear_bwd(lay, bf(16, 32), bf(16, 64), bf(16, 32), dA=torch.zeros(64, 8))
    with pytest.raises(ValueError, match="dB has shape"):
        ft.linear_bwd(lay, bf(16, 32), bf(16, 64), bf(16, 32), dB=torch.zeros(8, 32))


def test_mlp_refuses_mismatches():
    mlp = types.SimpleNamespace(fc1=_layer(K=64, N=128), fc2=_layer(K=128, N=64), H=128)
    with pytest.raises(ValueError, match="X has shape"):
        ft.mlp_fwd(mlp, bf(16, 32))
    with pytest.raises(ValueError, match="h has shape"):
        ft.mlp_bwd(mlp, bf(16, 64), bf(16, 64), bf(16, 64), bf(16, 32), bf(16, 32))


def test_quant_down_refuses_mismatched_projection():
    # W must be [R, K] with the input's K: a narrower W would be read past its end
    with pytest.raises(ValueError, match="W has shape"):
        ft.quant_down_static(bf(16, 64), bf(16, 32))
    with pytest.raises(ValueError, match="L has shape"):
        ft.quant_down_static(bf(16, 64), bf(32, 64), L=bf(16, 16))
