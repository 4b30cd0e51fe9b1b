"""The C-ABI library builds, loads and exports every entry point its header
declares; host-side argument checks reject bad calls before anything launches.
No GPU is needed (no call here reaches a kernel)."""
import ctypes
import os
import re

import pytest

from bit_lora_fine_b200 import build, fourtune

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fourtune", "fourtune.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return fourtune.load()


def declared():
    txt = open(HEADER).read()
    return sorted(set(re.findall(r"FT_API\s+[\w\s\*]+?\b(fourtune_\w+)\s*\(", txt)))


def test_header_declares_the_spec_calls():
    names = declared()
    for n in ("fourtune_quantize_block16", "fourtune_linear_fwd", "fourtune_linear_bwd"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    for n in declared():
        assert hasattr(lib, n), n
    assert set(declared()) == set(fourtune.EXPORTED)


def test_error_strings(lib):
    for code in range(0, -8, -1):
        assert lib.fourtune_error_string(code)


def _layer(K=64, N=64, r_s=16, r=16, ptr=256):
    p = ctypes.c_void_p(ptr)
    return fourtune.ft_linear_t(K, N, r_s, r, p, p, p, p, p, None, p, p)


def test_argument_checks_without_device(lib):
    s = None
    # null pointers
    assert lib.fourtune_quantize_block16(None, 16, 16, 16, None, None, None, s) == -1
    # shapes not multiples of 16 / ld too small / ld not a multiple of 8
    p = ctypes.c_void_p(256)
    assert lib.fourtune_quantize_block16(p, 20, 16, 16, p, p, None, s) == -2
    assert lib.fourtune_quantize_block16(p, 16, 32, 16, p, p, None, s) == -2
    assert lib.fourtune_quantize_block16(p, 16, 16, 20, p, p, None, s) == -2
    # misaligned input
    assert lib.fourtune_quantize_block16(ctypes.c_void_p(258), 16, 16, 16, p, p, None, s) == -3
    # layer checks: K not a multiple of 32, rank above the limit, misaligned factor
    L = _layer(K=48)
    assert lib.fourtune_linear_fwd(ctypes.byref(L), p, 16, p, 0, p, p, 1 << 20, s) == -2
    L = _layer(r=80)
    assert lib.fourtune_linear_fwd(ctypes.byref(L), p, 16, p, 0, p, p, 1 << 20, s) == -7
    L = _layer()
    L.D = ctypes.c_void_p(264)
    assert lib.fourtune_linear_fwd(ctypes.byref(L), p, 16, p, 0, p, p, 1 << 20, s) == -3
    # bad dtype code, bad M
    L = _layer()
    assert lib.fourtune_linear_fwd(ctypes.byref(L), p, 16, p, 7, p, p, 1 << 20, s) == -1
    assert lib.fourtune_linear_fwd(ctypes.byref(L), p, 24, p, 0, p, p, 1 << 20, s) == -2
    # backward needs the transposed codes
    L = _layer()
    L.R_codes_t = None
    assert lib.fourtune_linear_bwd(ctypes.byref(L), p, p, p, 16, p, 0, p, p, 0, p, 1 << 20, s) == -1
    assert lib.fourtune_linear_bwd_workspace_size(ctypes.byref(L), 16) == 0
    # ... and R's scales in the transposed MMA-ready layout; the forward needs R_sf
    L = _layer()
    L.R_sf_t = None
    assert lib.fourtune_linear_bwd(ctypes.byref(L), p, p, p, 16, p, 0, p, p, 0, p, 1 << 20, s) == -1
    L = _layer()
    L.R_sf = None
    assert lib.fourtune_linear_fwd(ctypes.byref(L), p, 16, p, 0, p, p, 1 << 20, s) == -1
    # MMA-ready scale layout: size formula, argument checks
    assert lib.fourtune_mma_scales_size(128, 64) == 512
    assert lib.fourtune_mma_scales_size(144, 96) == 2 * 2 * 512
    assert lib.fourtune_mma_scales_size(20, 64) == 0
    assert lib.fourtune_mma_scales(None, 16, 16, 0, p, s) == -1
    assert lib.fourtune_mma_scales(p, 16, 16, 2, p, s) == -1
    assert lib.fourtune_mma_scales(p, 16, 24, 0, p, s) == -2
    assert lib.fourtune_mma_scales(p, 16, 16, 0, ctypes.c_void_p(264), s) == -3
