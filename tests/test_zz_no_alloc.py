"""The allocation-free row pass, fourtune_quant_down_static.

Some callers cannot give the library a workspace (hosts that own all device
memory and offer no scratch allocator, runtimes that forbid allocation once
running), so this entry point keeps its scratch in a fixed device array inside
the library.  It must compute exactly what the workspace path computes: the
block16 codes and scales of X and L = bf16(X [S_dn | A]) that
fourtune_linear_fwd produces -- bit for bit, since both choose the same
split-K -- on two calls in a row (the array keeps the previous call's contents,
so the second call checks that the state is reset), and report through its own
status query that no wait expired.  This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest

from bit_lora_fine_b200 import synth
from tests.helpers import check_bf16_dot, random_layer, to_dev_bf16, to_host

pytestmark = pytest.mark.gpu


def _case(name):
    """(layer params, X) of a named workload, or of the small-M, wide-K case whose
    row pass splits K sixteen ways (M = 128, K = 4096, ranks 32 + 32)."""
    if name == "small-m-wide-k":
        p = random_layer(4096, 256, 32, 32, seed=5, M=128)
        return p, p["X"]
    wl = synth.WORKLOADS[name]
    return synth.layer_params(wl.layers[0]), synth.layer_input(wl)


@pytest.mark.parametrize("workload", ["flux-linear-3072", "linear-256x512x512", "small-m-wide-k"])
def test_static_scratch_row_pass_matches_workspace_path(cuda_lib, workload):
    import torch
    ft = cuda_lib
    p, Xh = _case(workload)
    X = to_dev_bf16(Xh)
    dev = {k: to_dev_bf16(p[k]) for k in ("R", "S_dn", "S_up", "A", "B")}
    lay = ft.Linear.from_weights(dev["R"], dev["S_dn"], dev["S_up"], dev["A"], dev["B"])
    M, K, R = X.shape[0], lay.K, lay.R_all

    # reference: the existing workspace path (forward), its L and its Q(X)
    Y, L_ref, ws = ft.linear_fwd(lay, X, torch.float32)
    ft.device_status(ws)
    co, so = lay.fwd_ws_offsets(M)
    codes_ref = ws[co:co + M * K // 2].view(M, K // 2).cpu().numpy()
    scales_ref = ws[so:so + (M // 16) * (K // 16)].view(M // 16, K // 16).cpu().numpy()

    W = torch.cat([dev["S_dn"], dev["A"]], dim=1).t().contiguous()     # [R, K]
    absdot = np.abs(Xh.astype(np.float64)) @ np.abs(to_host(W).T)
    for _ in range(2):
        codes, scales, L = ft.quant_down_static(X, W)
        ft.quant_down_static_status()
        np.testing.assert_array_equal(scales.cpu().numpy(), scales_ref)
        np.testing.assert_array_equal(codes.cpu().numpy(), codes_ref)
        check_bf16_dot(to_host(L), to_host(L_ref), absdot, K)
        assert torch.equal(L, L_ref)                                   # same split-K: same sums


def test_static_scratch_rejects_oversize(cuda_lib):
    """A problem whose split bookkeeping would not fit the fixed array is refused
    before anything is launched (M = 2^30 tokens would need 32 MiB of split counters)."""
    import torch
    lib = cuda_lib.load()
    X = torch.zeros((16, 64), dtype=torch.bfloat16, device="cuda")
    W = torch.zeros((16, 64), dtype=torch.bfloat16, device="cuda")
    out = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    rc = lib.fourtune_quant_down_static(p(X), 1 << 30, 64, p(W), 16, p(out), p(out), p(out), s)
    assert rc == -4   # FT_ERR_WORKSPACE
