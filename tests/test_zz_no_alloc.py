"""flexq_gemm_static_scratch: the GEMM for callers that cannot allocate device
memory when they call it (an engine plugin whose enqueue step may not
allocate, a server that hands all device memory to its own pool at start-up).
Its split-K scratch is a fixed array in device memory instead of a caller
workspace.  Checked through the C ABI against flexq_gemm_w6a6/w6a8 on the
same inputs, twice in a row (the second call finds the first call's leftovers
in the shared scratch).  Named to run after every other test file."""

import ctypes

import numpy as np
import pytest
import torch

from bit_group_quantized_flexq_b200 import flexq, inputs
from oracle import flexq_oracle as orc

pytestmark = pytest.mark.gpu

TOL = 1e-3          # max|dY| / max|Y|, as in the other GEMM tests


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


def _call_static(L, xq, xs, wp, ws, y, N, gs, bits):
    M, K = xq.shape
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return L.flexq_gemm_static_scratch(M, N, K, gs, bits, _ptr(xq), _ptr(xs), _ptr(wp), _ptr(ws),
                                       _ptr(y), stream)


@pytest.mark.parametrize("M,N,K,gs,bits", [
    (1, 4096, 4096, 128, 6),        # decode: K split 8 ways through the scratch
    (16, 11008, 4096, 128, 8),      # decode, W6A8
    (200, 384, 1024, 64, 6),        # two token tiles
])
def test_static_scratch_gemm_matches_the_workspace_gemm_on_two_calls(M, N, K, gs, bits):
    flexq.force_plan(0, 0)
    L = flexq.lib()
    seed = inputs.layer_seed("noalloc", M, N, K)
    x = inputs.activations(M, K, seed=seed).cuda()
    w = inputs.weights(N, K, seed=seed + 1).cuda()
    wp, ws = flexq.quantize_weight(w, gs)
    xq, xs = flexq.quantize_act(x, gs, bits)
    ref = flexq.gemm(xq, xs, wp, ws, N, gs, bits)          # caller-workspace entry point
    torch.cuda.synchronize()
    for _ in range(2):
        y = torch.full((M, N), float("nan"), dtype=torch.float16, device="cuda")
        rc = _call_static(L, xq, xs, wp, ws, y, N, gs, bits)
        assert rc == flexq.FLEXQ_OK, L.flexq_last_error_message().decode()
        torch.cuda.synchronize()
        err = orc.rel_err_vs_max(y.cpu().numpy().astype(np.float64),
                                 ref.cpu().numpy().astype(np.float64))
        assert err <= TOL, f"max|dY|/max|Y| = {err:.3e}"
    st, msg = flexq.device_status()
    assert st == flexq.FLEXQ_OK, msg


def test_static_scratch_rejects_plans_beyond_its_size():
    # a forced plan whose split-K partial tiles exceed the 16 MiB scratch:
    # 2 token tiles x 65 weight tiles, split 2, 128 x 128 FP32 tiles = 17 MB
    M, N, K, gs = 200, 8320, 1024, 128
    L = flexq.lib()
    xq = torch.zeros(M, K, dtype=torch.int8, device="cuda")
    xs = torch.zeros(K // gs, flexq.act_scales_ld(M), dtype=torch.float16, device="cuda")
    wp = torch.zeros(flexq.weight_packed_bytes(N, K, gs), dtype=torch.uint8, device="cuda")
    ws = torch.zeros(K // gs, N, dtype=torch.float16, device="cuda")
    y = torch.empty(M, N, dtype=torch.float16, device="cuda")
    flexq.force_plan(128, 2)
    try:
        assert flexq.plan(M, N, K, gs)[1] == 2
        rc = _call_static(L, xq, xs, wp, ws, y, N, gs, 6)
        msg = L.flexq_last_error_message()       # before the next call clears it
    finally:
        flexq.force_plan(0, 0)
    assert rc == flexq.FLEXQ_ERR_UNSUPPORTED
    assert b"static scratch" in msg
