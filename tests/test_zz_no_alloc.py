"""flexq_gemm_static_scratch: the GEMM for callers that cannot allocate device
memory when they call it (an engine plugin whose enqueue step may not
allocate, a server that hands all device memory to its own pool at start-up).
Its split-K scratch is a fixed array in device memory instead of a caller
workspace.  Checked through the C ABI against flexq_gemm_w6a6/w6a8: a run of
calls of different shapes and different inputs, each of which finds the
previous call's partial tiles in the shared scratch, must give exactly the
workspace entry point's output (same plan, same split order), and the run
must not change the device's free memory.  Named to run after every other
test file."""

import ctypes

import pytest
import torch

from bit_group_quantized_flexq_b200 import flexq, inputs

pytestmark = pytest.mark.gpu


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


def _call_static(L, xq, xs, wp, ws, y, N, gs, bits):
    M, K = xq.shape
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return L.flexq_gemm_static_scratch(M, N, K, gs, bits, _ptr(xq), _ptr(xs), _ptr(wp), _ptr(ws),
                                       _ptr(y), stream)


def _case(M, N, K, gs, bits, seed):
    x = inputs.activations(M, K, seed=seed).cuda()
    w = inputs.weights(N, K, seed=seed + 1).cuda()
    wp, ws = flexq.quantize_weight(w, gs)
    xq, xs = flexq.quantize_act(x, gs, bits)
    ref = flexq.gemm(xq, xs, wp, ws, N, gs, bits)          # caller-workspace entry point
    return (xq, xs, wp, ws, N, gs, bits), ref


# every shape is split along K, so each call writes partial tiles and arrival
# counters into the shared scratch; the last case repeats the first shape on
# other inputs, over the partial tiles the calls before it left behind
SEQUENCE = [
    (1, 4096, 4096, 128, 6, 11),      # decode: K split 8 ways through the scratch
    (16, 11008, 4096, 128, 8, 12),    # decode, W6A8, split 3
    (200, 384, 4096, 64, 6, 13),      # two 128-token tiles, split 2
    (1, 4096, 4096, 128, 6, 14),      # the first shape again, new inputs
]


def test_static_scratch_gemm_equals_the_workspace_gemm_across_calls():
    flexq.force_plan(0, 0)
    L = flexq.lib()
    cases = []
    for M, N, K, gs, bits, seed in SEQUENCE:
        assert flexq.plan(M, N, K, gs)[1] > 1
        cases.append(_case(M, N, K, gs, bits, inputs.layer_seed("noalloc", seed)))
    torch.cuda.synchronize()
    # the first call looks up the scratch's address; the free memory is read
    # after it, around the rest of the run
    y = torch.full((1, 4096), float("nan"), dtype=torch.float16, device="cuda")
    args0, _ = cases[0]
    assert _call_static(L, *args0[:4], y, *args0[4:]) == flexq.FLEXQ_OK
    outs = []
    for (args, ref) in cases:
        xq, xs, wp, ws, N, gs, bits = args
        y = torch.full((xq.shape[0], N), float("nan"), dtype=torch.float16, device="cuda")
        outs.append((y, ref))
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for (args, _), (y, _) in zip(cases, outs):
        xq, xs, wp, ws, N, gs, bits = args
        rc = _call_static(L, xq, xs, wp, ws, y, N, gs, bits)
        assert rc == flexq.FLEXQ_OK, L.flexq_last_error_message().decode()
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    for i, (y, ref) in enumerate(outs):
        assert torch.equal(y, ref), f"call {i}: static-scratch output differs from the workspace GEMM"
    assert free1 == free0, f"free device memory changed by {free0 - free1} bytes"
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
