"""Grouped launches (flexq_gemm_group / flexq_linear_group): layers that read
the same activations in one kernel launch, each with its own packed weights.
Every output is checked against the oracle's FP64 result, and against the
single-layer entry points under the same K split (bit-identical: the same
kernel computes each output tile with the same K ranges)."""

import numpy as np
import pytest
import torch

from bit_group_quantized_flexq_b200 import flexq, inputs
from oracle import flexq_oracle as orc
from tests.gpu_util import assert_within, np16

pytestmark = pytest.mark.gpu
TOL = 1e-3


def _layers(Ns, K, gs, seed):
    ws, packed = [], []
    for i, N in enumerate(Ns):
        w = inputs.weights(N, K, std=0.02, seed=seed + 17 * i)
        wp, sc = flexq.quantize_weight(w.cuda(), gs)
        ws.append(w)
        packed.append((wp, sc, N))
    return ws, packed


@pytest.mark.parametrize("M,Ns,K,gs,bits", [
    (1, [1024, 128, 128], 4096, 128, 6),        # q/k/v-like widths, split K
    (3, [512, 256], 2048, 64, 8),               # quantization inside the grouped launch
    (16, [384, 128, 256, 640], 1024, 32, 6),    # four layers
    (40, [256, 512], 2048, 256, 8),             # 32-token tiles, two token tiles
    (64, [256, 256], 1024, 128, 6),
    (130, [256, 384], 1024, 128, 8),            # 128-token tiles: one launch per layer
])
def test_linear_group_matches_the_oracle(M, Ns, K, gs, bits):
    flexq.force_plan(0, 0)
    seed = inputs.layer_seed("group", M, K, len(Ns))
    x = inputs.activations(M, K, seed=seed)
    ws, packed = _layers(Ns, K, gs, seed + 1)
    ys = flexq.linear_group(x.cuda(), packed, gs, bits)
    qa, sa = orc.quantize_act(x.numpy(), gs, bits)
    for w, y in zip(ws, ys):
        qw, sw = orc.quantize_weight(w.numpy(), gs)
        assert_within(np16(y), orc.gemm_fp64(qa, sa, qw, sw, gs), TOL)
    st, msg = flexq.device_status()
    assert st == flexq.FLEXQ_OK, msg


@pytest.mark.parametrize("M,split", [(1, 3), (5, 2), (16, 1), (2, 4)])
def test_gemm_group_equals_single_layer_calls_under_one_split(M, split):
    Ns, K, gs, bits = [768, 256, 128], 2048, 128, 6
    seed = inputs.layer_seed("group-eq", M, split)
    x = inputs.activations(M, K, seed=seed)
    _, packed = _layers(Ns, K, gs, seed + 1)
    xq, xs = flexq.quantize_act(x.cuda(), gs, bits)
    flexq.force_plan(16, split)
    try:
        ys = flexq.gemm_group(xq, xs, packed, gs, bits)
        refs = [flexq.gemm(xq, xs, wp, sc, N, gs, bits) for (wp, sc, N) in packed]
        # the linear route (quantization inside the launch where it applies)
        yl = flexq.linear_group(x.cuda(), packed, gs, bits)
        refl = [flexq.linear(x.cuda(), wp, sc, N, gs, bits) for (wp, sc, N) in packed]
    finally:
        flexq.force_plan(0, 0)
    for y, r in zip(ys, refs):
        assert torch.equal(y, r)
    for y, r in zip(yl, refl):
        assert torch.equal(y, r)


def test_group_without_workspace_runs_unsplit_and_matches():
    Ns, K, gs, M = [512, 128], 4096, 128, 4
    seed = inputs.layer_seed("group-nows", M)
    x = inputs.activations(M, K, seed=seed)
    _, packed = _layers(Ns, K, gs, seed + 1)
    xq, xs = flexq.quantize_act(x.cuda(), gs, 6)
    assert flexq.gemm_group_workspace_bytes(M, K, gs, Ns) > 0
    ys = flexq.gemm_group(xq, xs, packed, gs, 6,
                          workspace_buf=torch.empty(0, dtype=torch.uint8, device="cuda"))
    flexq.force_plan(16, 1)
    try:
        refs = [flexq.gemm(xq, xs, wp, sc, N, gs, 6) for (wp, sc, N) in packed]
    finally:
        flexq.force_plan(0, 0)
    for y, r in zip(ys, refs):
        assert torch.equal(y, r)


def test_group_counters_return_to_zero():
    Ns, K, gs, M = [1024, 1024], 4096, 128, 1
    seed = inputs.layer_seed("group-cnt", M)
    x = inputs.activations(M, K, seed=seed)
    _, packed = _layers(Ns, K, gs, seed + 1)
    need = flexq.linear_group_workspace_bytes(M, K, gs, Ns)
    buf = torch.zeros(need, dtype=torch.uint8, device="cuda")
    y1 = flexq.linear_group(x.cuda(), packed, gs, 6, workspace_buf=buf)
    y1 = [t.clone() for t in y1]
    torch.cuda.synchronize()
    assert int(buf[:4096].view(torch.int32).abs().sum()) == 0
    y2 = flexq.linear_group(x.cuda(), packed, gs, 6, workspace_buf=buf)
    for a, b in zip(y1, y2):
        assert torch.equal(a, b)


def test_group_llama2_70b_qkv_decode_rows():
    # the 70B attention input site: q 8192, k 1024, v 1024 wide, K = 8192
    Ns, K, gs = [8192, 1024, 1024], 8192, 128
    for M in (1, 16):
        seed = inputs.layer_seed("group70", M)
        x = inputs.activations(M, K, outlier_frac=0.005, outlier_scale=50.0, seed=seed)
        ws, packed = _layers(Ns, K, gs, seed + 1)
        ys = flexq.linear_group(x.cuda(), packed, gs, 6)
        rows = [0, M - 1]
        qa, sa = orc.quantize_act(x.numpy()[rows], gs, 6)
        for w, y in zip(ws, ys):
            qw, sw = orc.quantize_weight(w.numpy(), gs)
            assert_within(np16(y)[rows], orc.gemm_fp64(qa, sa, qw, sw, gs), TOL)
