"""The "4+2" bit-plane weight form on the GPU: packed bytes bit-exact against
the oracle's restatement, and the GEMM on 4+2 weights bit-identical to the
GEMM on the byte-aligned form of the same codes (only the unpack differs)
and within tolerance of the oracle, for every tile width, the in-kernel
quantization route, group sizes and adversarial codes (-32, 31)."""

import numpy as np
import pytest
import torch

from bit_group_quantized_flexq_b200 import flexq, inputs
from oracle import flexq_oracle as orc
from tests.gpu_util import assert_within, np16

pytestmark = pytest.mark.gpu
TOL = 1e-3
L42 = flexq.LAYOUT_4_2


@pytest.mark.parametrize("N,K,gs", [(128, 256, 32), (256, 512, 128), (384, 1024, 64),
                                    (1024, 4096, 256)])
def test_pack42_bytes_and_scales_match_the_oracle(N, K, gs):
    w = inputs.weights(N, K, std=0.02, seed=inputs.layer_seed("p42", N, K))
    wp, ws = flexq.quantize_weight(w.cuda(), gs, layout=L42)
    qw, sw = orc.quantize_weight(w.numpy(), gs)
    assert np.array_equal(np16(wp), orc.pack_device_form42(qw))
    assert np.array_equal(np16(ws).view(np.uint16), np.ascontiguousarray(sw.T).view(np.uint16))
    # the two layouts hold the same codes
    wp0, _ = flexq.quantize_weight(w.cuda(), gs)
    assert np.array_equal(orc.unpack_device_form(np16(wp0), N, K),
                          orc.unpack_device_form42(np16(wp), N, K))


@pytest.mark.parametrize("T,S", [(16, 1), (16, 4), (32, 2), (64, 1), (128, 1), (128, 2)])
@pytest.mark.parametrize("gs", [32, 128, 256])
def test_gemm42_equals_the_byte_aligned_gemm_and_the_oracle(T, S, gs):
    M, N, K = 70, 256, 2048
    seed = inputs.layer_seed("g42", T, S, gs)
    rng = np.random.default_rng(seed)
    qw = rng.integers(-32, 32, (N, K)).astype(np.int8)            # every 6-bit code
    qw[0, :] = -32
    qw[1, :] = 31
    qa = rng.integers(-127, 128, (M, K)).astype(np.int8)
    sw = inputs.random_scales((N, K // gs), 0.001, 0.01, seed + 1).numpy()
    sa = inputs.random_scales((M, K // gs), 0.001, 0.1, seed + 2).numpy()
    wp0 = torch.from_numpy(orc.pack_device_form(qw)).cuda()
    wp42 = torch.from_numpy(orc.pack_device_form42(qw)).cuda()
    ws = torch.from_numpy(np.ascontiguousarray(sw.T)).cuda()
    xq = torch.from_numpy(qa).cuda()
    ld = flexq.act_scales_ld(M)
    xs = torch.zeros(K // gs, ld, dtype=torch.float16)
    xs[:, :M] = torch.from_numpy(np.ascontiguousarray(sa.T))
    xs = xs.cuda()
    flexq.force_plan(T, S)
    try:
        y0 = flexq.gemm(xq, xs, wp0, ws, N, gs, 8)
        y42 = flexq.gemm(xq, xs, wp42, ws, N, gs, 8, layout=L42)
    finally:
        flexq.force_plan(0, 0)
    assert torch.equal(y0, y42)
    assert_within(np16(y42), orc.gemm_fp64(qa, sa, qw, sw, gs), TOL)


@pytest.mark.parametrize("M,N,K,bits", [(1, 4096, 4096, 6), (2, 1024, 2048, 8), (16, 8192, 8192, 6),
                                        (1, 8192, 28672, 8), (300, 512, 1024, 6)])
def test_linear42_matches_the_byte_aligned_layer(M, N, K, bits):
    gs = 128
    seed = inputs.layer_seed("l42", M, N, K)
    x = inputs.activations(M, K, outlier_frac=0.005, outlier_scale=50.0, seed=seed)
    w = inputs.weights(N, K, std=0.015, seed=seed + 1)
    wp0, ws = flexq.quantize_weight(w.cuda(), gs)
    wp42, ws42 = flexq.quantize_weight(w.cuda(), gs, layout=L42)
    assert torch.equal(ws, ws42)
    y0 = flexq.linear(x.cuda(), wp0, ws, N, gs, bits)
    y42 = flexq.linear(x.cuda(), wp42, ws, N, gs, bits, layout=L42)
    assert torch.equal(y0, y42)
    rows = sorted({0, M // 2, M - 1})
    qw, sw = orc.quantize_weight(w.numpy(), gs)
    qa, sa = orc.quantize_act(x.numpy()[rows], gs, bits)
    assert_within(np16(y42)[rows], orc.gemm_fp64(qa, sa, qw, sw, gs), TOL)
