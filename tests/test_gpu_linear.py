"""flexq_linear_w6a6 / w6a8: a linear layer from FP16 activations.  The GEMM
kernel can quantize the activations itself on 16-token tiles (the route the
library takes for few tokens on short K ranges per CTA; the tests force it at
other sizes too), or the activation quantizer runs first.  Either way the result
must be bit-identical to flexq_quantize_act followed by flexq_gemm_w6a6/w6a8
under the same plan (same codes, same scales, same arithmetic), and within
the GEMM tolerance of the oracle's FP64 linear layer."""

import numpy as np
import pytest
import torch

from bit_group_quantized_flexq_b200 import flexq, inputs
from oracle import flexq_oracle as orc
from tests.gpu_util import assert_within, np16

pytestmark = pytest.mark.gpu

TOL = 1e-3


@pytest.fixture(autouse=True)
def _auto_plan():
    flexq.force_plan(0, 0)
    flexq.force_linear_route(0)
    yield
    flexq.force_plan(0, 0)
    flexq.force_linear_route(0)


@pytest.fixture
def fused():
    """Quantization inside the GEMM wherever the plan's token tile is 16 rows."""
    flexq.force_linear_route(1)


def _layer(M, N, K, seed, std=0.02, frac=0.01, scale=20.0):
    x = inputs.activations(M, K, outlier_frac=frac, outlier_scale=scale, seed=seed)
    w = inputs.weights(N, K, std=std, seed=seed + 17)
    return x, w


def _two_launch(xc, wp, ws, N, gs, bits):
    xq, xs = flexq.quantize_act(xc, gs, bits)
    return flexq.gemm(xq, xs, wp, ws, N, gs, bits)


@pytest.mark.parametrize("bits", [6, 8])
@pytest.mark.parametrize("gs", [32, 64, 128, 256])
@pytest.mark.parametrize("M", [1, 5, 16])
def test_fused_quantization_matches_the_two_launch_path_bitwise(M, gs, bits, fused):
    N, K = 384, 2048
    x, w = _layer(M, N, K, seed=M * 100 + gs + bits)
    xc = x.cuda()
    wp, ws = flexq.quantize_weight(w.cuda(), gs)
    assert flexq.plan(M, N, K, gs)[0] == 16               # the fused route
    y = flexq.linear(xc, wp, ws, N, gs, bits)
    ref = _two_launch(xc, wp, ws, N, gs, bits)
    assert torch.equal(y, ref)
    assert_within(np16(y), orc.linear_layer(x.numpy(), w.numpy(), gs, bits)["y64"], TOL)


@pytest.mark.parametrize("S", [1, 2, 5, 8])
def test_fused_quantization_under_every_k_split(S, fused):
    M, N, K, gs, bits = 11, 256, 4096, 128, 6
    x, w = _layer(M, N, K, seed=300 + S)
    xc = x.cuda()
    wp, ws = flexq.quantize_weight(w.cuda(), gs)
    flexq.force_plan(16, S)
    y = flexq.linear(xc, wp, ws, N, gs, bits)
    ref = _two_launch(xc, wp, ws, N, gs, bits)
    assert torch.equal(y, ref)
    assert_within(np16(y), orc.linear_layer(x.numpy(), w.numpy(), gs, bits)["y64"], TOL)


@pytest.mark.parametrize("M", [17, 40, 100])
def test_fused_quantization_over_several_token_tiles(M, fused):
    # forced 16-token tiles for M > 16: every token tile quantizes its own rows
    N, K, gs, bits = 256, 1024, 64, 8
    x, w = _layer(M, N, K, seed=400 + M)
    xc = x.cuda()
    wp, ws = flexq.quantize_weight(w.cuda(), gs)
    flexq.force_plan(16, 2)
    y = flexq.linear(xc, wp, ws, N, gs, bits)
    ref = _two_launch(xc, wp, ws, N, gs, bits)
    assert torch.equal(y, ref)
    assert_within(np16(y), orc.linear_layer(x.numpy(), w.numpy(), gs, bits)["y64"], TOL)


@pytest.mark.parametrize("M", [3, 17, 64, 200])
def test_wide_plans_quantize_into_the_workspace(M):
    flexq.force_linear_route(2)
    N, K, gs, bits = 384, 2048, 128, 6
    x, w = _layer(M, N, K, seed=500 + M)
    xc = x.cuda()
    wp, ws = flexq.quantize_weight(w.cuda(), gs)
    assert flexq.linear_launches(M, N, K, gs) == 2
    need = flexq.linear_workspace_bytes(M, N, K, gs)
    assert need >= M * K                                   # holds the int8 codes
    buf = torch.zeros(need, dtype=torch.uint8, device="cuda")
    y = flexq.linear(xc, wp, ws, N, gs, bits, workspace_buf=buf)
    assert int(buf[:4096].count_nonzero()) == 0            # arrival counters untouched / reset
    ref = _two_launch(xc, wp, ws, N, gs, bits)
    assert torch.equal(y, ref)
    assert_within(np16(y), orc.linear_layer(x.numpy(), w.numpy(), gs, bits)["y64"], TOL)


def test_wide_plan_without_workspace_is_rejected():
    M, N, K, gs = 40, 256, 512, 128
    x, w = _layer(M, N, K, seed=600)
    wp, ws = flexq.quantize_weight(w.cuda(), gs)
    with pytest.raises(flexq.FlexQError) as ei:
        flexq.linear(x.cuda(), wp, ws, N, gs, 6,
                     workspace_buf=torch.empty(0, dtype=torch.uint8, device="cuda"))
    assert ei.value.status == flexq.FLEXQ_ERR_INVALID_ARG


def test_fused_route_without_workspace_runs_without_a_k_split(fused):
    M, N, K, gs, bits = 4, 256, 2048, 64, 8
    x, w = _layer(M, N, K, seed=601)
    xc = x.cuda()
    wp, ws = flexq.quantize_weight(w.cuda(), gs)
    assert flexq.plan(M, N, K, gs)[1] > 1
    empty = torch.empty(0, dtype=torch.uint8, device="cuda")
    y = flexq.linear(xc, wp, ws, N, gs, bits, workspace_buf=empty)
    xq, xs = flexq.quantize_act(xc, gs, bits)
    ref = flexq.gemm(xq, xs, wp, ws, N, gs, bits, workspace_buf=empty)
    assert torch.equal(y, ref)


def test_fused_quantization_ties_zero_groups_and_extremes(fused):
    # rows with exact half-integer quotients (round half to even), an all-zero
    # row (zero scale, zero codes), FP16 extremes and subnormals
    M, N, K, gs = 6, 128, 512, 32
    x = np.zeros((M, K), dtype=np.float16)
    k = np.arange(K)
    x[0] = ((k % 63) - 31).astype(np.float16)              # s = 1: integer codes
    x[0, 0::gs] = 31.0                                      # every group's absmax = 31
    x[1] = ((k % 62) - 30.5).astype(np.float16)            # ties at s = 1 ...
    x[1, 0::gs] = 31.0
    x[2] = 0.0                                              # zero scale
    x[3] = np.where(k % 2 == 0, 65504.0, -65504.0).astype(np.float16)
    x[4] = np.float16(2.0 ** -24) * ((k % 5) - 2)          # subnormal values
    x[5] = np.linspace(-3.0, 3.0, K).astype(np.float16)
    w = inputs.weights(N, K, seed=602)
    xc = torch.from_numpy(x).cuda()
    wp, ws = flexq.quantize_weight(w.cuda(), gs)
    for bits in (6, 8):
        y = flexq.linear(xc, wp, ws, N, gs, bits)
        ref = _two_launch(xc, wp, ws, N, gs, bits)
        assert torch.equal(y, ref)
        qa, sa = orc.quantize_act(x, gs, bits)
        xq, xs = flexq.quantize_act(xc, gs, bits)
        assert np.array_equal(np16(xq), qa)                # the shared code rule


def test_empty_batch_is_a_noop():
    N, K, gs = 256, 256, 128
    w = inputs.weights(N, K, seed=603)
    wp, ws = flexq.quantize_weight(w.cuda(), gs)
    y = flexq.linear(torch.empty(0, K, dtype=torch.float16, device="cuda"), wp, ws, N, gs)
    assert y.shape == (0, N)


DECODE = [
    # (M, N, K, gs, bits): LLaMA-2-7B decode shapes and a 70B MLP shape
    (1, 4096, 4096, 128, 6),
    (16, 11008, 4096, 128, 6),
    (8, 4096, 11008, 128, 8),
    (1, 8192, 28672, 128, 8),
]


@pytest.mark.parametrize("M,N,K,gs,bits", DECODE)
@pytest.mark.parametrize("route", [0, 1])
def test_decode_shapes_bitwise_and_against_the_oracle(M, N, K, gs, bits, route):
    flexq.force_linear_route(route)
    seed = inputs.layer_seed("fusedq", M, N, K)
    x, w = _layer(M, N, K, seed=seed)
    xc = x.cuda()
    wp, ws = flexq.quantize_weight(w.cuda(), gs)
    y = flexq.linear(xc, wp, ws, N, gs, bits)
    ref = _two_launch(xc, wp, ws, N, gs, bits)
    assert torch.equal(y, ref)
    qw, sw = orc.quantize_weight(w.numpy(), gs)
    qa, sa = orc.quantize_act(x.numpy(), gs, bits)
    assert_within(np16(y), orc.gemm_fp64(qa, sa, qw, sw, gs), TOL)


def test_fused_route_stall_reports_timeout_and_context_survives(fused):
    M, N, K, gs = 16, 256, 1024, 128
    x, w = _layer(M, N, K, seed=604)
    xc = x.cuda()
    wp, ws = flexq.quantize_weight(w.cuda(), gs)
    assert flexq.device_status()[0] == flexq.FLEXQ_OK
    flexq.set_wait_limit_ns(50_000_000)          # 50 ms
    try:
        flexq.inject_stall(True)
        flexq.linear(xc, wp, ws, N, gs, 6)
        status, msg = flexq.device_status()
        assert status == flexq.FLEXQ_ERR_DEVICE_TIMEOUT, msg
    finally:
        flexq.inject_stall(False)
        flexq.set_wait_limit_ns(2_000_000_000)
    y = flexq.linear(xc, wp, ws, N, gs, 6)
    assert torch.equal(y, _two_launch(xc, wp, ws, N, gs, 6))
    assert flexq.device_status()[0] == flexq.FLEXQ_OK


def test_route_by_shape():
    # one launch (quantization inside the GEMM) where (M + 2) * stages <= 28:
    # 4096^2 splits K 8 ways (2 stages per CTA), 1024x8192 8 ways (4
    # stages), 11008x4096 3 ways (6 stages), 28672x8192 not at all (32)
    for M, launches in [(1, 1), (2, 1), (8, 1), (12, 1), (13, 2), (16, 2), (17, 2), (2048, 2)]:
        assert flexq.linear_launches(M, 4096, 4096, 128) == launches, M
    for M, launches in [(1, 1), (5, 1), (6, 2)]:
        assert flexq.linear_launches(M, 1024, 8192, 128) == launches, M
    for M, launches in [(1, 1), (2, 1), (3, 2)]:
        assert flexq.linear_launches(M, 11008, 4096, 128) == launches, M
    assert flexq.linear_launches(1, 28672, 8192, 128) == 2
    flexq.force_linear_route(1)
    assert flexq.linear_launches(16, 4096, 4096, 128) == 1
    assert flexq.linear_launches(17, 4096, 4096, 128) == 2       # 32-token tiles
    flexq.force_linear_route(2)
    assert flexq.linear_launches(1, 4096, 4096, 128) == 2
