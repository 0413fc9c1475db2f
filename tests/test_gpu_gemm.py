"""The tcgen05 group GEMM against the oracle: per-group int32 partials bit for
bit, FP16 outputs within max|dY| / max|Y| <= 1e-3 of the oracle's FP64 Y."""

import numpy as np
import pytest
import torch

from bit_group_quantized_flexq_b200 import flexq, inputs
from oracle import flexq_oracle as orc
from tests.gpu_util import assert_within, np16, upload_codes_as_weights

pytestmark = pytest.mark.gpu

TOL = 1e-3


@pytest.fixture(autouse=True)
def _auto_plan():
    flexq.force_plan(0, 0)
    yield
    flexq.force_plan(0, 0)


def _codes(shape, lo, hi, seed):
    return inputs.random_codes(shape, lo, hi, seed).numpy()


# ------------------------------------------------------------- partials ----
@pytest.mark.parametrize("T", [16, 32, 64, 128])
@pytest.mark.parametrize("gs", [32, 64, 128, 256])
def test_partials_bit_exact_every_tile_width(T, gs):
    M = {16: 13, 32: 29, 64: 61, 128: 200}[T]       # ragged token tails
    N, K = 256, 512
    qa = _codes((M, K), -128, 127, seed=T * 7 + gs)
    qw = _codes((N, K), -32, 31, seed=T * 11 + gs)   # includes -32
    flexq.force_plan(T, 1)
    P = flexq.debug_group_partials(torch.from_numpy(qa).cuda(), upload_codes_as_weights(qw), N, gs)
    assert np.array_equal(np16(P), orc.group_partials(qa, qw, gs))


@pytest.mark.parametrize("M", [1, 2, 15, 17, 127, 129, 255, 257])
def test_partials_bit_exact_ragged_m(M):
    N, K, gs = 384, 1024, 128
    qa = _codes((M, K), -31, 31, seed=M)
    qw = _codes((N, K), -31, 31, seed=M + 1000)
    P = flexq.debug_group_partials(torch.from_numpy(qa).cuda(), upload_codes_as_weights(qw), N, gs)
    assert np.array_equal(np16(P), orc.group_partials(qa, qw, gs))


def test_partials_adversarial_codes():
    N, K, gs = 128, 512, 256
    M = 4
    qa = np.empty((M, K), dtype=np.int8)
    qa[0] = 127
    qa[1] = -128
    qa[2] = np.tile([127, -128], K // 2)
    qa[3] = -127
    qw = np.empty((N, K), dtype=np.int8)
    qw[0::4] = 31
    qw[1::4] = -32
    qw[2::4] = np.tile([31, -32], K // 2)
    qw[3::4] = -31
    P = flexq.debug_group_partials(torch.from_numpy(qa).cuda(), upload_codes_as_weights(qw), N, gs)
    assert np.array_equal(np16(P), orc.group_partials(qa, qw, gs))


# ------------------------------------------------------------ FP16 output --
def _layer(M, N, K, gs, bits, seed, std=0.02, frac=0.01, scale=20.0):
    x = inputs.activations(M, K, outlier_frac=frac, outlier_scale=scale, seed=seed)
    w = inputs.weights(N, K, std=std, seed=seed + 17)
    return x, w


@pytest.mark.parametrize("bits", [6, 8])
@pytest.mark.parametrize("gs", [32, 64, 128, 256])
def test_layer_tiny_config(gs, bits):
    # the tiny W6A6 configuration (and its W6A8 / group-size variants)
    M, N, K = 16, 256, 256
    x, w = _layer(M, N, K, gs, bits, seed=0)
    wp, ws = flexq.quantize_weight(w.cuda(), gs)
    y = flexq.linear(x.cuda(), wp, ws, N, gs, bits)
    ref = orc.linear_layer(x.numpy(), w.numpy(), gs, bits)
    assert_within(np16(y), ref["y64"], TOL)


@pytest.mark.parametrize("T,S", [(16, 1), (16, 2), (16, 3), (16, 8), (32, 1), (32, 6),
                                 (64, 1), (64, 4), (128, 1), (128, 2)])
def test_layer_every_plan(T, S):
    M = {16: 9, 32: 31, 64: 47, 128: 150}[T]
    N, K, gs, bits = 256, 2048, 128, 6
    x, w = _layer(M, N, K, gs, bits, seed=T + S)
    wp, ws = flexq.quantize_weight(w.cuda(), gs)
    flexq.force_plan(T, S)
    y = flexq.linear(x.cuda(), wp, ws, N, gs, bits)
    ref = orc.linear_layer(x.numpy(), w.numpy(), gs, bits)
    assert_within(np16(y), ref["y64"], TOL)


@pytest.mark.parametrize("gs", [32, 256])
def test_layer_split_with_group_sizes(gs):
    M, N, K, bits = 5, 384, 4096, 8
    x, w = _layer(M, N, K, gs, bits, seed=gs)
    wp, ws = flexq.quantize_weight(w.cuda(), gs)
    flexq.force_plan(16, 7)
    y = flexq.linear(x.cuda(), wp, ws, N, gs, bits)
    ref = orc.linear_layer(x.numpy(), w.numpy(), gs, bits)
    assert_within(np16(y), ref["y64"], TOL)


def test_gemm_empty_m_is_noop():
    N, K, gs = 256, 256, 128
    w = inputs.weights(N, K, seed=3)
    wp, ws = flexq.quantize_weight(w.cuda(), gs)
    xq = torch.empty(0, K, dtype=torch.int8, device="cuda")
    xs = torch.empty(K // gs, 0, dtype=torch.float16, device="cuda")
    y = flexq.gemm(xq, xs, wp, ws, N, gs)
    assert y.shape == (0, N)


def test_w6a6_and_w6a8_entry_points_share_the_kernel():
    M, N, K, gs = 33, 256, 512, 64
    x, w = _layer(M, N, K, gs, 8, seed=9)
    wp, ws = flexq.quantize_weight(w.cuda(), gs)
    xq, xs = flexq.quantize_act(x.cuda(), gs, 8)
    y6 = flexq.gemm(xq, xs, wp, ws, N, gs, 6)
    y8 = flexq.gemm(xq, xs, wp, ws, N, gs, 8)
    assert torch.equal(y6, y8)


# ------------------------------------------------- full benchmark shapes ---
FULL = [
    # (M, N, K, gs, bits, weight std, outlier frac, outlier scale)
    (1, 4096, 4096, 128, 6, 0.02, 0.01, 20.0),
    (16, 11008, 4096, 128, 6, 0.02, 0.01, 20.0),
    (256, 4096, 11008, 128, 6, 0.02, 0.01, 20.0),
    (2048, 4096, 4096, 128, 6, 0.02, 0.01, 20.0),
    (64, 13824, 5120, 128, 8, 0.02, 0.01, 20.0),
    (1, 8192, 28672, 128, 8, 0.015, 0.005, 50.0),
    # the LLaMA-2-13B W6A8 layers and the N = K = 8192 group-size sweep
    (4096, 5120, 13824, 128, 8, 0.02, 0.01, 20.0),
    (1, 5120, 5120, 128, 8, 0.02, 0.01, 20.0),
    (8, 8192, 8192, 32, 6, 0.02, 0.01, 20.0),
    (128, 8192, 8192, 64, 8, 0.02, 0.01, 20.0),
    (1024, 8192, 8192, 256, 6, 0.02, 0.01, 20.0),
    (16384, 8192, 8192, 32, 8, 0.02, 0.01, 20.0),
]


@pytest.mark.parametrize("M,N,K,gs,bits,std,frac,scale", FULL)
def test_full_size_sampled_rows(M, N, K, gs, bits, std, frac, scale):
    seed = inputs.layer_seed("full", M, N, K)
    x = inputs.activations(M, K, outlier_frac=frac, outlier_scale=scale, seed=seed)
    w = inputs.weights(N, K, std=std, seed=seed + 1)
    wp, ws = flexq.quantize_weight(w.cuda(), gs)
    y = np16(flexq.linear(x.cuda(), wp, ws, N, gs, bits))
    rows = sorted(set(np.random.default_rng(seed).integers(0, M, 6).tolist()) | {0, M - 1})
    qw, sw = orc.quantize_weight(w.numpy(), gs)
    qa, sa = orc.quantize_act(x.numpy()[rows], gs, bits)
    y64 = orc.gemm_fp64(qa, sa, qw, sw, gs)
    assert_within(y[rows], y64, TOL)


# the LLaMA-2-70B layers of the headline step at every one of its M: one weight
# draw per shape (quantized by the GPU and by the oracle once), sampled rows
_70B = {}


def _70b_layer(N, K):
    if (N, K) not in _70B:
        seed = inputs.layer_seed("full70", N, K)
        w = inputs.weights(N, K, std=0.015, seed=seed)
        wp, ws = flexq.quantize_weight(w.cuda(), 128)
        qw, sw = orc.quantize_weight(w.numpy(), 128)
        _70B.clear()
        _70B[(N, K)] = (wp, ws, qw, sw)
    return _70B[(N, K)]


@pytest.mark.parametrize("M", [1, 16, 512, 8192])
@pytest.mark.parametrize("N,K,bits", [(28672, 8192, 6), (8192, 8192, 6), (8192, 28672, 8)])
def test_llama2_70b_layers_sampled_rows(N, K, bits, M):
    wp, ws, qw, sw = _70b_layer(N, K)
    x = inputs.activations(M, K, outlier_frac=0.005, outlier_scale=50.0,
                           seed=inputs.layer_seed("full70-x", M, N, K))
    y = np16(flexq.linear(x.cuda(), wp, ws, N, 128, bits))
    rows = sorted(set(np.random.default_rng(M + N).integers(0, M, 5).tolist()) | {0, M - 1})
    qa, sa = orc.quantize_act(x.numpy()[rows], 128, bits)
    assert_within(y[rows], orc.gemm_fp64(qa, sa, qw, sw, 128), TOL)


# ------------------------------------------------------ bounded waits ------
def test_stalled_pipeline_reports_timeout_and_context_survives():
    M, N, K, gs = 16, 256, 1024, 128
    x, w = _layer(M, N, K, gs, 6, seed=4)
    wp, ws = flexq.quantize_weight(w.cuda(), gs)
    xq, xs = flexq.quantize_act(x.cuda(), gs, 6)
    assert flexq.device_status()[0] == flexq.FLEXQ_OK
    flexq.set_wait_limit_ns(50_000_000)          # 50 ms
    try:
        flexq.inject_stall(True)
        flexq.gemm(xq, xs, wp, ws, N, gs)
        status, msg = flexq.device_status()
        assert status == flexq.FLEXQ_ERR_DEVICE_TIMEOUT, msg
        assert flexq.device_status()[0] == flexq.FLEXQ_OK     # cleared
    finally:
        flexq.inject_stall(False)
        flexq.set_wait_limit_ns(2_000_000_000)
    y = flexq.gemm(xq, xs, wp, ws, N, gs)
    ref = orc.linear_layer(x.numpy(), w.numpy(), gs, 6)
    assert_within(np16(y), ref["y64"], TOL)
    assert flexq.device_status()[0] == flexq.FLEXQ_OK


# ------------------------------------------------------ split-K workspace --
def test_split_k_is_deterministic_and_leaves_the_workspace_zeroed():
    M, N, K, gs, bits = 7, 384, 4096, 128, 6
    x, w = _layer(M, N, K, gs, bits, seed=21)
    wp, ws = flexq.quantize_weight(w.cuda(), gs)
    xq, xs = flexq.quantize_act(x.cuda(), gs, bits)
    flexq.force_plan(16, 8)
    need = flexq.gemm_workspace_bytes(M, N, K, gs)
    assert need > 0
    buf = torch.zeros(need, dtype=torch.uint8, device="cuda")
    y1 = flexq.gemm(xq, xs, wp, ws, N, gs, bits, workspace_buf=buf).clone()
    assert int(buf.count_nonzero()) > 0                      # partial tiles were written
    counters = buf[:4096]                                    # fixed counter region
    assert int(counters.count_nonzero()) == 0                # every counter reset
    y2 = flexq.gemm(xq, xs, wp, ws, N, gs, bits, workspace_buf=buf)
    assert torch.equal(y1, y2)                               # fixed reduction order
    ref = orc.linear_layer(x.numpy(), w.numpy(), gs, bits)
    assert_within(np16(y1), ref["y64"], TOL)


def test_gemm_without_workspace_runs_without_a_k_split():
    M, N, K, gs, bits = 3, 256, 2048, 64, 8
    x, w = _layer(M, N, K, gs, bits, seed=22)
    wp, ws = flexq.quantize_weight(w.cuda(), gs)
    xq, xs = flexq.quantize_act(x.cuda(), gs, bits)
    assert flexq.plan(M, N, K, gs)[1] > 1
    y = flexq.gemm(xq, xs, wp, ws, N, gs, bits,
                   workspace_buf=torch.empty(0, dtype=torch.uint8, device="cuda"))
    ref = orc.linear_layer(x.numpy(), w.numpy(), gs, bits)
    assert_within(np16(y), ref["y64"], TOL)


def test_too_small_workspace_is_rejected():
    M, N, K, gs = 2, 256, 2048, 128
    x, w = _layer(M, N, K, gs, 6, seed=23)
    wp, ws = flexq.quantize_weight(w.cuda(), gs)
    xq, xs = flexq.quantize_act(x.cuda(), gs, 6)
    need = flexq.gemm_workspace_bytes(M, N, K, gs)
    assert need > 16
    small = torch.zeros(need - 16, dtype=torch.uint8, device="cuda")
    with pytest.raises(flexq.FlexQError) as ei:
        flexq.gemm(xq, xs, wp, ws, N, gs, 6, workspace_buf=small)
    assert ei.value.status == flexq.FLEXQ_ERR_INVALID_ARG


def test_whole_waves_and_split_last_wave():
    # 2 token tiles x 80 weight tiles = 160 output tiles: one whole wave on 148
    # SMs runs unsplit and the 12 tiles of the last wave are split along K
    M, N, K, gs, bits = 200, 10240, 1024, 128, 6
    t, s, c = flexq.plan(M, N, K, gs)
    assert (t, s) == (128, 4) and c == 148 + 4 * 12
    seed = inputs.layer_seed("tail", M, N, K)
    x = inputs.activations(M, K, seed=seed)
    w = inputs.weights(N, K, seed=seed + 1)
    wp, ws = flexq.quantize_weight(w.cuda(), gs)
    y = np16(flexq.linear(x.cuda(), wp, ws, N, gs, bits))
    rows = [0, 1, 127, 128, 150, 199]
    qw, sw = orc.quantize_weight(w.numpy(), gs)
    qa, sa = orc.quantize_act(x.numpy()[rows], gs, bits)
    assert_within(y[rows], orc.gemm_fp64(qa, sa, qw, sw, gs), TOL)
