"""Quantization kernels against the oracle: codes, scales and packed bytes
must match bit for bit."""

import numpy as np
import pytest
import torch

from bit_group_quantized_flexq_b200 import flexq, inputs
from oracle import flexq_oracle as orc
from tests.gpu_util import bits16, np16, oracle_weight_device_form

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("gs", [32, 64, 128, 256])
@pytest.mark.parametrize("bits", [6, 8])
@pytest.mark.parametrize("M,K", [(1, 256), (3, 512), (9, 2304), (16, 8192), (17, 1024), (130, 768)])
def test_act_quant_bit_exact(M, K, gs, bits):
    if K % gs:
        pytest.skip("K must be a multiple of the group size")
    x = inputs.activations(M, K, seed=inputs.layer_seed("act", M, K, gs, bits))
    xq, xs = flexq.quantize_act(x.cuda(), gs, bits)
    qa, sa = orc.quantize_act(x.numpy(), gs, bits)
    assert np.array_equal(np16(xq), qa)
    assert np.array_equal(bits16(np16(flexq.act_scales_view(xs, xq.shape[0]))), bits16(sa))


@pytest.mark.parametrize("bits", [6, 8])
def test_act_quant_edge_values(bits):
    gs, K = 32, 512
    rows = [
        np.zeros(K),                                            # all-zero groups
        np.full(K, 2.0 ** -24),                                 # scale underflows
        np.tile([46 * 2.0 ** -24, 3 * 2.0 ** -24, -46 * 2.0 ** -24, 0], K // 4),
        np.tile([31.0, 2.5, 3.5, -2.5, 0.5, 1.5, -31.0, 30.5], K // 8),   # ties
        np.tile([127.0, 126.5, -126.5, 0.5], K // 4),
        np.full(K, 65504.0),                                    # largest finite
        np.tile([-65504.0, 1e-3, 7.0, -0.0], K // 4),
        np.linspace(-3, 3, K),
    ]
    x = np.stack(rows).astype(np.float16)
    xq, xs = flexq.quantize_act(torch.from_numpy(x).cuda(), gs, bits)
    qa, sa = orc.quantize_act(x, gs, bits)
    assert np.array_equal(np16(xq), qa)
    assert np.array_equal(bits16(np16(flexq.act_scales_view(xs, xq.shape[0]))), bits16(sa))


def test_act_quant_full_row_width_sweep_shape():
    # the activation-quantization sweep shape [M, 8192], outlier channels
    M, K, gs = 2048, 8192, 128
    x = inputs.activations(M, K, outlier_frac=0.005, outlier_scale=50.0, seed=77)
    for bits in (6, 8):
        xq, xs = flexq.quantize_act(x.cuda(), gs, bits)
        qa, sa = orc.quantize_act(x.numpy(), gs, bits)
        assert np.array_equal(np16(xq), qa)
        assert np.array_equal(bits16(np16(flexq.act_scales_view(xs, xq.shape[0]))), bits16(sa))


def test_act_quant_empty_is_noop():
    x = torch.empty(0, 256, dtype=torch.float16, device="cuda")
    xq, xs = flexq.quantize_act(x, 128, 6)
    assert xq.shape == (0, 256) and xs.shape == (2, 0)


@pytest.mark.parametrize("gs", [32, 64, 128, 256])
@pytest.mark.parametrize("N,K", [(128, 256), (256, 512), (384, 1024)])
def test_weight_quant_pack_bit_exact(N, K, gs):
    w = inputs.weights(N, K, seed=inputs.layer_seed("w", N, K, gs))
    wp, ws = flexq.quantize_weight(w.cuda(), gs)
    qw, sw, dev = oracle_weight_device_form(w.numpy(), gs)
    assert np.array_equal(bits16(np16(flexq.weight_scales_view(ws))), bits16(sw))
    assert np.array_equal(np16(wp), dev)


def test_weight_quant_pack_edge_values():
    N, K, gs = 128, 256, 32
    w = np.zeros((N, K), dtype=np.float64)
    w[0, :32] = 0.0                                   # zero group
    w[1, :32] = 2.0 ** -24                            # scale underflows
    w[2, :32] = np.tile([46 * 2.0 ** -24, -46 * 2.0 ** -24], 16)   # clamp
    w[3, :32] = np.tile([31.0, -31.0, 2.5, 3.5], 8)
    w[4, :] = np.linspace(-1, 1, K)
    w[5:, :] = np.random.default_rng(1).standard_normal((N - 5, K)) * 0.02
    w16 = w.astype(np.float16)
    wp, ws = flexq.quantize_weight(torch.from_numpy(w16).cuda(), gs)
    qw, sw, dev = oracle_weight_device_form(w16, gs)
    assert np.array_equal(bits16(np16(flexq.weight_scales_view(ws))), bits16(sw))
    assert np.array_equal(np16(wp), dev)


def test_weight_quant_pack_llama_shape():
    N, K, gs = 4096, 4096, 128
    w = inputs.weights(N, K, seed=5)
    wp, ws = flexq.quantize_weight(w.cuda(), gs)
    qw, sw, dev = oracle_weight_device_form(w.numpy(), gs)
    assert np.array_equal(bits16(np16(flexq.weight_scales_view(ws))), bits16(sw))
    assert np.array_equal(np16(wp), dev)


def test_fast_code_rule_equals_the_ieee_division_rule_exhaustively():
    # every finite FP16 x against every positive finite FP16 scale, Q = 31 and
    # Q = 127: the division-free rule the kernels use gives the same code as
    # FP32 division + round half to even + clamp
    n, first = flexq.debug_check_quantizer()
    assert n == 0, f"{n} mismatches, first (x bits, s bits, Q) = {first}"
