"""Seeded random configurations against the oracle: shape, group size, bit
width, tile width, K split and linear route drawn together, so that
combinations no hand-written case names (a ragged token tail with a K split
at group 32 on 64-token tiles, ...) are covered too.  Every draw is fixed by
the seed; a failure prints its configuration."""

import numpy as np
import pytest
import torch

from bit_group_quantized_flexq_b200 import flexq, inputs
from oracle import flexq_oracle as orc
from tests.gpu_util import assert_within, np16

pytestmark = pytest.mark.gpu

TOL = 1e-3


def _draws(n, seed=20261202):
    rng = np.random.default_rng(seed)
    out = []
    for i in range(n):
        gs = int(rng.choice([32, 64, 128, 256]))
        K = int(rng.integers(1, 13)) * 256                  # 256 .. 3072
        N = int(rng.integers(1, 9)) * 128                   # 128 .. 1024
        M = int(rng.choice([1, 2, 3, 5, 8, 13, 16, 17, 31, 33, 47, 64, 65, 100, 129, 200]))
        bits = int(rng.choice([6, 8]))
        T = int(rng.choice([0, 16, 32, 64, 128]))           # 0: the planner's choice
        max_s = {0: 1, 16: 8, 32: 6, 64: 4, 128: 4}[T]
        S = int(rng.integers(0, min(max_s, K // 256) + 1)) if T else 0
        route = int(rng.choice([0, 1, 2]))
        out.append((i, M, N, K, gs, bits, T, S, route))
    return out


@pytest.fixture(autouse=True)
def _restore():
    yield
    flexq.force_plan(0, 0)
    flexq.force_linear_route(0)


@pytest.mark.parametrize("i,M,N,K,gs,bits,T,S,route", _draws(40))
def test_random_configuration(i, M, N, K, gs, bits, T, S, route):
    seed = inputs.layer_seed("random", i, M, N, K, gs)
    x = inputs.activations(M, K, outlier_frac=0.01, outlier_scale=20.0, seed=seed)
    w = inputs.weights(N, K, std=0.02, seed=seed + 1)
    wp, ws = flexq.quantize_weight(w.cuda(), gs)
    flexq.force_plan(T, S)
    flexq.force_linear_route(route)
    xc = x.cuda()
    y = flexq.linear(xc, wp, ws, N, gs, bits)
    xq, xs = flexq.quantize_act(xc, gs, bits)
    y2 = flexq.gemm(xq, xs, wp, ws, N, gs, bits)
    assert torch.equal(y, y2), (M, N, K, gs, bits, T, S, route)   # same plan, same arithmetic
    ref = orc.linear_layer(x.numpy(), w.numpy(), gs, bits)
    assert np.array_equal(np16(xq), ref["qa"])
    assert_within(np16(y), ref["y64"], TOL)
    assert flexq.device_status()[0] == flexq.FLEXQ_OK
