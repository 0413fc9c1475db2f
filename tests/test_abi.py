"""The C-ABI library without a GPU: it loads, exports every entry point that
include/flexq.h declares, and rejects invalid arguments before touching CUDA."""

import ctypes
import os
import re

import pytest

from bit_group_quantized_flexq_b200 import build as flexq_build
from bit_group_quantized_flexq_b200 import flexq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    flexq_build.build()
    return flexq.lib()


def declared_functions():
    text = open(os.path.join(ROOT, "include", "flexq.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(flexq_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ["flexq_quantize_weight", "flexq_quantize_act", "flexq_gemm_w6a6",
                     "flexq_gemm_w6a8", "flexq_debug_group_partials",
                     "flexq_get_device_status", "flexq_weight_packed_bytes"]:
        assert required in names


def test_library_exports_every_declared_symbol(L):
    for name in declared_functions():
        assert hasattr(L, name), name


def test_status_strings(L):
    assert L.flexq_status_string(0) == b"FLEXQ_OK"
    assert L.flexq_status_string(5) == b"FLEXQ_ERR_DEVICE_TIMEOUT"
    assert L.flexq_status_string(99) == b"FLEXQ_ERR_UNKNOWN"


def test_packed_size(L):
    assert L.flexq_weight_packed_bytes(4096, 4096, 128) == 4096 * 4096 * 3 // 4
    assert L.flexq_weight_packed_bytes(28672, 8192, 32) == 28672 * 8192 * 3 // 4
    assert L.flexq_weight_packed_bytes(100, 4096, 128) == 0        # N % 128
    assert L.flexq_weight_packed_bytes(128, 4096, 48) == 0         # bad gs
    assert L.flexq_weight_packed_bytes(128, 192, 64) == 0          # K % 256
    assert L.flexq_weight_packed_bytes(128, 384, 128) == 0         # K % 256


FAKE = ctypes.c_void_p(1 << 20)          # never dereferenced: validation fails first
MISALIGNED = ctypes.c_void_p((1 << 20) + 8)
NULL = ctypes.c_void_p(0)


def test_validation_before_any_launch(L):
    # bad bit width
    assert L.flexq_quantize_act(4, 256, 128, 7, FAKE, FAKE, FAKE, NULL) == flexq.FLEXQ_ERR_INVALID_ARG
    assert b"bits" in L.flexq_last_error_message()
    # bad group size / K not a multiple of the group
    assert L.flexq_quantize_act(4, 256, 48, 6, FAKE, FAKE, FAKE, NULL) == flexq.FLEXQ_ERR_UNSUPPORTED
    assert L.flexq_quantize_act(4, 160, 64, 6, FAKE, FAKE, FAKE, NULL) == flexq.FLEXQ_ERR_UNSUPPORTED
    # null and misaligned pointers
    assert L.flexq_quantize_act(4, 256, 128, 6, NULL, FAKE, FAKE, NULL) == flexq.FLEXQ_ERR_INVALID_ARG
    assert L.flexq_quantize_act(4, 256, 128, 6, FAKE, MISALIGNED, FAKE, NULL) == flexq.FLEXQ_ERR_MISALIGNED
    # negative sizes
    assert L.flexq_quantize_act(-1, 256, 128, 6, FAKE, FAKE, FAKE, NULL) == flexq.FLEXQ_ERR_INVALID_ARG
    # GEMM shape rules
    g = L.flexq_gemm_w6a6
    assert g(4, 200, 256, 128, FAKE, FAKE, FAKE, FAKE, FAKE, NULL, 0, NULL) == flexq.FLEXQ_ERR_UNSUPPORTED
    assert g(4, 256, 200, 128, FAKE, FAKE, FAKE, FAKE, FAKE, NULL, 0, NULL) == flexq.FLEXQ_ERR_UNSUPPORTED
    assert g(4, 256, 384, 256, FAKE, FAKE, FAKE, FAKE, FAKE, NULL, 0, NULL) == flexq.FLEXQ_ERR_UNSUPPORTED
    assert g(4, 256, 256, 128, FAKE, NULL, FAKE, FAKE, FAKE, NULL, 0, NULL) == flexq.FLEXQ_ERR_INVALID_ARG
    assert g(4, 256, 256, 128, FAKE, FAKE, FAKE, FAKE, MISALIGNED, NULL, 0, NULL) == flexq.FLEXQ_ERR_MISALIGNED
    assert L.flexq_gemm_w6a8(-3, 256, 256, 128, FAKE, FAKE, FAKE, FAKE, FAKE, NULL, 0, NULL) == \
        flexq.FLEXQ_ERR_INVALID_ARG
    w = L.flexq_quantize_weight
    assert w(130, 256, 128, FAKE, FAKE, FAKE, NULL) == flexq.FLEXQ_ERR_UNSUPPORTED
    assert w(128, 256, 128, FAKE, NULL, FAKE, NULL) == flexq.FLEXQ_ERR_INVALID_ARG
    assert L.flexq_debug_force_plan(48, 0) == flexq.FLEXQ_ERR_INVALID_ARG
    assert L.flexq_debug_force_plan(16, 9) == flexq.FLEXQ_ERR_INVALID_ARG
    assert L.flexq_set_wait_limit_ns(0) == flexq.FLEXQ_ERR_INVALID_ARG


def test_plan_is_host_only_and_sane(L):
    # tokens per tile follow M; K splits fill the machine at decode sizes
    for M, T in [(1, 16), (16, 16), (17, 32), (64, 32), (65, 128), (2048, 128)]:
        t, s, c = flexq.plan(M, 4096, 4096, 128)
        assert t == T
        assert 1 <= s <= 8
        tiles = (4096 // 128) * ((M + t - 1) // t)
        if tiles < 148:                   # fewer tiles than SMs: every tile split
            assert c == s * tiles
        else:                             # whole waves unsplit, the last wave split
            assert tiles <= c <= s * tiles
    # M = 2048, N = K = 4096: 512 tiles = 3 waves of 148 + 68; those 68 split in 2
    assert flexq.plan(2048, 4096, 4096, 128) == (128, 2, 444 + 2 * 68)
    # N = 11008: 1376 tiles = 9 waves + 44; those 44 split in 3
    assert flexq.plan(2048, 11008, 4096, 128) == (128, 3, 1332 + 3 * 44)
    t, s, c = flexq.plan(1, 4096, 4096, 128)
    assert s > 1                      # 32 weight tiles alone would idle most SMs
    t, s, c = flexq.plan(1, 4096, 256, 256)
    assert s == 1                     # one group: nothing to split
    # the split units never exceed one wave of CTA slots (2 per SM at T = 16)
    for N, K in [(8192, 8192), (11008, 4096), (4096, 11008), (28672, 8192)]:
        t, s, c = flexq.plan(1, N, K, 128)
        assert c <= 2 * 148
    assert flexq.plan(1, 8192, 8192, 128) == (16, 4, 256)
    # 33..64 tokens: two 32-token tiles while they fit one wave, else one 64-token tile
    assert flexq.plan(64, 5120, 5120, 128) == (32, 3, 240)
    assert flexq.plan(64, 28672, 8192, 128)[0] == 64
    assert flexq.plan(0, 256, 256, 128) == (0, 0, 0)


def test_workspace_size_follows_the_plan(L):
    # no K split: no workspace; a K split: FP32 partial tiles + one counter per tile
    assert flexq.gemm_workspace_bytes(2048, 4096, 4096, 128) == 0 or flexq.plan(2048, 4096, 4096, 128)[1] > 1
    for M, N, K in [(1, 4096, 4096), (16, 11008, 4096), (5, 384, 4096), (2048, 4096, 4096)]:
        t, s, c = flexq.plan(M, N, K, 128)
        tiles = (N // 128) * ((M + t - 1) // t)
        n_split = (c - tiles) // (s - 1) if s > 1 else 0
        want = 0 if s == 1 else 4096 + n_split * s * t * 128 * 4
        assert flexq.gemm_workspace_bytes(M, N, K, 128) == want
    assert flexq.gemm_workspace_bytes(0, 4096, 4096, 128) == 0
    assert flexq.gemm_workspace_bytes(4, 200, 4096, 128) == 0


def test_linear_validation_before_any_launch(L):
    f = L.flexq_linear_w6a6
    # bad bit width (the w6a6/w6a8 wrappers fix it), shapes, pointers
    assert f(4, 200, 256, 128, FAKE, FAKE, FAKE, FAKE, NULL, 0, NULL) == flexq.FLEXQ_ERR_UNSUPPORTED
    assert f(4, 256, 256, 48, FAKE, FAKE, FAKE, FAKE, NULL, 0, NULL) == flexq.FLEXQ_ERR_UNSUPPORTED
    assert f(4, 256, 256, 128, NULL, FAKE, FAKE, FAKE, NULL, 0, NULL) == flexq.FLEXQ_ERR_INVALID_ARG
    assert b"X_fp16" in L.flexq_last_error_message()
    assert f(4, 256, 256, 128, MISALIGNED, FAKE, FAKE, FAKE, NULL, 0, NULL) == flexq.FLEXQ_ERR_MISALIGNED
    assert L.flexq_linear_w6a8(-1, 256, 256, 128, FAKE, FAKE, FAKE, FAKE, NULL, 0, NULL) == \
        flexq.FLEXQ_ERR_INVALID_ARG
    assert f(0, 256, 256, 128, FAKE, FAKE, FAKE, FAKE, NULL, 0, NULL) == flexq.FLEXQ_OK   # empty batch


def test_linear_workspace_layout(L):
    # small batches on short K ranges quantize inside the GEMM: the GEMM's workspace alone
    for M, N, K in [(1, 4096, 4096), (2, 1024, 8192), (1, 384, 1024), (8, 4096, 4096),
                    (1, 11008, 4096)]:
        assert flexq.linear_launches(M, N, K, 128) == 1
        assert flexq.linear_workspace_bytes(M, N, K, 128) == flexq.gemm_workspace_bytes(M, N, K, 128)
    # the others add the codes and the scales after the GEMM region
    for M, N, K, gs in [(4, 11008, 4096, 128), (16, 11008, 4096, 128), (17, 4096, 4096, 128),
                        (1, 28672, 8192, 128), (256, 4096, 11008, 64), (2048, 4096, 4096, 128)]:
        assert flexq.linear_launches(M, N, K, gs) == 2
        head = max(flexq.gemm_workspace_bytes(M, N, K, gs), 4096)
        xq_off = (head + 255) // 256 * 256
        xs_off = (xq_off + M * K + 255) // 256 * 256
        want = xs_off + (K // gs) * flexq.act_scales_ld(M) * 2
        assert flexq.linear_workspace_bytes(M, N, K, gs) == want
    assert flexq.linear_workspace_bytes(0, 4096, 4096, 128) == 0
    assert flexq.linear_workspace_bytes(4, 200, 4096, 128) == 0
    assert flexq.linear_launches(0, 4096, 4096, 128) == 0
    assert L.flexq_debug_force_linear_route(3) == flexq.FLEXQ_ERR_INVALID_ARG


def test_static_scratch_validation_before_any_launch(L):
    f = L.flexq_gemm_static_scratch
    args = (FAKE, FAKE, FAKE, FAKE, FAKE, NULL)
    assert f(4, 256, 256, 128, 7, *args) == flexq.FLEXQ_ERR_INVALID_ARG       # act_bits
    assert b"act_bits" in L.flexq_last_error_message()
    assert f(4, 200, 256, 128, 6, *args) == flexq.FLEXQ_ERR_UNSUPPORTED       # N % 128
    assert f(4, 256, 256, 48, 8, *args) == flexq.FLEXQ_ERR_UNSUPPORTED        # group size
    assert f(4, 256, 384, 256, 6, *args) == flexq.FLEXQ_ERR_UNSUPPORTED       # K % 256
    assert f(-1, 256, 256, 128, 6, *args) == flexq.FLEXQ_ERR_INVALID_ARG
    assert f(0, 256, 256, 128, 6, *args) == flexq.FLEXQ_OK                    # empty batch
    # pointers are checked before the counter clear is enqueued: no GPU needed
    assert f(4, 256, 256, 128, 6, FAKE, NULL, FAKE, FAKE, FAKE, NULL) == flexq.FLEXQ_ERR_INVALID_ARG
    assert b"X_scales" in L.flexq_last_error_message()
    assert f(4, 256, 256, 128, 8, FAKE, FAKE, FAKE, FAKE, MISALIGNED, NULL) == \
        flexq.FLEXQ_ERR_MISALIGNED


def test_group_validation_before_any_launch(L):
    Layer = flexq.Layer
    arr = (Layer * 2)(Layer(256, 1 << 20, 1 << 20, 1 << 20), Layer(384, 1 << 20, 1 << 20, 1 << 20))
    g = L.flexq_gemm_group
    assert g(4, 256, 128, 6, FAKE, FAKE, 0, arr, NULL, 0, NULL) == flexq.FLEXQ_ERR_INVALID_ARG
    assert g(4, 256, 128, 6, FAKE, FAKE, 5, arr, NULL, 0, NULL) == flexq.FLEXQ_ERR_INVALID_ARG
    assert g(4, 256, 128, 6, FAKE, FAKE, 2, None, NULL, 0, NULL) == flexq.FLEXQ_ERR_INVALID_ARG
    assert g(4, 256, 128, 7, FAKE, FAKE, 2, arr, NULL, 0, NULL) == flexq.FLEXQ_ERR_INVALID_ARG
    bad = (Layer * 1)(Layer(200, 1 << 20, 1 << 20, 1 << 20))
    assert g(4, 256, 128, 6, FAKE, FAKE, 1, bad, NULL, 0, NULL) == flexq.FLEXQ_ERR_UNSUPPORTED
    assert g(4, 256, 128, 6, NULL, FAKE, 2, arr, NULL, 0, NULL) == flexq.FLEXQ_ERR_INVALID_ARG
    nul = (Layer * 1)(Layer(256, 1 << 20, 0, 1 << 20))
    assert g(4, 256, 128, 6, FAKE, FAKE, 1, nul, NULL, 0, NULL) == flexq.FLEXQ_ERR_INVALID_ARG
    assert g(0, 256, 128, 6, FAKE, FAKE, 2, arr, NULL, 0, NULL) == flexq.FLEXQ_OK
    f = L.flexq_linear_group
    assert f(4, 256, 128, 8, NULL, 2, arr, NULL, 0, NULL) == flexq.FLEXQ_ERR_INVALID_ARG
    assert f(4, 256, 48, 8, FAKE, 2, arr, NULL, 0, NULL) == flexq.FLEXQ_ERR_UNSUPPORTED


def test_group_plan_is_host_only_and_sane(L):
    # LLaMA-2-70B q/k/v at one token: 80 weight tiles, split 3 -> 240 CTAs
    assert flexq.group_plan(1, 8192, 128, [8192, 1024, 1024])[:3] == (16, 3, 240)
    # one layer: the grouped plan splits like the single-layer one when it fits a wave
    t, s, c, n = flexq.group_plan(1, 4096, 128, [4096])
    assert (t, s, c) == flexq.plan(1, 4096, 4096, 128)
    # 128-token tiles: one launch per layer after the quantizer
    assert flexq.group_plan(512, 8192, 128, [28672, 28672]) == (128, 0, 0, 3)
    assert flexq.gemm_group_workspace_bytes(1, 8192, 128, [8192, 1024, 1024]) == \
        4096 + 80 * 3 * 16 * 128 * 4


def test_layout_validation_before_any_launch(L):
    assert L.flexq_quantize_weight_layout(128, 256, 128, 2, FAKE, FAKE, FAKE, NULL) == \
        flexq.FLEXQ_ERR_INVALID_ARG
    assert L.flexq_quantize_weight_layout(128, 256, 128, 1, FAKE, NULL, FAKE, NULL) == \
        flexq.FLEXQ_ERR_INVALID_ARG
    g = L.flexq_gemm_layout
    assert g(4, 256, 256, 128, 6, 3, FAKE, FAKE, FAKE, FAKE, FAKE, NULL, 0, NULL) == \
        flexq.FLEXQ_ERR_INVALID_ARG
    assert g(4, 256, 256, 128, 5, 1, FAKE, FAKE, FAKE, FAKE, FAKE, NULL, 0, NULL) == \
        flexq.FLEXQ_ERR_INVALID_ARG
    assert g(4, 200, 256, 128, 6, 1, FAKE, FAKE, FAKE, FAKE, FAKE, NULL, 0, NULL) == \
        flexq.FLEXQ_ERR_UNSUPPORTED
    f = L.flexq_linear_layout
    assert f(4, 256, 256, 128, 6, -1, FAKE, FAKE, FAKE, FAKE, NULL, 0, NULL) == \
        flexq.FLEXQ_ERR_INVALID_ARG
    assert f(0, 256, 256, 128, 6, 1, FAKE, FAKE, FAKE, FAKE, NULL, 0, NULL) == flexq.FLEXQ_OK


def test_export_canonical_validation_before_any_launch(L):
    f = L.flexq_debug_export_canonical
    assert f(256, 512, 2, FAKE, FAKE, NULL) == flexq.FLEXQ_ERR_INVALID_ARG          # layout
    assert f(200, 512, 0, FAKE, FAKE, NULL) == flexq.FLEXQ_ERR_UNSUPPORTED          # N % 128
    assert f(256, 384, 1, FAKE, FAKE, NULL) == flexq.FLEXQ_ERR_UNSUPPORTED          # K % 256
    assert f(0, 512, 0, FAKE, FAKE, NULL) == flexq.FLEXQ_ERR_INVALID_ARG            # N <= 0
    assert f(256, 512, 0, NULL, FAKE, NULL) == flexq.FLEXQ_ERR_INVALID_ARG
    assert b"Wq_packed" in L.flexq_last_error_message()
    assert f(256, 512, 0, FAKE, MISALIGNED, NULL) == flexq.FLEXQ_ERR_MISALIGNED
    assert b"W_canonical" in L.flexq_last_error_message()
