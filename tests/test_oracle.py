"""Pins for the CPU oracle (no GPU).

The pages print no worked example and no table, so the oracle is pinned to
things outside itself: hand-worked cases in tests/golden/, an independent
exact-rational quantizer, the round-to-nearest-even definition at every FP16
midpoint, torch's converter, exhaustive pack/unpack identity, brute-force FP64
matmul of the dequantized operands and the one-group unit-scale closed form.
"""

import json
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import flexq_oracle as orc
from bit_group_quantized_flexq_b200 import inputs


# ------------------------------------------------------------ helpers ------
def fp16_from_bits(bits):
    return np.array([bits], dtype=np.uint16).view(np.float16)[0]


def fp16_value(v):
    if isinstance(v, str) and v.startswith("h:"):
        return fp16_from_bits(int(v[2:], 16))
    return np.float16(v)


def exact_fp16_rne(fr):
    """Round a Fraction to the nearest FP16 value (ties to even mantissa),
    written from the binary16 definition; returns the value as a Fraction or
    None for overflow.  Independent of numpy's and torch's converters."""
    if fr == 0:
        return Fraction(0)
    sign = -1 if fr < 0 else 1
    a = abs(fr)
    # binary16: normal numbers (1 + f/1024) * 2^e for e in [-14, 15];
    # subnormals f/1024 * 2^-14; the quantum at exponent e is 2^(e-10).
    e = 15
    while e > -14 and a < Fraction(2) ** e:
        e -= 1
    quantum = Fraction(2) ** (e - 10)
    q, r = divmod(a, quantum)            # a = q*quantum + r, 0 <= r < quantum
    half = quantum / 2
    if r > half or (r == half and q % 2 == 1):
        q += 1
    v = q * quantum
    if v > Fraction(65504):
        return None
    return sign * v


def exact_quantize_group(xs, qmax):
    """Quantize one group with exact rational arithmetic (no floating point):
    s = fp16_rne(amax / Q); q = round_half_even(x / s) clamped to [-Q, Q]."""
    fx = [Fraction(float(x)) for x in xs]      # fp16 -> exact rational
    amax = max(abs(v) for v in fx)
    s = exact_fp16_rne(amax / qmax)
    if s == 0:
        return [0] * len(xs), Fraction(0)
    codes = []
    for v in fx:
        r = v / s
        fl = r.numerator // r.denominator
        rem = r - fl
        if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
            fl += 1
        codes.append(max(-qmax, min(qmax, fl)))
    return codes, s


# ------------------------------------------------------------ FP16 codec ----
def all_fp16():
    return np.arange(65536, dtype=np.uint32).astype(np.uint16).view(np.float16)


def test_fp16_widening_matches_torch_exhaustive():
    h = all_fp16()
    ours = h.astype(np.float32)
    theirs = torch.from_numpy(h.copy()).to(torch.float32).numpy()
    nan = np.isnan(ours)
    assert np.array_equal(nan, np.isnan(theirs))
    assert np.array_equal(ours[~nan], theirs[~nan])
    # round trip through float32 is the identity on every non-NaN pattern
    back = ours.astype(np.float16).view(np.uint16)
    assert np.array_equal(back[~nan], h.view(np.uint16)[~nan])


def _adjacent_pairs():
    bits = np.arange(0, 0x7BFF, dtype=np.uint16)   # lower neighbour, < max
    lo = bits.view(np.float16).astype(np.float64)
    hi = (bits + 1).view(np.float16).astype(np.float64)
    return bits, lo, hi


@pytest.mark.parametrize("dtype", [np.float32, np.float64])
def test_fp16_rounding_is_nearest_even_at_every_midpoint(dtype):
    bits, lo, hi = _adjacent_pairs()
    mid = ((lo + hi) / 2).astype(dtype)           # exact in both widths
    assert np.array_equal(mid.astype(np.float64), (lo + hi) / 2)
    got = mid.astype(np.float16).view(np.uint16)
    even = np.where(bits % 2 == 0, bits, bits + 1).astype(np.uint16)
    assert np.array_equal(got, even)
    # just above / below a midpoint goes to the nearer neighbour
    up = np.nextafter(mid, dtype(np.inf)).astype(np.float16).view(np.uint16)
    dn = np.nextafter(mid, dtype(-np.inf)).astype(np.float16).view(np.uint16)
    assert np.array_equal(up, (bits + 1).astype(np.uint16))
    assert np.array_equal(dn, bits)
    # negative values mirror
    neg = (-mid).astype(np.float16).view(np.uint16)
    assert np.array_equal(neg, even | np.uint16(0x8000))


@pytest.mark.parametrize("dtype", [np.float32, np.float64])
def test_fp16_overflow_boundary(dtype):
    # 65520 is the midpoint between 65504 (odd mantissa) and 2^16: ties away
    # from the odd neighbour, i.e. to infinity
    assert np.isinf(dtype(65520.0).astype(np.float16))
    below = np.nextafter(dtype(65520.0), dtype(0))
    assert below.astype(np.float16) == np.float16(65504.0)
    assert dtype(-65520.0).astype(np.float16) == -np.inf


def test_fp16_narrowing_from_fp32_matches_torch_random():
    rng = np.random.default_rng(5)
    v = np.concatenate([
        rng.standard_normal(200_000) * 10.0 ** rng.integers(-9, 5, 200_000),
        rng.uniform(-65000, 65000, 20_000)]).astype(np.float32)
    ours = v.astype(np.float16).view(np.uint16)
    theirs = torch.from_numpy(v.copy()).to(torch.float16).numpy().view(np.uint16)
    assert np.array_equal(ours, theirs)


def test_fp16_narrowing_from_fp64_is_single_rounding():
    # torch narrows FP64 through FP32 (two roundings); the oracle must round
    # once, so FP64 is checked against the exact rational converter instead
    rng = np.random.default_rng(6)
    v = rng.standard_normal(20_000) * 10.0 ** rng.integers(-9, 5, 20_000)
    # include values just below FP16 midpoints, where double rounding errs
    bits, lo, hi = _adjacent_pairs()
    pick = rng.choice(bits.size, 2000, replace=False)
    v = np.concatenate([v, np.nextafter((lo[pick] + hi[pick]) / 2, 0)])
    ours = v.astype(np.float16)
    for x, h in zip(v, ours):
        assert Fraction(float(h)) == exact_fp16_rne(Fraction(float(x)))


def test_exact_converter_agrees_with_numpy_on_samples():
    rng = np.random.default_rng(11)
    vals = rng.standard_normal(3000) * 10.0 ** rng.integers(-8, 4, 3000)
    for v in vals:
        ref = exact_fp16_rne(Fraction(float(v)))
        assert Fraction(float(np.float64(v).astype(np.float16))) == ref


# ------------------------------------------------------------ quantizer -----
def _golden(name, golden_dir):
    with open(os.path.join(golden_dir, name)) as f:
        return json.load(f)


def test_quantizer_hand_worked_cases(golden_dir):
    g = _golden("quant_cases.json", golden_dir)
    gs = g["group_size"]
    for case in g["cases"]:
        x = np.zeros((1, gs), dtype=np.float16)
        for i, v in case["x"]:
            x[0, i] = fp16_value(v)
        codes, scales = orc.quantize_groups(x, gs, case["Q"])
        want = np.zeros(gs, dtype=np.int8)
        for i, c in case["codes"]:
            want[i] = c
        assert np.array_equal(codes[0], want), case["name"]
        assert int(scales.view(np.uint16)[0, 0]) == int(case["scale_bits"], 16), case["name"]


@pytest.mark.parametrize("qmax", [31, 127])
def test_quantizer_matches_exact_rational_quantizer(qmax):
    rng = np.random.default_rng(qmax)
    gs = 32
    rows = []
    # ordinary, outlier-heavy, tiny (subnormal scales) and tie-rich groups
    rows.append(rng.standard_normal((24, gs)))
    rows.append(rng.standard_normal((8, gs)) * np.where(rng.random((8, gs)) < 0.1, 50, 1))
    rows.append(rng.standard_normal((8, gs)) * 1e-6)
    rows.append(rng.integers(-62, 63, (8, gs)) / 4.0)
    x = np.concatenate(rows).astype(np.float16)
    codes, scales = orc.quantize_groups(x, gs, qmax)
    for r in range(x.shape[0]):
        want_codes, want_s = exact_quantize_group(x[r], qmax)
        assert list(codes[r].astype(int)) == want_codes, r
        assert Fraction(float(scales[r, 0])) == want_s, r


@pytest.mark.parametrize("gs", [32, 64, 128, 256])
@pytest.mark.parametrize("qmax", [31, 127])
def test_quantizer_invariants(gs, qmax):
    x = inputs.activations(16, 1024, seed=3).numpy()
    codes, s16 = orc.quantize_groups(x, gs, qmax)
    G = 1024 // gs
    assert codes.min() >= -qmax and codes.max() <= qmax
    s = s16.astype(np.float64)
    xg = x.astype(np.float64).reshape(16, G, gs)
    qg = codes.astype(np.float64).reshape(16, G, gs)
    amax = np.abs(xg).max(axis=2)
    # stored scale within one fp16 rounding of amax / Q
    assert np.all(np.abs(s - amax / qmax) <= (amax / qmax) * 2.0 ** -11)
    # every value is within half a step of its dequantized code (no clamp
    # happens for normal scales, since amax / s <= Q (1 + 2^-11) < Q + 1/2)
    err = np.abs(qg * s[:, :, None] - xg)
    assert np.all(err <= s[:, :, None] / 2 * (1 + 1e-6))
    # the absmax element maps to +-Q
    idx = np.abs(xg).argmax(axis=2)
    top = np.take_along_axis(np.abs(qg), idx[:, :, None], axis=2)[..., 0]
    assert np.all(top == qmax)


def test_weight_and_act_wrappers():
    w = inputs.weights(8, 256, seed=4).numpy()
    qw, sw = orc.quantize_weight(w, 128)
    assert qw.min() >= -31 and qw.max() <= 31 and sw.shape == (8, 2)
    x = inputs.activations(3, 256, seed=5).numpy()
    for bits, q in [(6, 31), (8, 127)]:
        qa, sa = orc.quantize_act(x, 64, bits)
        assert np.abs(qa).max() == q and sa.shape == (3, 4)


# ------------------------------------------------------------ packing -------
def test_pack_hand_worked_cases(golden_dir):
    g = _golden("pack_cases.json", golden_dir)
    for case in g["cases"]:
        codes = np.array([case["codes"]], dtype=np.int8)
        packed = orc.pack_canonical(codes)
        assert packed.tobytes().hex() == case["bytes"], case
        assert np.array_equal(orc.unpack_canonical(packed, 4), codes)


def test_pack_unpack_identity_exhaustive():
    # all 64^4 tuples of 6-bit codes, including -32
    c = np.arange(-32, 32, dtype=np.int8)
    grid = np.stack(np.meshgrid(c, c, c, c, indexing="ij"), axis=-1).reshape(-1, 4)
    rows = grid.reshape(4096, 4096 * 4)        # [4096 rows, 16384 codes]
    packed = orc.pack_canonical(rows)
    assert packed.shape == (4096, 12288)
    assert np.array_equal(orc.unpack_canonical(packed, rows.shape[1]), rows)
    # the packing is injective: 24 distinct bits per tuple
    words = packed.reshape(-1, 3).astype(np.uint32)
    w = words[:, 0] | (words[:, 1] << 8) | (words[:, 2] << 16)
    assert np.unique(w).size == 64 ** 4


def _block_codes(spec):
    c = np.zeros(16, dtype=np.int8)
    if spec == "all -1":
        c[:] = -1
    else:
        for j, v in spec.items():
            c[int(j)] = v
    return c


def test_device_block_hand_worked_cases(golden_dir):
    g = _golden("device_form_cases.json", golden_dir)
    for case in g["cases"]:
        codes = _block_codes(case["codes"])
        words = orc.pack_block_words(codes)
        assert words.astype("<u4").tobytes().hex() == case["bytes"], case
        assert np.array_equal(orc.unpack_block_words(words), codes)


def test_device_block_is_a_bit_permutation():
    # setting one bit of one code's 6-bit field sets exactly one bit of the
    # block, and the 96 (code, bit) pairs land on 96 distinct bits: the block
    # is a bijection of 16 six-bit fields onto 96 bits
    seen = set()
    for j in range(16):
        for bit in range(6):
            u = 1 << bit
            c = np.zeros(16, dtype=np.int8)
            c[j] = u - 64 if u >= 32 else u
            w = orc.pack_block_words(c).astype(np.uint64)
            value = int(w[0]) | (int(w[1]) << 32) | (int(w[2]) << 64)
            assert bin(value).count("1") == 1, (j, bit)
            seen.add(value.bit_length() - 1)
    assert seen == set(range(96))


def test_device_block_roundtrip_every_value_at_every_position():
    rng = np.random.default_rng(4)
    base = rng.integers(-32, 32, (64, 16)).astype(np.int8)
    for j in range(16):
        c = base.copy()
        c[:, j] = np.arange(-32, 32, dtype=np.int8)
        assert np.array_equal(orc.unpack_block_words(orc.pack_block_words(c)), c)


def test_device_form_tile_positions():
    N, K = 256, 384
    rng = np.random.default_rng(9)
    codes = rng.integers(-32, 32, (N, K)).astype(np.int8)
    dev = orc.pack_device_form(codes)
    assert dev.size == N * K * 3 // 4
    assert np.array_equal(orc.unpack_device_form(dev, N, K), codes)
    # spot-check the stated position formula with plain index arithmetic:
    # row n, block b (codes 16b..16b+15) -> row byte 12b + 4i + t of word i
    KB = K // 128
    for n in (0, 1, 127, 128, 200, 255):
        for b in (0, 5, 7, 8, 15, 23):
            words = orc.pack_block_words(codes[n, 16 * b:16 * b + 16])
            row_bytes = words.astype("<u4").tobytes()
            for pos in range(12):
                cb = 12 * b + pos                     # byte index within the row
                nt, r = divmod(n, 128)
                kb, within = divmod(cb, 96)
                j, byte = divmod(within, 16)
                off = ((nt * KB + kb) * 6 + j) * 128 * 16 + r * 16 + byte
                assert dev[off] == row_bytes[pos], (n, b, pos)


# --------------------------------------------------- "4+2" bit planes ------
def _block42_codes(spec):
    c = np.zeros(16, dtype=np.int8)
    if spec == "all -1":
        c[:] = -1
    elif spec == "all 1":
        c[:] = 1
    else:
        for j, v in spec.items():
            c[int(j)] = v
    return c


def test_planes42_hand_worked_cases(golden_dir):
    g = _golden("planes42_cases.json", golden_dir)
    for case in g["cases"]:
        codes = _block42_codes(case["codes"])
        nib, two = orc.pack_planes42(codes)
        assert nib.tobytes().hex() == case["nib"], case
        assert two.tobytes().hex() == case["two"], case
        assert np.array_equal(orc.unpack_planes42(nib, two), codes)


def test_planes42_is_a_bit_permutation():
    # one bit of one code's 6-bit field sets exactly one of the block's 96
    # bits, and the 96 (code, bit) pairs land on 96 distinct bits
    seen = set()
    for j in range(16):
        for bit in range(6):
            u = 1 << bit
            c = np.zeros(16, dtype=np.int8)
            c[j] = u - 64 if u >= 32 else u
            nib, two = orc.pack_planes42(c)
            value = int.from_bytes(nib.tobytes() + two.tobytes(), "little")
            assert bin(value).count("1") == 1, (j, bit)
            seen.add(value.bit_length() - 1)
    assert seen == set(range(96))
    # the high four bits of a code go to the 4-bit plane, the low two to the 2-bit plane
    for j in range(16):
        nib, two = orc.pack_planes42(np.eye(16, dtype=np.int8)[j] * 3)          # u = 0b000011
        assert not nib.any() and two.any()
        nib, two = orc.pack_planes42(np.eye(16, dtype=np.int8)[j] * -4)         # u = 0b111100
        assert nib.any() and not two.any()


def test_planes42_roundtrip_every_value_at_every_position():
    rng = np.random.default_rng(14)
    base = rng.integers(-32, 32, (64, 16)).astype(np.int8)
    for j in range(16):
        c = base.copy()
        c[:, j] = np.arange(-32, 32, dtype=np.int8)
        assert np.array_equal(orc.unpack_planes42(*orc.pack_planes42(c)), c)


def test_device_form42_tile_positions():
    N, K = 256, 384
    rng = np.random.default_rng(19)
    codes = rng.integers(-32, 32, (N, K)).astype(np.int8)
    dev = orc.pack_device_form42(codes)
    assert dev.size == N * K * 3 // 4
    assert np.array_equal(orc.unpack_device_form42(dev, N, K), codes)
    KB = K // 128
    for n in (0, 1, 127, 128, 200, 255):
        nt, r = divmod(n, 128)
        for b in (0, 5, 7, 8, 15, 23):
            nib, two = orc.pack_planes42(codes[n, 16 * b:16 * b + 16])
            kb, bt = divmod(b, 8)                  # tile along K, block within the tile
            tile = (nt * KB + kb) * 12288
            for pos in range(8):                   # 4-bit plane: row byte 8*bt + pos, chunks 0..3
                j, byte = divmod(8 * bt + pos, 16)
                assert dev[tile + (j * 128 + r) * 16 + byte] == nib[pos], (n, b, pos)
            for pos in range(4):                   # 2-bit plane: row byte 4*bt + pos, chunks 4, 5
                j, byte = divmod(4 * bt + pos, 16)
                assert dev[tile + ((4 + j) * 128 + r) * 16 + byte] == two[pos], (n, b, pos)
    # the planes are contiguous regions of each tile
    t0 = dev[:12288].reshape(6, 128, 16)
    nib_rows = t0[:4].transpose(1, 0, 2).reshape(128, 64)
    assert np.array_equal(nib_rows[3], np.concatenate(
        [orc.pack_planes42(codes[3, 16 * b:16 * b + 16])[0] for b in range(8)]))


# ------------------------------------------------------------ GEMM ----------
def test_gemm_hand_worked_case(golden_dir):
    g = _golden("gemm_case.json", golden_dir)
    K, gs = g["K"], g["group_size"]
    qa = np.zeros((1, K), dtype=np.int8)
    qw = np.zeros((1, K), dtype=np.int8)
    for i, v in g["qa"]:
        qa[0, i] = v
    for i, v in g["qw"]:
        qw[0, i] = v
    sa = np.array([g["sa"]], dtype=np.float16)
    sw = np.array([g["sw"]], dtype=np.float16)
    P = orc.group_partials(qa, qw, gs)
    assert list(P[:, 0, 0]) == g["partials"]
    y = orc.rescale_fp64(P, sa, sw)
    assert y[0, 0] == g["y"]
    assert orc.to_fp16(y)[0, 0] == np.float16(g["y"])


def test_partials_match_python_loops_tiny():
    rng = np.random.default_rng(2)
    M, N, K, gs = 3, 4, 64, 32
    qa = rng.integers(-127, 128, (M, K)).astype(np.int8)
    qw = rng.integers(-32, 32, (N, K)).astype(np.int8)
    P = orc.group_partials(qa, qw, gs)
    for g in range(K // gs):
        for m in range(M):
            for n in range(N):
                s = 0
                for k in range(g * gs, (g + 1) * gs):
                    s += int(qa[m, k]) * int(qw[n, k])
                assert P[g, m, n] == s


@pytest.mark.parametrize("gs", [32, 64, 128, 256])
def test_group_gemm_equals_dequantized_fp64_matmul(gs):
    x = inputs.activations(5, 512, seed=7).numpy()
    w = inputs.weights(24, 512, seed=8).numpy()
    for bits in (6, 8):
        r = orc.linear_layer(x, w, gs, bits)
        brute = orc.dequantize(r["qa"], r["sa"], gs) @ orc.dequantize(r["qw"], r["sw"], gs).T
        assert np.allclose(r["y64"], brute, rtol=1e-12, atol=1e-12 * np.abs(brute).max())
        # a transposed scale or a wrong group index would not survive this
        wrong = orc.rescale_fp64(r["P"], r["sa"][:, ::-1].copy(), r["sw"])
        if (r["sa"][:, ::-1] != r["sa"]).any():
            assert not np.allclose(wrong, brute, rtol=1e-6)


def test_one_group_unit_scales_is_integer_matmul():
    rng = np.random.default_rng(4)
    M, N, K = 6, 10, 256
    qa = rng.integers(-127, 128, (M, K)).astype(np.int8)
    qw = rng.integers(-32, 32, (N, K)).astype(np.int8)
    ones_a = np.ones((M, 1), dtype=np.float16)
    ones_w = np.ones((N, 1), dtype=np.float16)
    y = orc.gemm_fp64(qa, ones_a, qw, ones_w, K)
    exact = np.array([[sum(int(a) * int(b) for a, b in zip(qa[m], qw[n]))
                       for n in range(N)] for m in range(M)], dtype=np.float64)
    assert np.array_equal(y, exact)
    # |y| <= 256*127*32 < 2^24: the FP16 output is the RNE of the integer
    y16 = orc.to_fp16(y)
    for v, h in zip(exact.ravel(), y16.ravel()):
        assert Fraction(float(h)) == exact_fp16_rne(Fraction(int(v)))


def test_fp16_output_and_error_measure():
    y = np.array([[1.0, -2.0], [0.5, 4.0]])
    assert orc.rel_err_vs_max(y, y) == 0
    assert orc.rel_err_vs_max(y + np.array([[0, 0], [0, 0.004]]), y) == pytest.approx(1e-3)
    assert orc.to_fp16(np.array([1 + 2.0 ** -11]))[0] == np.float16(1.0)


def test_partial_bound_assertion():
    qa = np.full((1, 256), -128, dtype=np.int8)
    qw = np.full((1, 256), -32, dtype=np.int8)
    P = orc.group_partials(qa, qw, 256)
    assert P[0, 0, 0] == 256 * 128 * 32
