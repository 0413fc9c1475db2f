"""CPU oracle for FlexQ's group-quantized W6A6 / W6A8 linear layer.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this module:
only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may call it.  It shares no code, table or constant generator with
the CUDA library; it is a slow, literal restatement of what the method
computes, written so that each step can be checked against the method's
description by eye.

What the method computes (FlexQ: Efficient Post-training INT6 Quantization
for LLM Serving via Algorithm-System Co-Design):

* Weights are quantized uniformly to 6 bits in every layer (arXiv abstract);
  activations to 6 bits, or to 8 bits in sensitive layers (abstract; drgamma
  blog, "Fine-Grained Quantization and Layer Sensitivity").
* Both operands use fine-grained group quantization: values are split into
  small groups that share one scale (blog, "Fine-Grained Quantization and
  Layer Sensitivity"), and the groups run along the K dimension (blog,
  "Bridging Software and Hardware with BTC").
* The product is a sum of integer products that is recombined with the
  scales, with dequantization fused into the GEMM (blog, "Bridging Software
  and Hardware with BTC").  Per K-group g this is the exact integer partial
  P_g[m, n] = sum_{k in g} qa[m, k] * qw[n, k], and the output is
  Y[m, n] = sum_g P_g[m, n] * sa[m, g] * sw[n, g].

Readings where the pages are silent (each listed in the design notes):

* symmetric codes, no zero point; code range [-Q, Q] with Q = 31 for 6 bits
  and Q = 127 for 8 bits, scale = absmax / Q;
* the scale is computed in FP32 (IEEE division), stored as FP16
  (round-to-nearest-even), and the codes divide by the *stored* FP16 scale
  (IEEE FP32 division), round half to even, then clamp to [-Q, Q];
* a group whose FP16 scale is zero (all-zero, or underflowing) has scale 0
  and all codes 0;
* the 6-bit weight container packs 4 codes into 3 bytes, little endian,
  code i in bits [6i, 6i+6) as 6-bit two's complement ("canonical form");
  the device form keeps 4 codes per 3 bytes but places twelve of every
  sixteen codes byte-aligned (``pack_block_words``) and tiles the rows into
  128 x 128-code tiles (``pack_device_form``);
* Y is formed in FP64 from the exact integer partials and the exact FP16
  scales, then rounded once to FP16 (round-to-nearest-even).

The FP16 codec is numpy's float16 conversion (a library primitive); the tests
pin it against torch's independent converter and against the round-to-
nearest-even definition at every midpoint between adjacent FP16 values.
"""

import numpy as np

Q_WEIGHT = 31
Q_ACT = {6: 31, 8: 127}


# --------------------------------------------------------------------------
# group quantization (weights: rows = output channels n; activations: rows =
# tokens m; groups of ``gs`` consecutive k within a row)
# --------------------------------------------------------------------------
def quantize_groups(x16, gs, qmax):
    """Symmetric per-group quantization of an FP16 matrix.

    x16  : float16 array [R, K]; K % gs == 0; all values finite.
    gs   : group size along K.
    qmax : largest code magnitude Q (31 for 6-bit, 127 for 8-bit).
    Returns (codes int8 [R, K], scales float16 [R, K // gs]).

    Per group: amax = max |x| (exact in FP32); s = fp16_rne(amax / Q) with an
    IEEE FP32 division; code = clamp(rint_half_even(x / s), -Q, Q) with an IEEE
    FP32 division by the stored FP16 scale; a zero scale gives zero codes.
    """
    x16 = np.asarray(x16, dtype=np.float16)
    R, K = x16.shape
    assert K % gs == 0, "K must be a multiple of the group size"
    G = K // gs
    x32 = x16.astype(np.float32).reshape(R, G, gs)          # exact widening
    assert np.all(np.isfinite(x32)), "non-finite inputs are out of contract"
    amax = np.abs(x32).max(axis=2)                           # exact
    s32 = amax / np.float32(qmax)                            # IEEE fp32 divide
    assert s32.dtype == np.float32
    s16 = s32.astype(np.float16)                             # RNE to fp16
    s16_as_f32 = s16.astype(np.float32)                      # exact widening
    zero = s16_as_f32 == 0
    safe = np.where(zero, np.float32(1), s16_as_f32)
    ratio = x32 / safe[:, :, None]                           # IEEE fp32 divide
    assert ratio.dtype == np.float32
    q = np.rint(ratio)                                       # half to even
    q = np.clip(q, -qmax, qmax)
    q = np.where(zero[:, :, None], np.float32(0), q)
    return q.astype(np.int8).reshape(R, K), s16


def quantize_weight(w16, gs):
    """6-bit weight quantization: codes in [-31, 31], FP16 scales [N, K/gs]."""
    return quantize_groups(w16, gs, Q_WEIGHT)


def quantize_act(x16, gs, bits):
    """6- or 8-bit activation quantization: codes in [-Q, Q], scales [M, K/gs]."""
    return quantize_groups(x16, gs, Q_ACT[bits])


def dequantize(codes, scales, gs):
    """codes * scale per group, in FP64 (exact: code and FP16 scale products
    need at most 18 significant bits)."""
    R, K = codes.shape
    s = np.repeat(scales.astype(np.float64), gs, axis=1)
    return codes.astype(np.float64) * s


# --------------------------------------------------------------------------
# 6-bit container: canonical packing (4 codes -> 3 bytes)
# --------------------------------------------------------------------------
def pack_canonical(codes):
    """Pack int8 codes in [-32, 31] of shape [N, K] (K % 4 == 0) into uint8
    [N, 3K/4].  For codes c0..c3 at k = 4j..4j+3 with u_i = c_i & 0x3F, the
    24-bit word u0 | u1<<6 | u2<<12 | u3<<18 is stored little endian at bytes
    3j, 3j+1, 3j+2."""
    codes = np.asarray(codes)
    N, K = codes.shape
    assert K % 4 == 0
    assert codes.min(initial=0) >= -32 and codes.max(initial=0) <= 31
    u = (codes.astype(np.int32) & 0x3F).astype(np.uint32).reshape(N, K // 4, 4)
    word = u[..., 0] | (u[..., 1] << 6) | (u[..., 2] << 12) | (u[..., 3] << 18)
    out = np.empty((N, K // 4, 3), dtype=np.uint8)
    out[..., 0] = word & 0xFF
    out[..., 1] = (word >> 8) & 0xFF
    out[..., 2] = (word >> 16) & 0xFF
    return out.reshape(N, 3 * K // 4)


def unpack_canonical(packed, K):
    """Inverse of pack_canonical: uint8 [N, 3K/4] -> int8 codes [N, K]."""
    packed = np.asarray(packed, dtype=np.uint8)
    N = packed.shape[0]
    b = packed.reshape(N, K // 4, 3).astype(np.uint32)
    word = b[..., 0] | (b[..., 1] << 8) | (b[..., 2] << 16)
    fields = np.stack([(word >> (6 * i)) & 0x3F for i in range(4)], axis=-1)
    signed = fields.astype(np.int32) - 64 * (fields >= 32)
    return signed.reshape(N, K).astype(np.int8)


# --------------------------------------------------------------------------
# device form: the 6-bit codes of 16 consecutive k in 12 bytes, laid out so
# that twelve codes sit byte-aligned; rows tiled into 128 x 128-code tiles
# --------------------------------------------------------------------------
TILE_ROWS = 128          # weight rows per tile
TILE_K = 128             # codes per row per tile (96 packed bytes)
CHUNK = 16               # bytes per chunk; 6 chunks per row per tile
BLOCK = 16               # codes per 12-byte block


def pack_block_words(codes16):
    """The three 32-bit words of one 16-code block.

    codes16: int array [..., 16] of 6-bit codes in [-32, 31]; u_j = c_j & 63.
    For word i in {0, 1, 2} and byte t in {0, 1, 2, 3}:
      bits [8t+2, 8t+8) hold u_{4i+t}                (twelve aligned codes),
      bits [8t,   8t+2) hold bits [2i, 2i+2) of u_{12+t} (the four codes
                                                     12..15, two bits per word).
    Four codes per three bytes, every field two's complement.
    """
    c = np.asarray(codes16)
    assert c.shape[-1] == BLOCK
    assert c.min(initial=0) >= -32 and c.max(initial=0) <= 31
    u = (c.astype(np.int64) & 0x3F).astype(np.uint64)
    words = np.zeros(c.shape[:-1] + (3,), dtype=np.uint64)
    for i in range(3):
        for t in range(4):
            aligned = u[..., 4 * i + t] << np.uint64(8 * t + 2)
            spread = ((u[..., 12 + t] >> np.uint64(2 * i)) & np.uint64(3)) << np.uint64(8 * t)
            words[..., i] |= aligned | spread
    return words.astype(np.uint32)


def unpack_block_words(words):
    """Inverse of pack_block_words: uint32 [..., 3] -> int8 codes [..., 16]."""
    w = np.asarray(words).astype(np.uint64)
    assert w.shape[-1] == 3
    u = np.zeros(w.shape[:-1] + (BLOCK,), dtype=np.int64)
    for i in range(3):
        for t in range(4):
            u[..., 4 * i + t] = (w[..., i] >> np.uint64(8 * t + 2)) & np.uint64(0x3F)
            piece = (w[..., i] >> np.uint64(8 * t)) & np.uint64(3)
            u[..., 12 + t] |= (piece << np.uint64(2 * i)).astype(np.int64)
    signed = u - 64 * (u >= 32)
    return signed.astype(np.int8)


def pack_device_form(codes):
    """6-bit codes [N, K] (N % 128 == 0, K % 128 == 0) -> device-form bytes.

    Each row is cut into 16-code blocks, block b of row n becoming the 12
    little-endian bytes of pack_block_words(codes[n, 16b:16b+16]); a row's 128
    codes of K-block kb are its 96 bytes kb*96 .. kb*96+95.  Those 96 bytes are
    cut into six 16-byte chunks and tiled: tile (nt, kb) (rows nt*128 ..
    nt*128+127, codes kb*128 .. kb*128+127) is 12288 contiguous bytes at
    offset (nt*(K/128) + kb) * 12288, and byte b of chunk j of row r sits at
    offset (j*128 + r)*16 + b inside the tile.
    """
    codes = np.asarray(codes)
    N, K = codes.shape
    assert N % TILE_ROWS == 0 and K % TILE_K == 0
    words = pack_block_words(codes.reshape(N, K // BLOCK, BLOCK))      # [N, K/16, 3]
    row_bytes = words.astype("<u4").view(np.uint8).reshape(N, 3 * K // 4)
    NT, KB = N // TILE_ROWS, K // TILE_K
    v = row_bytes.reshape(NT, TILE_ROWS, KB, 6, CHUNK)
    return np.ascontiguousarray(v.transpose(0, 2, 3, 1, 4)).reshape(-1)


def unpack_device_form(dev, N, K):
    """Inverse of pack_device_form: device-form bytes -> int8 codes [N, K]."""
    NT, KB = N // TILE_ROWS, K // TILE_K
    v = np.asarray(dev, dtype=np.uint8).reshape(NT, KB, 6, TILE_ROWS, CHUNK)
    row_bytes = np.ascontiguousarray(v.transpose(0, 3, 1, 2, 4)).reshape(N, 3 * K // 4)
    words = row_bytes.view("<u4").reshape(N, K // BLOCK, 3)
    return unpack_block_words(words).reshape(N, K)


# --------------------------------------------------------------------------
# the "4+2" bit-plane form (after the split storage of 6-bit values into a
# 4-bit and a 2-bit part, ZeroQuant(4+2) abstract): each code's top four
# bits go to a 4-bit plane, its low two bits to a 2-bit plane
# --------------------------------------------------------------------------
def pack_planes42(codes16):
    """The 4-bit and the 2-bit plane of one 16-code block.

    codes16: int array [..., 16] of 6-bit codes in [-32, 31]; u_j = c_j & 63,
    h_j = u_j >> 2 (bits 5:2), l_j = u_j & 3 (bits 1:0).
    4-bit plane, 8 bytes: byte t (t = 0..3) holds h_t in its high nibble and
      h_{4+t} in its low nibble; byte 4+t holds h_{8+t} high, h_{12+t} low.
    2-bit plane, 4 bytes: byte t holds l_t in bits 1:0, l_{4+t} in bits 3:2,
      l_{8+t} in bits 5:4 and l_{12+t} in bits 7:6.
    Returns (nibble bytes uint8 [..., 8], two-bit bytes uint8 [..., 4]).
    """
    c = np.asarray(codes16)
    assert c.shape[-1] == BLOCK
    assert c.min(initial=0) >= -32 and c.max(initial=0) <= 31
    u = c.astype(np.int64) & 0x3F
    h, l = u >> 2, u & 3
    nib = np.zeros(c.shape[:-1] + (8,), dtype=np.int64)
    two = np.zeros(c.shape[:-1] + (4,), dtype=np.int64)
    for t in range(4):
        nib[..., t] = (h[..., t] << 4) | h[..., 4 + t]
        nib[..., 4 + t] = (h[..., 8 + t] << 4) | h[..., 12 + t]
        two[..., t] = l[..., t] | (l[..., 4 + t] << 2) | (l[..., 8 + t] << 4) | (l[..., 12 + t] << 6)
    return nib.astype(np.uint8), two.astype(np.uint8)


def unpack_planes42(nib, two):
    """Inverse of pack_planes42: (uint8 [..., 8], uint8 [..., 4]) -> int8 [..., 16]."""
    nib = np.asarray(nib).astype(np.int64)
    two = np.asarray(two).astype(np.int64)
    u = np.zeros(nib.shape[:-1] + (BLOCK,), dtype=np.int64)
    for t in range(4):
        u[..., t] = ((nib[..., t] >> 4) << 2) | (two[..., t] & 3)
        u[..., 4 + t] = ((nib[..., t] & 15) << 2) | ((two[..., t] >> 2) & 3)
        u[..., 8 + t] = ((nib[..., 4 + t] >> 4) << 2) | ((two[..., t] >> 4) & 3)
        u[..., 12 + t] = ((nib[..., 4 + t] & 15) << 2) | ((two[..., t] >> 6) & 3)
    return (u - 64 * (u >= 32)).astype(np.int8)


def pack_device_form42(codes):
    """6-bit codes [N, K] (N % 128 == 0, K % 128 == 0) -> "4+2" device bytes.

    Tiles as in pack_device_form: tile (nt, kb) (rows nt*128 .. nt*128+127,
    codes kb*128 .. kb*128+127) is 12288 contiguous bytes at offset
    (nt*(K/128) + kb) * 12288.  Inside a tile the 4-bit plane comes first:
    byte b of 16-byte chunk j (j = 0..3) of row r at (j*128 + r)*16 + b, where
    a row's 64 nibble bytes are its eight blocks' 8-byte nibble planes in
    order; then the 2-bit plane: chunk 4 + j (j = 0, 1) holds the row's 32
    two-bit bytes, the eight blocks' 4-byte planes in order.  Each plane is a
    contiguous, 16-byte aligned 8192- (4-bit) or 4096-byte (2-bit) region of
    the tile.
    """
    codes = np.asarray(codes)
    N, K = codes.shape
    assert N % TILE_ROWS == 0 and K % TILE_K == 0
    nib, two = pack_planes42(codes.reshape(N, K // BLOCK, BLOCK))      # [N, K/16, 8|4]
    NT, KB = N // TILE_ROWS, K // TILE_K
    nib_rows = nib.reshape(NT, TILE_ROWS, KB, 4, CHUNK)                # 64 B per row and tile
    two_rows = two.reshape(NT, TILE_ROWS, KB, 2, CHUNK)                # 32 B per row and tile
    chunks = np.concatenate([nib_rows, two_rows], axis=3)              # [NT, 128, KB, 6, 16]
    return np.ascontiguousarray(chunks.transpose(0, 2, 3, 1, 4)).reshape(-1)


def unpack_device_form42(dev, N, K):
    """Inverse of pack_device_form42: "4+2" device bytes -> int8 codes [N, K]."""
    NT, KB = N // TILE_ROWS, K // TILE_K
    v = np.asarray(dev, dtype=np.uint8).reshape(NT, KB, 6, TILE_ROWS, CHUNK)
    rows = np.ascontiguousarray(v.transpose(0, 3, 1, 2, 4))            # [NT, 128, KB, 6, 16]
    nib = rows[:, :, :, :4, :].reshape(N, K // BLOCK, 8)
    two = rows[:, :, :, 4:, :].reshape(N, K // BLOCK, 4)
    return unpack_planes42(nib, two).reshape(N, K)


# --------------------------------------------------------------------------
# the GEMM: exact per-group integer partials, FP64 rescale, one FP16 rounding
# --------------------------------------------------------------------------
def group_partials(qa, qw, gs):
    """P[g, m, n] = sum_{k in group g} qa[m, k] * qw[n, k], in int64.

    qa: int codes [M, K]; qw: int codes [N, K].  Asserts that every partial
    fits in int32 (the device accumulates each group exactly in int32)."""
    qa = np.asarray(qa).astype(np.int64)
    qw = np.asarray(qw).astype(np.int64)
    M, K = qa.shape
    N = qw.shape[0]
    assert qw.shape[1] == K and K % gs == 0
    G = K // gs
    P = np.empty((G, M, N), dtype=np.int64)
    for g in range(G):
        ks = slice(g * gs, (g + 1) * gs)
        P[g] = qa[:, ks] @ qw[:, ks].T
    assert np.abs(P).max(initial=0) < 2**31
    return P


def rescale_fp64(P, sa, sw):
    """Y64[m, n] = sum_g P[g, m, n] * sa[m, g] * sw[n, g] in FP64.

    For codes the quantizers produce (|P| < 2^21) each term is exact in FP64
    (P times two 11-bit FP16 significands); only the sum over groups rounds,
    at FP64 precision."""
    G, M, N = P.shape
    sa64 = np.asarray(sa).astype(np.float64)    # [M, G], exact widening
    sw64 = np.asarray(sw).astype(np.float64)    # [N, G]
    Y = np.zeros((M, N), dtype=np.float64)
    for g in range(G):
        Y += P[g].astype(np.float64) * sa64[:, g][:, None] * sw64[:, g][None, :]
    return Y


def gemm_fp64(qa, sa, qw, sw, gs):
    """Y64 for codes + scales of both operands."""
    return rescale_fp64(group_partials(qa, qw, gs), sa, sw)


def to_fp16(y64):
    """Round FP64 values once to FP16 (round to nearest even, overflow to inf)."""
    return np.asarray(y64, dtype=np.float64).astype(np.float16)


def linear_layer(x16, w16, gs, act_bits):
    """The whole layer on FP16 inputs: quantize both operands, form Y64 and
    its FP16 rounding.  Returns a dict of every intermediate."""
    qw, sw = quantize_weight(w16, gs)
    qa, sa = quantize_act(x16, gs, act_bits)
    P = group_partials(qa, qw, gs)
    y64 = rescale_fp64(P, sa, sw)
    return {"qw": qw, "sw": sw, "qa": qa, "sa": sa, "P": P, "y64": y64,
            "y16": to_fp16(y64)}


def rel_err_vs_max(y_test, y_ref):
    """max |y_test - y_ref| / max |y_ref| (the output tolerance measure)."""
    y_test = np.asarray(y_test, dtype=np.float64)
    y_ref = np.asarray(y_ref, dtype=np.float64)
    denom = np.abs(y_ref).max(initial=0.0)
    diff = np.abs(y_test - y_ref).max(initial=0.0)
    return diff / denom if denom > 0 else diff
