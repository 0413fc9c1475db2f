// flexq_quant.cuh -- group quantization kernels.
//
// FlexQ quantizes weights to 6 bits and activations to 6 or 8 bits with
// fine-grained groups along K that share one scale (FlexQ paper, arXiv
// abstract; drgamma blog, "Fine-Grained Quantization and Layer Sensitivity").
// Scale rule: s = fp16_rne(absmax / Q) with an IEEE FP32 division; codes =
// clamp(round_half_even(x / s), -Q, Q) with an IEEE FP32 division by the
// stored FP16 scale; a zero FP16 scale gives zero codes.
//
// Scales are stored group-major (scale of row r, group g at g * ld + r) so
// that the GEMM can fetch eight groups of a tile's scales with one TMA box.
#pragma once

#include <cuda_fp16.h>
#include <cstdint>

#include "flexq_ptx.cuh"

namespace flexq {

// Scale of a group from its absolute maximum.
__device__ __forceinline__ __half group_scale(float amax, float qmax) {
  return __float2half_rn(__fdiv_rn(amax, qmax));
}

// One code by the defining route: IEEE FP32 division by the stored scale,
// round half to even, clamp (0 for a zero scale).
__device__ __forceinline__ int quant_code_div(float x, float s, int qmax) {
  if (s == 0.0f) return 0;
  int q = __float2int_rn(__fdiv_rn(x, s));
  return max(-qmax, min(qmax, q));
}

// The same code without a division, for FP16 x and FP16 s > 0 (passed as
// FP32) and rs ~ 1/s.  Both are multiples of a power of two with at most 11
// significant bits, so a quotient x/s that is not a half-integer lies at
// least 2^-12 away from every half-integer, further than half an FP32 ulp at
// the magnitudes a code can have (< 2^8): rounding the FP32 quotient to an
// integer (half to even) therefore equals rounding the exact quotient.  The
// estimate k0 = rint(x * rs) can only miss it at such a tie, by one.  The
// residual r = x - k0 * s is exact (k0 * s has at most 19 significant bits
// and lies within a factor 2 of x unless k0 = 0, where r = x), so comparing
// |r| with s/2 decides exactly: beyond it, step towards r; at it (a tie),
// step only if k0 is odd.
__device__ __forceinline__ int quant_code_fast(float x, float s, float rs, int qmax) {
  // estimates beyond +-(Q+2) only feed the clamp; bounding them keeps the
  // integer arithmetic far from overflow
  const float qb = static_cast<float>(qmax + 2);
  const float k0 = fminf(fmaxf(rintf(x * rs), -qb), qb);
  const float r = fmaf(-k0, s, x);
  const float h = 0.5f * s;
  const float ar = fabsf(r);
  const int k = static_cast<int>(k0);
  const bool step = ar > h || (ar == h && (k & 1));
  const int q = step ? (r > 0.0f ? k + 1 : k - 1) : k;
  return max(-qmax, min(qmax, q));
}

// One code, given the group's stored scale as FP32 (0 for a zero scale) and
// its reciprocal estimate.
__device__ __forceinline__ int quant_code(float x, float s, float rs, int qmax) {
  return s == 0.0f ? 0 : quant_code_fast(x, s, rs, qmax);
}

// ---- the route the quantizers take (division-free, no conversion unit) ----
// s32 = RN(a / Q) for a finite FP16 value a >= 0 and Q in {31, 127}, given
// rq = RN(1 / Q): the estimate q0 = RN(a * rq) is corrected once by its
// exact residual a - q0 * Q (q0 has 24 significant bits, Q at most 7, and
// the residual is far below a).  The result equals the IEEE division for
// every FP16 a and both Q (flexq_debug_check_quantizer checks all of them).
__device__ __forceinline__ float div_by_q(float a, float fq, float rq) {
  const float q0 = __fmul_rn(a, rq);
  const float r = __fmaf_rn(-q0, fq, a);
  return __fmaf_rn(r, rq, q0);
}

__device__ __forceinline__ __half group_scale_fast(float amax, float fq, float rq) {
  return __float2half_rn(div_by_q(amax, fq, rq));
}

// Reciprocal estimate of a positive FP32 value converted from FP16 (a normal
// FP32 number): one approximate reciprocal, within about one ulp.  Both code
// routes only need x * rs to land within 2^-14 of x / s (quant_code_fast).
__device__ __forceinline__ float rcp_estimate(float s) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(s));
  return r;
}

// Common route for one value whose group has a normal FP16 scale s, so that
// |x / s| < Q + 1/2 (the stored scale is within 2^-11 of amax / Q): with
// t = RN(x * rs + 1.5 * 2^23), the low mantissa bits of t hold the integer
// k = rint(x * rs), so the low byte of t's bit pattern is k's two's
// complement byte.  k equals round_half_even(x / s) unless x / s is exactly a
// half-integer, which shows as an exact residual |x - k * s| = s / 2 and is
// flagged in `tie` for the full rule.  No clamp is needed below Q + 1/2.
constexpr float kRoundMagic = 12582912.0f;            // 1.5 * 2^23

__device__ __forceinline__ uint32_t code_bits_common(float x, float s, float rs, float half_s,
                                                     bool& tie) {
  const float t = __fmaf_rn(x, rs, kRoundMagic);
  const float k = __fsub_rn(t, kRoundMagic);
  tie |= fabsf(__fmaf_rn(-k, s, x)) == half_s;
  return __float_as_uint(t);
}

// Eight consecutive values of one group -> their codes' low bytes in order,
// packed in two words.  Values whose group scale is subnormal or zero, and
// groups of this lane that meet a tie, take the full rule (quant_code).
__device__ __forceinline__ uint2 quantize8(const float (&v)[8], float sc, float rs, int qmax) {
  const float half_s = 0.5f * sc;
  bool exact = !(sc >= 6.103515625e-05f);             // subnormal or zero scale
  uint32_t b[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) b[i] = code_bits_common(v[i], sc, rs, half_s, exact);
  if (exact) {
#pragma unroll
    for (int i = 0; i < 8; ++i) b[i] = static_cast<uint32_t>(quant_code(v[i], sc, rs, qmax));
  }
  const uint32_t lo = __byte_perm(__byte_perm(b[0], b[1], 0x0040), __byte_perm(b[2], b[3], 0x0040), 0x5410);
  const uint32_t hi = __byte_perm(__byte_perm(b[4], b[5], 0x0040), __byte_perm(b[6], b[7], 0x0040), 0x5410);
  return make_uint2(lo, hi);
}

// --------------------------------------------------------------------------
// Activation quantization: each thread owns 8 consecutive values (one 16-byte
// load); a group is gs/8 consecutive lanes (4..32), reduced with shuffles.
// --------------------------------------------------------------------------
template <int GS>
__global__ void __launch_bounds__(256) quant_act_kernel(
    const uint4* __restrict__ X, uint2* __restrict__ Xq, __half* __restrict__ Xs,
    int M, int chunks_per_row, int rows_per_step, int ld_scales, int qmax) {
  constexpr int LANES = GS / 8;            // lanes per group
  constexpr int U = 4;                     // independent 16-byte loads in flight per thread
  static_assert(LANES >= 4 && LANES <= 32, "group size 32..256");
  // X may be the output of the previous kernel of the stream, and Xq / Xs
  // may still be read by it: wait for it before touching either
  grid_launch_dependents();
  grid_wait_dependencies();
  // The grid covers rows_per_step whole rows per step (its thread count is a
  // multiple of the row length in chunks), so each thread keeps one column c
  // and advances by rows_per_step rows; a warp never straddles two rows in a
  // way that splits a group, and every lane of a warp runs the same steps,
  // so the shuffles below are always full-warp.
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  const int c = t % chunks_per_row;
  const int row0 = t / chunks_per_row;
  const float fq = static_cast<float>(qmax);
  const float rq = __frcp_rn(fq);
  const int steps = (M + rows_per_step - 1) / rows_per_step;
  for (int st0 = 0; st0 < steps; st0 += U) {
    uint4 raw[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int row = row0 + (st0 + u) * rows_per_step;
      raw[u] = make_uint4(0, 0, 0, 0);
      if (st0 + u < steps && row < M)
        raw[u] = __ldg(X + static_cast<long long>(row) * chunks_per_row + c);
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      if (st0 + u >= steps) break;           // uniform across the grid
      const int row = row0 + (st0 + u) * rows_per_step;
      const __half2* h2 = reinterpret_cast<const __half2*>(&raw[u]);
      float v[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 f = __half22float2(h2[i]);
        v[2 * i] = f.x;
        v[2 * i + 1] = f.y;
      }
      float amax = 0.0f;
#pragma unroll
      for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(v[i]));
#pragma unroll
      for (int off = 1; off < LANES; off <<= 1)
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
      const __half s16 = group_scale_fast(amax, fq, rq);
      const float sc = __half2float(s16);
      const uint2 codes = quantize8(v, sc, rcp_estimate(sc), qmax);
      if (row < M) {
        Xq[static_cast<long long>(row) * chunks_per_row + c] = codes;
        if ((c % LANES) == 0) Xs[static_cast<long long>(c / LANES) * ld_scales + row] = s16;
      }
    }
  }
}

// --------------------------------------------------------------------------
// Weight quantization, pass 1: one thread per (row n, group g) computes the
// group's FP16 scale, stored at Ws[g * N + n].
// --------------------------------------------------------------------------
__global__ void __launch_bounds__(256) weight_scale_kernel(
    const __half* __restrict__ W, __half* __restrict__ Ws, int N, int K, int gs) {
  const int G = K / gs;
  const long long t = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t >= static_cast<long long>(N) * G) return;
  const int g = static_cast<int>(t / N);
  const int n = static_cast<int>(t - static_cast<long long>(g) * N);
  const uint4* p = reinterpret_cast<const uint4*>(W + static_cast<long long>(n) * K + g * gs);
  float amax = 0.0f;
  for (int c = 0; c < gs / 8; ++c) {
    uint4 raw = __ldg(p + c);
    const __half2* h2 = reinterpret_cast<const __half2*>(&raw);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __half22float2(h2[i]);
      amax = fmaxf(amax, fmaxf(fabsf(f.x), fabsf(f.y)));
    }
  }
  Ws[t] = group_scale(amax, 31.0f);
}

// --------------------------------------------------------------------------
// Device form of the packed weights.  The codes of 16 consecutive k of a row
// form one 12-byte block of three little-endian 32-bit words w0, w1, w2:
// byte t of word i holds the 6-bit code 4i+t in its bits [7:2] and bits
// [2i+1:2i] of code 12+t in its bits [1:0].  Twelve codes are thus already
// in place as int8 values code*4 (w & 0xFCFCFCFC), and the last four are
// gathered from the three 2-bit pieces.  Rows are tiled as 128 rows x 128
// codes (12288 bytes): tile (nt, kb) at (nt*(K/128) + kb) * 12288, and the
// 96 bytes of row r inside it as six 16-byte chunks, chunk j at
// (j*128 + r) * 16.
// --------------------------------------------------------------------------
__device__ __forceinline__ void pack_block(const uint32_t (&u)[16], uint32_t& w0,
                                           uint32_t& w1, uint32_t& w2) {
  uint32_t w[3] = {0u, 0u, 0u};
#pragma unroll
  for (int i = 0; i < 3; ++i)
#pragma unroll
    for (int t = 0; t < 4; ++t)
      w[i] |= (u[4 * i + t] << (8 * t + 2)) | (((u[12 + t] >> (2 * i)) & 3u) << (8 * t));
  w0 = w[0];
  w1 = w[1];
  w2 = w[2];
}

// --------------------------------------------------------------------------
// Weight quantization, pass 2: one thread per (row n, 64-code half of a
// 128-code K-block).  It quantizes 64 values into four 16-code blocks (48
// bytes) and stores them as three 16-byte chunks at their tile positions.
// --------------------------------------------------------------------------
__global__ void __launch_bounds__(256) weight_pack_kernel(
    const __half* __restrict__ W, const __half* __restrict__ Ws,
    uint8_t* __restrict__ Wp, int N, int K, int gs) {
  const int KB = K / 128;
  const long long t = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t >= static_cast<long long>(N) * KB * 2) return;
  const int half_idx = static_cast<int>(t & 1);
  const long long nk = t >> 1;
  const int n = static_cast<int>(nk / KB);
  const int kb = static_cast<int>(nk - static_cast<long long>(n) * KB);
  const int k0 = kb * 128 + half_idx * 64;
  const uint4* p = reinterpret_cast<const uint4*>(W + static_cast<long long>(n) * K + k0);
  uint32_t word[12];
#pragma unroll
  for (int blk = 0; blk < 4; ++blk) {          // 16 codes = two 16-byte loads
    uint32_t u[16];
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      uint4 raw = __ldg(p + 2 * blk + c);
      const __half2* h2 = reinterpret_cast<const __half2*>(&raw);
      const int kk = k0 + 16 * blk + 8 * c;
      const float s = __half2float(Ws[static_cast<long long>(kk / gs) * N + n]);
      const float rs = s == 0.0f ? 0.0f : __frcp_rn(s);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 f = __half22float2(h2[i]);
        u[8 * c + 2 * i] = static_cast<uint32_t>(quant_code(f.x, s, rs, 31)) & 0x3Fu;
        u[8 * c + 2 * i + 1] = static_cast<uint32_t>(quant_code(f.y, s, rs, 31)) & 0x3Fu;
      }
    }
    pack_block(u, word[3 * blk], word[3 * blk + 1], word[3 * blk + 2]);
  }
  const int nt = n >> 7, r = n & 127;
  uint8_t* tile = Wp + (static_cast<long long>(nt) * KB + kb) * 12288;
#pragma unroll
  for (int jj = 0; jj < 3; ++jj) {
    const int j = half_idx * 3 + jj;
    uint4* dst = reinterpret_cast<uint4*>(tile + (j * 128 + r) * 16);
    *dst = make_uint4(word[4 * jj], word[4 * jj + 1], word[4 * jj + 2], word[4 * jj + 3]);
  }
}

// --------------------------------------------------------------------------
// The "4+2" bit-plane form (layout 1): the top four bits h of each 6-bit code
// u go to a 4-bit plane, the low two bits l to a 2-bit plane.  Per 16-code
// block: nibble words N0, N1 (byte t of N0 = h_t << 4 | h_{4+t}, byte t of
// N1 = h_{8+t} << 4 | h_{12+t}) and one 2-bit word L (byte t = l_t |
// l_{4+t} << 2 | l_{8+t} << 4 | l_{12+t} << 6).  Tiles as in the byte-aligned
// form; inside a tile, chunks 0..3 of each row are its nibble plane (block b
// at row bytes 8b..8b+7) and chunks 4, 5 its 2-bit plane (block b at row
// bytes 4b..4b+3): each plane is one contiguous 16-byte aligned region.
// --------------------------------------------------------------------------
__device__ __forceinline__ void pack_block42(const uint32_t (&u)[16], uint32_t& n0, uint32_t& n1,
                                             uint32_t& l) {
  n0 = n1 = l = 0u;
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    n0 |= (((u[t] >> 2) << 4) | (u[4 + t] >> 2)) << (8 * t);
    n1 |= (((u[8 + t] >> 2) << 4) | (u[12 + t] >> 2)) << (8 * t);
    l |= ((u[t] & 3u) | ((u[4 + t] & 3u) << 2) | ((u[8 + t] & 3u) << 4) | ((u[12 + t] & 3u) << 6))
         << (8 * t);
  }
}

// Weight quantization, pass 2 for the "4+2" form: one thread per (row n,
// 64-code half of a 128-code K-block): four blocks, i.e. two 16-byte chunks
// of the nibble plane and one of the 2-bit plane.
__global__ void __launch_bounds__(256) weight_pack42_kernel(
    const __half* __restrict__ W, const __half* __restrict__ Ws,
    uint8_t* __restrict__ Wp, int N, int K, int gs) {
  const int KB = K / 128;
  const long long t = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t >= static_cast<long long>(N) * KB * 2) return;
  const int half_idx = static_cast<int>(t & 1);
  const long long nk = t >> 1;
  const int n = static_cast<int>(nk / KB);
  const int kb = static_cast<int>(nk - static_cast<long long>(n) * KB);
  const int k0 = kb * 128 + half_idx * 64;
  const uint4* p = reinterpret_cast<const uint4*>(W + static_cast<long long>(n) * K + k0);
  uint32_t nib[8], two[4];
#pragma unroll
  for (int blk = 0; blk < 4; ++blk) {
    uint32_t u[16];
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      uint4 raw = __ldg(p + 2 * blk + c);
      const __half2* h2 = reinterpret_cast<const __half2*>(&raw);
      const int kk = k0 + 16 * blk + 8 * c;
      const float s = __half2float(Ws[static_cast<long long>(kk / gs) * N + n]);
      const float rs = s == 0.0f ? 0.0f : __frcp_rn(s);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 f = __half22float2(h2[i]);
        u[8 * c + 2 * i] = static_cast<uint32_t>(quant_code(f.x, s, rs, 31)) & 0x3Fu;
        u[8 * c + 2 * i + 1] = static_cast<uint32_t>(quant_code(f.y, s, rs, 31)) & 0x3Fu;
      }
    }
    pack_block42(u, nib[2 * blk], nib[2 * blk + 1], two[blk]);
  }
  const int nt = n >> 7, r = n & 127;
  uint8_t* tile = Wp + (static_cast<long long>(nt) * KB + kb) * 12288;
#pragma unroll
  for (int jj = 0; jj < 2; ++jj) {              // nibble chunks 2h, 2h + 1
    uint4* dst = reinterpret_cast<uint4*>(tile + ((2 * half_idx + jj) * 128 + r) * 16);
    *dst = make_uint4(nib[4 * jj], nib[4 * jj + 1], nib[4 * jj + 2], nib[4 * jj + 3]);
  }
  uint4* dst = reinterpret_cast<uint4*>(tile + ((4 + half_idx) * 128 + r) * 16);
  *dst = make_uint4(two[0], two[1], two[2], two[3]);
}

// --------------------------------------------------------------------------
// Test hook: for FP16 scale patterns [s_first, s_first + n_s) (positive,
// finite) against every finite FP16 value x, for Q = 31 and Q = 127, counts
// the (x, s) pairs where a route of the quantizers differs from
// quant_code_div: quant_code_fast with either reciprocal, and the common
// route wherever a group can take it (its tie flag must be raised exactly at
// the half-integer quotients); with the first scale pattern, also every
// non-negative FP16 x as a group maximum through group_scale_fast.  Records
// the first mismatch.  One thread per (x, s) pair.
// --------------------------------------------------------------------------
__global__ void __launch_bounds__(256) check_quantizer_kernel(unsigned s_first, unsigned n_s,
                                                              unsigned long long* mismatches,
                                                              unsigned* first) {
  const unsigned long long t = static_cast<unsigned long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t >= static_cast<unsigned long long>(n_s) * 65536ull) return;
  const unsigned xb = static_cast<unsigned>(t & 0xFFFFu);
  const unsigned sb = s_first + static_cast<unsigned>(t >> 16);
  if ((xb & 0x7C00u) == 0x7C00u) return;                      // x infinite or NaN
  const float x = __half2float(__ushort_as_half(static_cast<unsigned short>(xb)));
  const float s = __half2float(__ushort_as_half(static_cast<unsigned short>(sb)));
  const float rs = __frcp_rn(s);
  const float rse = rcp_estimate(s);
  const int qs[2] = {31, 127};
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int want = quant_code_div(x, s, qs[i]);
    // the full rule, with the correctly rounded and with the estimated
    // reciprocal
    bool bad = quant_code_fast(x, s, rs, qs[i]) != want || quant_code_fast(x, s, rse, qs[i]) != want;
    // the common route, wherever a group can use it: a normal scale and
    // |x / s| <= Q + 1/2 (a tie there must be flagged)
    if (s >= 6.103515625e-05f && fabsf(x) <= (static_cast<float>(qs[i]) + 0.5f) * s) {
      bool tie = false;
      const uint32_t t = code_bits_common(x, s, rse, 0.5f * s, tie);
      // (a flagged pair takes the full rule, checked above)
      if (!tie) bad |= static_cast<int>(static_cast<int8_t>(t & 0xFFu)) != want;
    }
    // the scale: every FP16 value as a group's absolute maximum
    if (sb == 1u && !(xb & 0x8000u))
      bad |= __half_as_ushort(group_scale_fast(x, static_cast<float>(qs[i]), __frcp_rn(static_cast<float>(qs[i])))) !=
             __half_as_ushort(group_scale(x, static_cast<float>(qs[i])));
    if (bad) {
      if (atomicAdd(mismatches, 1ull) == 0ull) {
        first[0] = xb;
        first[1] = sb;
        first[2] = static_cast<unsigned>(qs[i]);
      }
    }
  }
}

}  // namespace flexq
