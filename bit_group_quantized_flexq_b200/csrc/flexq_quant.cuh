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

// One code, given the group's stored scale as FP32 (0 for a zero scale).
__device__ __forceinline__ int quant_code(float x, float s, int qmax) {
  if (s == 0.0f) return 0;
  int q = __float2int_rn(__fdiv_rn(x, s));
  return max(-qmax, min(qmax, q));
}

// --------------------------------------------------------------------------
// Activation quantization: each thread owns 8 consecutive values (one 16-byte
// load); a group is gs/8 consecutive lanes (4..32), reduced with shuffles.
// --------------------------------------------------------------------------
template <int GS>
__global__ void __launch_bounds__(256) quant_act_kernel(
    const uint4* __restrict__ X, uint2* __restrict__ Xq, __half* __restrict__ Xs,
    long long chunks, int chunks_per_row, int ld_scales, int qmax) {
  constexpr int LANES = GS / 8;            // lanes per group
  static_assert(LANES >= 4 && LANES <= 32, "group size 32..256");
  // X may be the output of the previous kernel of the stream, and Xq / Xs
  // may still be read by it: wait for it before touching either
  grid_launch_dependents();
  grid_wait_dependencies();
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  const long long first = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  // every lane of a warp runs the same number of iterations (the stride and
  // the start are warp-aligned), so the shuffles below are always full-warp
  const long long base_iters = (chunks + stride - 1) / stride;
  const float fq = static_cast<float>(qmax);
  for (long long it = 0; it < base_iters; ++it) {
    const long long idx = first + it * stride;
    const bool valid = idx < chunks;
    uint4 raw = make_uint4(0, 0, 0, 0);
    if (valid) raw = __ldg(X + idx);
    const __half2* h2 = reinterpret_cast<const __half2*>(&raw);
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
    const __half s16 = group_scale(amax, fq);
    const float s = __half2float(s16);
    uint32_t lo = 0, hi = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      lo |= (static_cast<uint32_t>(quant_code(v[i], s, qmax)) & 0xFFu) << (8 * i);
      hi |= (static_cast<uint32_t>(quant_code(v[4 + i], s, qmax)) & 0xFFu) << (8 * i);
    }
    if (valid) {
      Xq[idx] = make_uint2(lo, hi);
      const long long row = idx / chunks_per_row;
      const int c = static_cast<int>(idx - row * chunks_per_row);
      if ((c % LANES) == 0) Xs[static_cast<long long>(c / LANES) * ld_scales + row] = s16;
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
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 f = __half22float2(h2[i]);
        u[8 * c + 2 * i] = static_cast<uint32_t>(quant_code(f.x, s, 31)) & 0x3Fu;
        u[8 * c + 2 * i + 1] = static_cast<uint32_t>(quant_code(f.y, s, 31)) & 0x3Fu;
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

}  // namespace flexq
