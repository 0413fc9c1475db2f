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
// Weight quantization, pass 2: one thread per (row n, 64-code half of a
// 128-code K-block).  It quantizes 64 values, packs them canonically into 48
// bytes (four 6-bit codes per 24-bit little-endian word) and stores the three
// 16-byte chunks at their device-form positions:
//   tile (n/128, kb) at ((n/128)*(K/128) + kb) * 12288,
//   chunk j of row r inside the tile at (j*128 + r) * 16.
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
  for (int i = 0; i < 12; ++i) word[i] = 0;
#pragma unroll
  for (int c = 0; c < 8; ++c) {               // 8 values per 16-byte load
    uint4 raw = __ldg(p + c);
    const __half2* h2 = reinterpret_cast<const __half2*>(&raw);
    const int kk = k0 + c * 8;
    const float s = __half2float(Ws[static_cast<long long>(kk / gs) * N + n]);
    uint32_t u[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __half22float2(h2[i]);
      u[2 * i] = static_cast<uint32_t>(quant_code(f.x, s, 31)) & 0x3Fu;
      u[2 * i + 1] = static_cast<uint32_t>(quant_code(f.y, s, 31)) & 0x3Fu;
    }
    // two quads -> two 24-bit words -> bytes 6c .. 6c+5 of the 48-byte run
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const uint32_t w24 = u[4 * q] | (u[4 * q + 1] << 6) | (u[4 * q + 2] << 12) |
                           (u[4 * q + 3] << 18);
#pragma unroll
      for (int b = 0; b < 3; ++b) {
        const int pos = 6 * c + 3 * q + b;    // byte position, compile time
        word[pos >> 2] |= ((w24 >> (8 * b)) & 0xFFu) << (8 * (pos & 3));
      }
    }
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
