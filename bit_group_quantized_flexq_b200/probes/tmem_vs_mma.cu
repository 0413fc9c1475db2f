// Does epilogue-style TMEM traffic slow the tensor core?  One thread issues groups of 4
// int8 MMAs 128x128x32 (A in TMEM cols 448.., D rotating over cols 0/128/256) while W
// other warps load (and optionally refill) TMEM columns 0..383 in a loop.
#include <cstdio>
#include <cstdint>
#include <cuda_runtime.h>
#include "../csrc/flexq_ptx.cuh"
using namespace flexq;

__global__ void __launch_bounds__(512, 1) k(int mode, int loaders, int groups, long long* cyc, unsigned* sink) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  __shared__ uint64_t done_bar;
  __shared__ uint32_t tbase;
  __shared__ volatile int stop;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < 65536 / 4; i += blockDim.x) reinterpret_cast<uint32_t*>(base)[i] = 0;
  if (threadIdx.x == 0) { mbar_init(&done_bar, 1); fence_barrier_init(); stop = 0; }
  if (warp == 0) tmem_alloc(&tbase, 512);
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = tbase;
  unsigned acc = 0;
  if (threadIdx.x == 0) {
    const uint64_t bd = smem_desc_k_sw128(smem_u32(base + 16384));
    const uint32_t idesc = idesc_i8(128, 128);
    const long long t0 = clock64();
    uint32_t pb = 0;
    for (int g = 0; g < groups; ++g) {
      const uint32_t d = tm + pb * 128u;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) mma_i8_tmem_a(d, tm + 448 + kk * 8, bd + ((kk * 32) >> 4), idesc, 1u);
      pb = (pb == 2) ? 0 : pb + 1;
    }
    mma_commit(&done_bar);
    const bool ok = mbar_wait(&done_bar, 0, 2000000000ull);
    const long long t1 = clock64();
    cyc[blockIdx.x * 2] = ok ? (t1 - t0) : -1;
    stop = 1;
  } else if (warp >= 4 && warp < 4 + loaders) {
    // loader warps: lane quarter (warp & 3), columns cycling over 0..383
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    long long n = 0;
    const long long t0 = clock64();
    uint32_t r[32];
    int c = ((warp - 4) >> 2) * 32;
    for (int it = 0; it < 1000000 && !stop; ++it) {
      const uint32_t a = tm + lane_base + c;
      if (mode == 0 || mode == 1) { tmem_ld32(a, r); tmem_wait_ld(); acc ^= r[0] ^ r[31]; }
      if (mode == 1) { tmem_fill32(a, 0x4B400000u); tmem_wait_st(); }
      if (mode == 2) { tmem_ld_16x256b_x8(a, r); tmem_wait_ld(); acc ^= r[0] ^ r[31]; }
      if (mode == 3) { tmem_ld_16x256b_x8(a, r); tmem_wait_ld(); acc ^= r[0] ^ r[31]; tmem_fill_16x256b_x8(a, 0x4B400000u); tmem_wait_st(); }
      c += 64; if (c >= 384) c -= 384;
      ++n;
    }
    const long long t1 = clock64();
    if (lane == 0 && warp == 4) cyc[blockIdx.x * 2 + 1] = (t1 - t0) / (n ? n : 1);
  }
  if (acc == 0x1234567u) sink[threadIdx.x] = acc;
  tc_fence_before();
  __syncthreads();
  if (warp == 0) { tc_fence_after(); tmem_dealloc(tm, 512); }
}

int main() {
  long long* cyc; unsigned* sink;
  cudaMalloc(&cyc, 296 * sizeof(long long));
  cudaMalloc(&sink, 512 * 4);
  cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, 150 * 1024);
  const char* names[] = {"ld32x32b", "ld32x32b + fill", "ld16x256b", "ld16x256b + fill"};
  const int groups = 1024;
  for (int mode = 0; mode < 4; ++mode)
    for (int loaders : {0, 4, 8}) {
      if (loaders == 0 && mode > 0) continue;
      cudaMemset(cyc, 0, 296 * sizeof(long long));
      k<<<148, 512, 150 * 1024>>>(mode, loaders, groups, cyc, sink);
      cudaError_t e = cudaDeviceSynchronize();
      if (e != cudaSuccess) { printf("error %s\n", cudaGetErrorString(e)); return 1; }
      long long h[296];
      cudaMemcpy(h, cyc, sizeof(h), cudaMemcpyDeviceToHost);
      long long mx = 0; for (int b = 0; b < 148; ++b) mx = mx > h[2 * b] ? mx : h[2 * b];
      printf("%-18s loaders=%d  MMA cycles/MMA=%6.1f  loader cycles/iter=%lld\n", names[mode], loaders,
             (double)mx / (groups * 4), h[1]);
    }
  return 0;
}
