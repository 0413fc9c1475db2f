// tcgen05.mma.kind::i8 128x128x32 (A in TMEM) issue patterns, one thread per CTA, 148 CTAs.
#include <cstdio>
#include <cstdint>
#include <cuda_runtime.h>
#include "../csrc/flexq_ptx.cuh"
using namespace flexq;

// mode 0: groups of 4 MMAs into one D, straight-line unrolled 32 MMAs per outer iteration
// mode 1: groups of 4 MMAs, D rotating over 3 buffers, commit per group, no branch between groups
// mode 2: as 1 with a non-blocking barrier probe (always complete) + branch before each group
// mode 3: as 1 but no commit
// mode 4: N = 256, one D of 256 columns at column 0 (A at column 384, clear of it)
__global__ void __launch_bounds__(128, 1) mma_kernel(int mode, int groups, long long* cyc) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  __shared__ uint64_t bar, done_bar, probe;
  __shared__ uint32_t tbase;
  const int warp = threadIdx.x >> 5;
  for (int i = threadIdx.x; i < 65536 / 4; i += 128) reinterpret_cast<uint32_t*>(base)[i] = 0;
  if (threadIdx.x == 0) { mbar_init(&bar, 1); mbar_init(&done_bar, 1); mbar_init(&probe, 1); fence_barrier_init(); }
  if (warp == 0) tmem_alloc(&tbase, 512);
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) mbar_arrive(&probe);   // phase 0 of `probe` completes
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = tbase;
  if (threadIdx.x == 32) {
    const uint32_t b_s = smem_u32(base + 16384);
    const uint64_t bd = smem_desc_k_sw128(b_s);
    const uint32_t idesc = idesc_i8(128, mode == 4 ? 256 : 128);
    const long long t0 = clock64();
    uint32_t pb = 0;
    for (int g = 0; g < groups; ++g) {
      if (mode == 2) {
        if (!mbar_test_wait(smem_u32(&probe), 0)) { cyc[blockIdx.x] = -2; }
        tc_fence_after();
      }
      const uint32_t d = tm + (mode == 0 || mode == 4 ? 0u : pb * 128u);
      const uint32_t a = tm + 384;
#pragma unroll
      for (int k = 0; k < 4; ++k) mma_i8_tmem_a(d, a + k * 8, bd + ((k * 32) >> 4), idesc, 1u);
      if (mode == 1 || mode == 2) mma_commit(&bar);
      pb = (pb == 2) ? 0 : pb + 1;
    }
    mma_commit(&done_bar);
    const bool ok = mbar_wait(&done_bar, 0, 2000000000ull);
    const long long t1 = clock64();
    if (cyc[blockIdx.x] != -2) cyc[blockIdx.x] = ok ? (t1 - t0) : -1;
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) { tc_fence_after(); tmem_dealloc(tm, 512); }
}

int main() {
  long long* cyc;
  cudaMalloc(&cyc, 148 * sizeof(long long));
  cudaFuncSetAttribute(mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 150 * 1024);
  const char* names[] = {"4/group, same D, no commit", "4/group, 3 D rotating, commit",
                         "probe+branch, 3 D, commit", "3 D rotating, no commit", "N=256 same D"};
  const int groups = 512;
  for (int mode = 0; mode < 5; ++mode) {
    cudaMemset(cyc, 0, 148 * sizeof(long long));
    mma_kernel<<<148, 128, 150 * 1024>>>(mode, groups, cyc);
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) { printf("error %s\n", cudaGetErrorString(e)); return 1; }
    long long h[148];
    cudaMemcpy(h, cyc, sizeof(h), cudaMemcpyDeviceToHost);
    long long mx = 0, mn = 1ll << 60;
    for (int b = 0; b < 148; ++b) { mx = mx > h[b] ? mx : h[b]; mn = mn < h[b] ? mn : h[b]; }
    const int n = (mode == 4) ? 256 : 128;
    printf("%-30s cycles/MMA=%6.1f  MAC/clk/SM=%6.0f  (min %lld)\n", names[mode], (double)mx / (groups * 4),
           128.0 * n * 32 * groups * 4 / mx, mn);
  }
  return 0;
}
