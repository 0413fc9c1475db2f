// L2 -> SMEM bulk-copy throughput per SM for the GEMM's stage pattern (56 KB per stage:
// 24 KB + 16 KB + 16 KB) with different issue patterns.  One CTA per SM, 3-stage ring,
// a consumer warp that waits for each stage and releases it at once.  Source: a 96 MB
// buffer read in a rotating pattern (mostly L2 hits after the first pass).
#include <cstdio>
#include <cstdint>
#include <cuda_runtime.h>
#include "../csrc/flexq_ptx.cuh"
using namespace flexq;

constexpr int kStages = 3;
constexpr int kStage = 57344;

// mode 0: one thread issues 3 copies per stage (24K, 16K, 16K)
// mode 1: three warps each issue one copy per stage
// mode 2: one thread issues one 56K copy per stage
// mode 3: one thread issues 7 copies of 8K per stage
// mode 4: two CTAs per SM? (not here)
__global__ void __launch_bounds__(128, 1) tma_kernel(const uint8_t* src, size_t src_bytes, int mode,
                                                      int iters, long long* cyc, unsigned* err) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  __shared__ uint64_t full[kStages], empty[kStages];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    fence_barrier_init();
  }
  __syncthreads();
  const uint64_t lim = 2000000000ull;
  const size_t nchunks = src_bytes / kStage;
  long long t0 = clock64();
  if (warp < 3 && lane == 0) {
    bool ok = true;
    for (int i = 0; i < iters && ok; ++i) {
      const int s = i % kStages;
      if (i >= kStages && !mbar_wait(&empty[s], ((i / kStages) - 1) & 1, lim)) { ok = false; break; }
      const uint8_t* g = src + ((blockIdx.x * 131 + i) % nchunks) * kStage;
      uint8_t* d = base + s * kStage;
      if (mode == 1) {
        if (warp == 0) {
          mbar_arrive_expect_tx(&full[s], kStage);
          bulk_load(d, g, 24576, &full[s]);
        } else if (warp == 1) {
          bulk_load(d + 24576, g + 24576, 16384, &full[s]);
        } else {
          bulk_load(d + 40960, g + 40960, 16384, &full[s]);
        }
      } else if (warp == 0) {
        mbar_arrive_expect_tx(&full[s], kStage);
        if (mode == 0) {
          bulk_load(d, g, 24576, &full[s]);
          bulk_load(d + 24576, g + 24576, 16384, &full[s]);
          bulk_load(d + 40960, g + 40960, 16384, &full[s]);
        } else if (mode == 2) {
          bulk_load(d, g, kStage, &full[s]);
        } else {
          for (int c = 0; c < 7; ++c) bulk_load(d + c * 8192, g + c * 8192, 8192, &full[s]);
        }
      }
    }
    if (!ok) atomicAdd(err, 1u);
  } else if (warp == 3) {
    bool ok = true;
    for (int i = 0; i < iters && ok; ++i) {
      const int s = i % kStages;
      if (lane == 0) {
        if (!mbar_wait(&full[s], (i / kStages) & 1, lim)) ok = false;
        else mbar_arrive(&empty[s]);
      }
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
    }
    if (!ok && lane == 0) atomicAdd(err, 1u);
  }
  __syncthreads();
  const long long t1 = clock64();
  if (threadIdx.x == 96) cyc[blockIdx.x] = t1 - t0;
  // every issued copy has landed: the consumer waited for all of them
}

int main() {
  const size_t bytes = 96ull << 20;
  uint8_t* src;
  cudaMalloc(&src, bytes);
  cudaMemset(src, 1, bytes);
  long long* cyc; unsigned* err;
  cudaMalloc(&cyc, 296 * sizeof(long long));
  cudaMalloc(&err, sizeof(unsigned));
  cudaMemset(err, 0, sizeof(unsigned));
  const int smem = kStages * kStage + 1024;
  cudaFuncSetAttribute(tma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  const char* names[] = {"1 thread, 3 copies/stage", "3 warps, 1 copy each", "1 thread, 1 x 56K",
                         "1 thread, 7 x 8K"};
  const int iters = 400;
  for (int rep = 0; rep < 2; ++rep)
    for (int mode = 0; mode < 4; ++mode) {
      cudaEvent_t e0, e1;
      cudaEventCreate(&e0); cudaEventCreate(&e1);
      cudaEventRecord(e0);
      tma_kernel<<<148, 128, smem>>>(src, bytes, mode, iters, cyc, err);
      cudaEventRecord(e1);
      cudaError_t e = cudaDeviceSynchronize();
      if (e != cudaSuccess) { printf("error %s\n", cudaGetErrorString(e)); return 1; }
      float ms; cudaEventElapsedTime(&ms, e0, e1);
      long long h[148];
      cudaMemcpy(h, cyc, sizeof(h), cudaMemcpyDeviceToHost);
      long long mx = 0; for (int b = 0; b < 148; ++b) mx = mx > h[b] ? mx : h[b];
      unsigned he; cudaMemcpy(&he, err, 4, cudaMemcpyDeviceToHost);
      printf("%-26s cycles/stage=%7.1f  B/clk/SM=%6.1f  total %.2f TB/s  err=%u\n", names[mode],
             (double)mx / iters, (double)kStage * iters / mx, 148.0 * kStage * iters / (ms * 1e-3) / 1e12, he);
    }
  return 0;
}
