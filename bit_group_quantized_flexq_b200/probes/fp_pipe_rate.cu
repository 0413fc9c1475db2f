// Throughput of the epilogue's instruction kinds with independent chains (registers only).
#include <cstdio>
#include <cstdint>
#include <cuda_runtime.h>

// each iteration: 16 independent float2 chains
template <int MODE>
__global__ void __launch_bounds__(512, 1) pipe_kernel(int iters, long long* cyc, float* sink, int warps_active) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float2 a[16], b[16];
  int ib[16];
  for (int j = 0; j < 16; ++j) {
    a[j] = make_float2(1.0f + j * lane, 2.0f - j);
    b[j] = make_float2(0.999f, 1.001f);
    ib[j] = 12345 * j + lane;
  }
  if (warp < warps_active) {
    const long long t0 = clock64();
    for (int it = 0; it < iters; ++it) {
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        if (MODE == 0) a[j] = __ffma2_rn(a[j], b[j], b[(j + 1) & 15]);          // FFMA2
        if (MODE == 1) { a[j].x = fmaf(a[j].x, b[j].x, b[j].y); a[j].y = fmaf(a[j].y, b[j].y, b[j].x); }
        if (MODE == 2) a[j] = __fmul2_rn(a[j], b[j]);                           // FMUL2
        if (MODE == 3) a[j] = __fadd2_rn(a[j], b[j]);                           // FADD2
        if (MODE == 4) { a[j].x += __int2float_rn(ib[j] + it); a[j].y += __int2float_rn(ib[j] - it); } // I2F + FADD
        if (MODE == 5) {   // the epilogue's mix per 4 outputs: 2 FMUL2, 4 I2F, 2 FFMA2 (here per j pair)
          const float2 s = __fmul2_rn(b[j], b[(j + 3) & 15]);
          const float2 p = make_float2(__int2float_rn(ib[j] ^ it), __int2float_rn(ib[j] + it));
          a[j] = __ffma2_rn(p, s, a[j]);
        }
        if (MODE == 6) {   // FADD2 route: FMUL2, FADD2, FFMA2
          const float2 s = __fmul2_rn(b[j], b[(j + 3) & 15]);
          const float2 p = __fadd2_rn(make_float2(__int_as_float(ib[j] ^ it), __int_as_float(ib[j] + it)),
                                      make_float2(-1.5f, -1.5f));
          a[j] = __ffma2_rn(p, s, a[j]);
        }
        if (MODE == 7) {   // scalar FP32 route: FMUL, FMUL, I2F x2, FFMA x2 per 2 outputs
          const float s0 = b[j].x * b[(j + 3) & 15].x, s1 = b[j].y * b[(j + 3) & 15].y;
          a[j].x = fmaf(__int2float_rn(ib[j] ^ it), s0, a[j].x);
          a[j].y = fmaf(__int2float_rn(ib[j] + it), s1, a[j].y);
        }
      }
    }
    const long long t1 = clock64();
    if (lane == 0) cyc[blockIdx.x * 16 + warp] = t1 - t0;
  }
  float f = 0;
  for (int j = 0; j < 16; ++j) f += a[j].x + a[j].y;
  if (f == 1.2345f) sink[threadIdx.x] = f;
}

template <int MODE>
void run(const char* name, int per_j_ops, long long* cyc, float* sink) {
  for (int wa : {4, 8, 16}) {
    const int iters = 4096;
    pipe_kernel<MODE><<<148, 512>>>(iters, cyc, sink, wa);
    cudaDeviceSynchronize();
    long long h[148 * 16];
    cudaMemcpy(h, cyc, sizeof(h), cudaMemcpyDeviceToHost);
    long long mx = 0;
    for (int w = 0; w < wa; ++w) mx = mx > h[w] ? mx : h[w];
    // per iteration per warp: 16 j-steps; per j-step per lane: 2 outputs (float2)
    const double outputs_per_clk = 2.0 * 16 * 32 * wa * iters / mx;
    const double warp_instr_per_clk = (double)per_j_ops * 16 * wa * iters / mx;
    printf("%-34s warps=%2d  lane-results/clk/SM=%6.1f  warp-instr/clk/SM=%5.2f\n", name, wa,
           outputs_per_clk, warp_instr_per_clk);
  }
}

int main() {
  long long* cyc; float* sink;
  cudaMalloc(&cyc, 148 * 16 * sizeof(long long));
  cudaMalloc(&sink, 512 * sizeof(float));
  run<0>("FFMA2 (2 results/instr)", 1, cyc, sink);
  run<1>("FFMA scalar x2", 2, cyc, sink);
  run<2>("FMUL2", 1, cyc, sink);
  run<3>("FADD2", 1, cyc, sink);
  run<4>("I2F x2 + FADD x2", 4, cyc, sink);
  run<5>("mix FMUL2 + 2 I2F + FFMA2", 4, cyc, sink);
  run<6>("mix FMUL2 + FADD2 + FFMA2", 3, cyc, sink);
  run<7>("scalar FMUL x2 + I2F x2 + FFMA x2", 6, cyc, sink);
  cudaError_t e = cudaGetLastError();
  printf("%s\n", cudaGetErrorString(e));
  return 0;
}
