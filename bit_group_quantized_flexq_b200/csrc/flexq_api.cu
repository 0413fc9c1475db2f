// flexq_api.cu -- host side of the C ABI declared in include/flexq.h:
// argument validation, launch planning, tensor-map encoding, kernel launches
// and the device status word.  Every kernel lives in this translation unit
// so that they share the status word without relocatable device code.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>

#include "../../include/flexq.h"
#include "flexq_gemm.cuh"
#include "flexq_gemm_wide.cuh"
#include "flexq_quant.cuh"

namespace {

// Status word written by kernels: [0] code, [1] where, [2] block, [3] unused.
__device__ unsigned int g_flexq_status[4];

thread_local std::string t_last_error;

int fail(int status, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  t_last_error = buf;
  return status;
}

int ok() {
  t_last_error.clear();
  return FLEXQ_OK;
}

int cuda_fail(cudaError_t e, const char* what) {
  return fail(FLEXQ_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) {
  return (reinterpret_cast<uintptr_t>(p) & 15u) == 0;
}

bool valid_gs(int gs) { return gs == 32 || gs == 64 || gs == 128 || gs == 256; }

std::atomic<int> g_force_tokens{0};
std::atomic<int> g_force_split{0};
std::atomic<unsigned long long> g_wait_limit_ns{2000000000ull};
std::atomic<int> g_inject_stall{0};
std::atomic<int> g_force_linear_route{0};   // 0 by plan, 1 fused quantization, 2 separate quantizer

// ---------------------------------------------------------- device state --
constexpr int kMaxDevices = 64;
struct DeviceState {
  bool ready = false;
  int sms = 148;
  unsigned int* status = nullptr;
  unsigned long long attr_mask = 0;   // which GEMM instantiations got their smem limit
};
DeviceState g_dev[kMaxDevices];
std::mutex g_dev_mutex;

int device_state(DeviceState** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(FLEXQ_ERR_UNSUPPORTED, "device index %d", dev);
  std::lock_guard<std::mutex> lock(g_dev_mutex);
  DeviceState& st = g_dev[dev];
  if (!st.ready) {
    int sms = 0;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_flexq_status);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(status)");
    st.sms = sms;
    st.status = static_cast<unsigned int*>(p);
    st.ready = true;
  }
  *out = &st;
  return FLEXQ_OK;
}

int sm_count_or_default() {
  int n = 0;
  if (cudaGetDeviceCount(&n) != cudaSuccess || n == 0) {
    cudaGetLastError();
    return 148;
  }
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    cudaGetLastError();
    return 148;
  }
  return sms;
}

// ------------------------------------------------------------ validation --
int check_gemm_shape(int M, int N, int K, int gs) {
  if (M < 0 || N <= 0 || K <= 0)
    return fail(FLEXQ_ERR_INVALID_ARG, "sizes must be M >= 0, N > 0, K > 0 (M=%d N=%d K=%d)", M, N, K);
  if (!valid_gs(gs)) return fail(FLEXQ_ERR_UNSUPPORTED, "group_size %d not in {32,64,128,256}", gs);
  if (N % 128) return fail(FLEXQ_ERR_UNSUPPORTED, "N=%d is not a multiple of 128", N);
  if (K % 256) return fail(FLEXQ_ERR_UNSUPPORTED, "K=%d is not a multiple of 256", K);
  if (K % gs) return fail(FLEXQ_ERR_UNSUPPORTED, "K=%d is not a multiple of group_size %d", K, gs);
  if (N / 128 > 65535) return fail(FLEXQ_ERR_UNSUPPORTED, "N=%d too large", N);
  return FLEXQ_OK;
}

int check_ptrs(int n, const void* const* ptrs, const char* const* names) {
  for (int i = 0; i < n; ++i) {
    if (!ptrs[i]) return fail(FLEXQ_ERR_INVALID_ARG, "%s is NULL", names[i]);
    if (!aligned16(ptrs[i])) return fail(FLEXQ_ERR_MISALIGNED, "%s is not 16-byte aligned", names[i]);
  }
  return FLEXQ_OK;
}

// --------------------------------------------------------------- planning --
int max_split_for(int T) {
  switch (T) {
    case 16: return flexq::GemmCfg<16>::kMaxSplit;
    case 32: return flexq::GemmCfg<32>::kMaxSplit;
    case 64: return flexq::GemmCfg<64>::kMaxSplit;
    default: return flexq::WideCfg::kMaxSplit;
  }
}

// Split-K workspace: kCounterBytes of arrival counters (one per output tile,
// zero between calls) at a fixed place, then per output tile `split` FP32
// partial tiles of T x 128.  The counters never move, so calls of different
// shapes can share one workspace without their partial tiles landing on
// another shape's counters.
int min_blocks_for(int T) {
  switch (T) {
    case 16: return flexq::GemmCfg<16>::kMinBlocks;
    case 32: return flexq::GemmCfg<32>::kMinBlocks;
    case 64: return flexq::GemmCfg<64>::kMinBlocks;
    default: return 1;                       // the wide kernel: one CTA per SM
  }
}

constexpr size_t kCounterBytes = 4096;
constexpr long long kMaxSplitTiles = kCounterBytes / sizeof(unsigned);

struct Plan {
  int T;
  int split;             // K split of the split tiles (1: none)
  long long n_full;      // output tiles run whole, first
  long long n_split;     // output tiles split `split` ways, after them
  long long ctas;
};

// Tokens per tile follow M.  With fewer output tiles than CTA slots (SMs x
// CTAs per SM) every tile is split along K to fill the machine; otherwise the
// whole waves run unsplit and only the tiles of a partial last wave are split,
// so that the last wave is as full as the others.
Plan make_plan(int M, int N, int K, int gs, int sms, bool partials) {
  Plan p;
  const int units = K / 256;                          // K stages of the kernel
  p.T = M <= 16 ? 16 : M <= 32 ? 32 : M <= 64 ? 64 : 128;
  // 33..64 tokens: two 32-token tiles (each weight tile read twice, the
  // second time mostly from L2) beat one 64-token tile whenever both fit in
  // one wave of CTA slots (M = 64: 5120^2 14.9 us against 21.9, 5120x13824
  // 28.0 against 38.0); with more weight tiles than that (N = 28672) the
  // 64-token tile keeps one wave and wins
  if (p.T == 64 && 2LL * (N / 128) <= static_cast<long long>(sms) * min_blocks_for(32)) p.T = 32;
  const int fT = g_force_tokens.load(), fS = g_force_split.load();
  if (fT == 16 || fT == 32 || fT == 64 || fT == 128) p.T = fT;   // any width: more or fewer token tiles
  const long long tiles = static_cast<long long>(N / 128) * ((M + p.T - 1) / p.T);
  const long long slots = static_cast<long long>(sms) * min_blocks_for(p.T);
  const long long max_s = std::min<long long>(max_split_for(p.T), units);
  long long s = 1, n_split = 0;
  // the split never makes the split tiles' units exceed one wave of slots:
  // a second, partial wave costs more than the split saves
  if (tiles < slots) {
    s = slots / tiles;
    // 128-token tiles hand 64 KB partial tiles to the reduction: below 8
    // stages of K per CTA the tail costs more than the extra CTAs bring
    // (M = 128, 4096^2: split 2 19.3 us, split 4 21.2 us)
    if (p.T == 128) s = std::min<long long>(s, std::max(1, units / 8));
    n_split = tiles;
  } else if (tiles % slots) {
    n_split = tiles % slots;                          // the partial last wave
    s = slots / n_split;
  }
  s = std::max<long long>(1, std::min(s, max_s));
  if (fS >= 1 && fS <= max_split_for(p.T) && fS <= units) {
    s = fS;                                           // forced: every tile split fS ways
    n_split = tiles;
  }
  if (partials || s == 1 || n_split > kMaxSplitTiles) {
    s = 1;
    n_split = 0;
  }
  p.split = static_cast<int>(s);
  p.n_split = n_split;
  p.n_full = tiles - n_split;
  p.ctas = p.n_full + p.n_split * p.split;
  return p;
}

size_t workspace_bytes_for(const Plan& p, int /*M*/, int /*N*/) {
  if (p.split <= 1 || p.n_split == 0) return 0;
  return kCounterBytes + static_cast<size_t>(p.n_split) * p.split * p.T * 128 * sizeof(float);
}

// ------------------------------------------------------------ tensor map --
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = []() {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      p = nullptr;
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }();
  return fn;
}

// int8 activations [M, K] row-major; box = 128 bytes x T rows, 128-byte
// swizzle; rows past M read as zero.
int encode_x_map(CUtensorMap* map, const void* xq, int M, int K, int T) {
  auto fn = encode_fn();
  if (!fn) return fail(FLEXQ_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(M)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(K)};
  cuuint32_t box[2] = {128u, static_cast<cuuint32_t>(T)};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(xq), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(FLEXQ_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return FLEXQ_OK;
}

// FP16 scales stored group-major: [G rows][ld elements]; box = `box_rows`
// consecutive elements (tokens or weight rows) x 8 groups; elements past
// `extent` and groups past G read as zero.
int encode_scale_map(CUtensorMap* map, const void* scales, int extent, int ld, int G,
                     int box_rows) {
  auto fn = encode_fn();
  if (!fn) return fail(FLEXQ_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(extent), static_cast<cuuint64_t>(G)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld) * 2};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(box_rows), 8u};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(scales), dims,
                  strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return fail(FLEXQ_ERR_CUDA, "cuTensorMapEncodeTiled (scales) failed (%d)", static_cast<int>(r));
  return FLEXQ_OK;
}

int act_scales_ld(int M) { return (M + 7) / 8 * 8; }

// --------------------------------------------------------------- launches --
template <int T>
int ctrl_offset_for() {
  return (flexq::GemmCfg<T>::kMainBytes + 15) & ~15;
}

// the fused activation quantizer's block (barriers and scale slots) follows
// the control block
template <int T>
int fq_offset_for() {
  return (ctrl_offset_for<T>() + static_cast<int>(sizeof(flexq::GemmCtrl<T>)) + 15) & ~15;
}

template <int T, bool FUSEDQ = false>
int smem_bytes_for() {
  if (FUSEDQ) return 1024 + fq_offset_for<T>() + flexq::FusedQLayout<T>::kBytes;
  return 1024 + ctrl_offset_for<T>() + static_cast<int>(sizeof(flexq::GemmCtrl<T>));
}

template <int T, bool PARTIALS, bool FUSEDQ = false, int LAYOUT = 0>
int launch_gemm_t(DeviceState* st, const CUtensorMap& map, const CUtensorMap& map_sa,
                  const flexq::LayerTable& tab, flexq::GemmArgs a, long long grid_ctas,
                  cudaStream_t stream) {
  using Cfg = flexq::GemmCfg<T>;
  auto kern = flexq::gemm_w6ax_kernel<T, PARTIALS, FUSEDQ, LAYOUT>;
  const unsigned long long bit =
      1ull << ((T == 16 ? 0 : T == 32 ? 1 : 2) + (PARTIALS ? 4 : 0) + (FUSEDQ ? 8 : 0) + 16 * LAYOUT);
  const int smem = smem_bytes_for<T, FUSEDQ>();
  {
    std::lock_guard<std::mutex> lock(g_dev_mutex);
    if (!(st->attr_mask & bit)) {
      cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
      if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
      st->attr_mask |= bit;
    }
  }
  a.ctrl_offset = ctrl_offset_for<T>();
  a.fq_offset = FUSEDQ ? fq_offset_for<T>() : 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid_ctas), 1, 1);
  cfg.blockDim = dim3(Cfg::kThreads, 1, 1);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = stream;
  // programmatic stream serialization: the kernel may start while the
  // previous kernel of the stream finishes (it prefetches its weights, then
  // waits for that kernel before reading activations)
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, map, map_sa, tab, a);
  if (e != cudaSuccess) return cuda_fail(e, "GEMM launch");
  return FLEXQ_OK;
}

// The layer table of a launch with one layer.
flexq::LayerTable single_layer_table(const CUtensorMap& map_sw, const void* Wp, void* Y, int N,
                                     const Plan& plan) {
  flexq::LayerTable t;
  memset(&t, 0, sizeof(t));
  t.sw[0] = map_sw;
  t.wp[0] = static_cast<const uint8_t*>(Wp);
  t.y[0] = static_cast<__half*>(Y);
  t.part0[0] = 0;
  t.N[0] = N;
  t.unit0[0] = 0;
  t.unit0[1] = static_cast<int>(plan.ctas);
  t.n_full[0] = static_cast<int>(plan.n_full);
  t.split[0] = plan.split;
  t.tile0[0] = 0;
  t.n_layers = 1;
  return t;
}

// 128-token tiles: the warpgroup-role kernel of flexq_gemm_wide.cuh.
template <bool PARTIALS, int LAYOUT = 0>
int launch_gemm_wide(DeviceState* st, const CUtensorMap& map, flexq::GemmArgs a,
                     long long grid_ctas, cudaStream_t stream) {
  using Cfg = flexq::WideCfg;
  auto kern = flexq::gemm_w6ax_wide_kernel<PARTIALS, LAYOUT>;
  const unsigned long long bit = 1ull << (32 + (PARTIALS ? 1 : 0) + 2 * LAYOUT);
  const int ctrl_off = (Cfg::kMainBytes + 15) & ~15;
  const int smem = 1024 + ctrl_off + static_cast<int>(sizeof(flexq::WideCtrl));
  {
    std::lock_guard<std::mutex> lock(g_dev_mutex);
    if (!(st->attr_mask & bit)) {
      // the warpgroups' register budgets must fit in what the CTA launches
      // with, or the epilogue's increase would wait for registers that never
      // come: refuse to launch instead
      cudaFuncAttributes fa;
      cudaError_t e = cudaFuncGetAttributes(&fa, kern);
      if (e != cudaSuccess) return cuda_fail(e, "cudaFuncGetAttributes");
      const long long launch_regs = static_cast<long long>(fa.numRegs) * Cfg::kThreads;
      const long long budget = 128LL * Cfg::kRegsCtl + 128LL * Cfg::kRegsUnpack + 256LL * Cfg::kRegsEpi;
      if (launch_regs < budget)
        return fail(FLEXQ_ERR_CUDA, "wide GEMM compiled with %d registers per thread; its register "
                    "split needs %lld per CTA", fa.numRegs, budget);
      e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
      if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
      st->attr_mask |= bit;
    }
  }
  a.ctrl_offset = ctrl_off;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid_ctas), 1, 1);
  cfg.blockDim = dim3(Cfg::kThreads, 1, 1);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, map, a);
  if (e != cudaSuccess) return cuda_fail(e, "GEMM launch");
  return FLEXQ_OK;
}

// The caller's split-K workspace against the plan: none (NULL, 0 bytes)
// runs every tile whole; one too small for the plan is an error.
int apply_workspace(Plan* plan, int M, int N, void* workspace, size_t workspace_bytes) {
  const size_t need = workspace_bytes_for(*plan, M, N);
  if (need > 0) {
    if (workspace == nullptr && workspace_bytes == 0) {
      // no workspace: no K split (below)
    } else if (workspace == nullptr || workspace_bytes < need) {
      return fail(FLEXQ_ERR_INVALID_ARG, "workspace of %zu bytes at %p, the plan needs %zu",
                  workspace_bytes, workspace, need);
    } else if (!aligned16(workspace)) {
      return fail(FLEXQ_ERR_MISALIGNED, "workspace is not 16-byte aligned");
    }
  }
  if (plan->split > 1 && (workspace == nullptr || need == 0)) {   // run every tile whole
    plan->split = 1;
    plan->n_full += plan->n_split;
    plan->n_split = 0;
    plan->ctas = plan->n_full;
  }
  return FLEXQ_OK;
}

int gemm_common(int M, int N, int K, int gs, const int8_t* Xq, const void* Xs, const void* Wp,
                const void* Ws, void* Y, int32_t* P, bool partials, void* workspace,
                size_t workspace_bytes, void* stream, int layout = 0) {
  int rc = check_gemm_shape(M, N, K, gs);
  if (rc) return rc;
  if (M == 0) return ok();               // empty batch: nothing to read or write
  if (partials) {
    const void* ptrs[] = {Xq, Wp, P};
    const char* names[] = {"Xq", "Wq_packed", "P"};
    if ((rc = check_ptrs(3, ptrs, names))) return rc;
  } else {
    const void* ptrs[] = {Xq, Xs, Wp, Ws, Y};
    const char* names[] = {"Xq", "X_scales", "Wq_packed", "W_scales", "Y"};
    if ((rc = check_ptrs(5, ptrs, names))) return rc;
  }
  DeviceState* st = nullptr;
  if ((rc = device_state(&st))) return rc;
  Plan plan = make_plan(M, N, K, gs, st->sms, partials);
  if ((rc = apply_workspace(&plan, M, N, workspace, workspace_bytes))) return rc;
  CUtensorMap map, map_sa, map_sw;
  if ((rc = encode_x_map(&map, Xq, M, K, plan.T))) return rc;
  memset(&map_sa, 0, sizeof(map_sa));
  memset(&map_sw, 0, sizeof(map_sw));
  if (!partials) {
    const int G = K / gs;
    if ((rc = encode_scale_map(&map_sa, Xs, M, act_scales_ld(M), G, plan.T))) return rc;
    if ((rc = encode_scale_map(&map_sw, Ws, N, N, G, 128))) return rc;
  }
  flexq::GemmArgs a = {};
  a.wp = static_cast<const uint8_t*>(Wp);
  a.y = static_cast<__half*>(Y);
  a.p = P;
  a.sa = static_cast<const __half*>(Xs);
  a.sw = static_cast<const __half*>(Ws);
  a.sa_ld = act_scales_ld(M);
  if (plan.split > 1) {
    a.ws_cnt = static_cast<unsigned int*>(workspace);
    a.ws_part = reinterpret_cast<float*>(static_cast<char*>(workspace) + kCounterBytes);
  }
  a.status = st->status;
  a.wait_limit_ns = g_wait_limit_ns.load();
  a.M = M; a.N = N; a.K = K; a.gs = gs;
  a.tiles_n = N / 128;
  a.n_full = static_cast<int>(plan.n_full);
  a.split = plan.split;
  a.stall = g_inject_stall.exchange(0);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const flexq::LayerTable tab = single_layer_table(map_sw, Wp, Y, N, plan);
  if (layout == 1 && !partials) {
    switch (plan.T) {
      case 16: rc = launch_gemm_t<16, false, false, 1>(st, map, map_sa, tab, a, plan.ctas, s); break;
      case 32: rc = launch_gemm_t<32, false, false, 1>(st, map, map_sa, tab, a, plan.ctas, s); break;
      case 64: rc = launch_gemm_t<64, false, false, 1>(st, map, map_sa, tab, a, plan.ctas, s); break;
      default: rc = launch_gemm_wide<false, 1>(st, map, a, plan.ctas, s); break;
    }
    return rc ? rc : ok();
  }
  switch (plan.T) {
    case 16: rc = partials ? launch_gemm_t<16, true>(st, map, map_sa, tab, a, plan.ctas, s) : launch_gemm_t<16, false>(st, map, map_sa, tab, a, plan.ctas, s); break;
    case 32: rc = partials ? launch_gemm_t<32, true>(st, map, map_sa, tab, a, plan.ctas, s) : launch_gemm_t<32, false>(st, map, map_sa, tab, a, plan.ctas, s); break;
    case 64: rc = partials ? launch_gemm_t<64, true>(st, map, map_sa, tab, a, plan.ctas, s) : launch_gemm_t<64, false>(st, map, map_sa, tab, a, plan.ctas, s); break;
    default: rc = partials ? launch_gemm_wide<true>(st, map, a, plan.ctas, s) : launch_gemm_wide<false>(st, map, a, plan.ctas, s); break;
  }
  return rc ? rc : ok();
}

// ------------------------------------------------------- linear layers --
// A linear layer from FP16 activations: quantize them (bits 6 or 8), then the
// group GEMM, in one of two routes.  Inside the GEMM (16-token tiles, one
// launch) the quantization saves the separate quantizer's launch and its
// dependency (about 1.5 us per layer) but adds the quantization of the
// tile's rows to every pipeline stage of the unpack warps, a cost that grows
// with the tokens and the stages of a CTA; it is taken where
// (M + 2) * stages <= 28 (measured per layer on the LLaMA-2 7B, 13B and 70B
// shapes, weights cold: at one token, 2 to 8 stages per CTA gain 2-18 %, 10
// stages lose 4 %, 28 or 32 stages 10-22 %; at 8 tokens 2 stages gain 7 %,
// 3 lose 4 %; at 12 tokens 2 stages gain 3 %).
// Otherwise the activation quantizer runs first, its codes and scales in
// the caller's workspace after the GEMM's region, whose arrival counters
// keep their fixed place at the start.
bool fused_by_shape(int T, int M, int K, int split) {
  const int route = g_force_linear_route.load();
  if (T != 16) return false;
  if (route != 0) return route == 1;
  const int stages = (K / 256 + split - 1) / split;         // per CTA
  return (M + 2) * stages <= 28;
}

bool linear_fused(const Plan& p, int M, int K) { return fused_by_shape(p.T, M, K, p.split); }

struct LinearLayout {
  bool fused;
  size_t gemm_bytes;     // GEMM region from offset 0 (counters, partial tiles)
  size_t xq_off, xs_off; // separate quantizer: codes [M, K] and scales [G][ld]
  size_t total;
};

LinearLayout linear_layout(const Plan& p, int M, int N, int K, int gs) {
  LinearLayout L = {};
  L.fused = linear_fused(p, M, K);
  L.gemm_bytes = workspace_bytes_for(p, M, N);
  if (L.fused) {
    L.total = L.gemm_bytes;
    return L;
  }
  const size_t head = std::max(L.gemm_bytes, kCounterBytes);
  L.xq_off = (head + 255) & ~static_cast<size_t>(255);
  L.xs_off = (L.xq_off + static_cast<size_t>(M) * K + 255) & ~static_cast<size_t>(255);
  L.total = L.xs_off + static_cast<size_t>(K / gs) * act_scales_ld(M) * sizeof(__half);
  return L;
}

int linear_common(int M, int N, int K, int gs, int bits, const void* X, const void* Wp,
                  const void* Ws, void* Y, void* workspace, size_t workspace_bytes, void* stream,
                  int layout = 0) {
  if (bits != 6 && bits != 8) return fail(FLEXQ_ERR_INVALID_ARG, "bits=%d is not 6 or 8", bits);
  int rc = check_gemm_shape(M, N, K, gs);
  if (rc) return rc;
  if (M == 0) return ok();               // empty batch: nothing to read or write
  const void* ptrs[] = {X, Wp, Ws, Y};
  const char* names[] = {"X_fp16", "Wq_packed", "W_scales", "Y"};
  if ((rc = check_ptrs(4, ptrs, names))) return rc;
  DeviceState* st = nullptr;
  if ((rc = device_state(&st))) return rc;
  Plan plan = make_plan(M, N, K, gs, st->sms, false);
  const LinearLayout L = linear_layout(plan, M, N, K, gs);
  if (!L.fused) {
    if (workspace == nullptr || workspace_bytes < L.total)
      return fail(FLEXQ_ERR_INVALID_ARG,
                  "workspace of %zu bytes at %p: this shape quantizes its activations "
                  "separately and needs %zu", workspace_bytes, workspace, L.total);
    if (!aligned16(workspace)) return fail(FLEXQ_ERR_MISALIGNED, "workspace is not 16-byte aligned");
    int8_t* xq = reinterpret_cast<int8_t*>(static_cast<char*>(workspace) + L.xq_off);
    void* xs = static_cast<char*>(workspace) + L.xs_off;
    if ((rc = flexq_quantize_act(M, K, gs, bits, X, xq, xs, stream))) return rc;
    return gemm_common(M, N, K, gs, xq, xs, Wp, Ws, Y, nullptr, false, workspace, L.xq_off,
                       stream, layout);
  }
  if ((rc = apply_workspace(&plan, M, N, workspace, workspace_bytes))) return rc;
  CUtensorMap map_x, map_sa, map_sw;     // activations and their scales: read by the kernel itself
  memset(&map_x, 0, sizeof(map_x));
  memset(&map_sa, 0, sizeof(map_sa));
  if ((rc = encode_scale_map(&map_sw, Ws, N, N, K / gs, 128))) return rc;
  flexq::GemmArgs a = {};
  a.wp = static_cast<const uint8_t*>(Wp);
  a.y = static_cast<__half*>(Y);
  a.x = static_cast<const __half*>(X);
  a.qmax = bits == 6 ? 31 : 127;
  if (plan.split > 1) {
    a.ws_cnt = static_cast<unsigned int*>(workspace);
    a.ws_part = reinterpret_cast<float*>(static_cast<char*>(workspace) + kCounterBytes);
  }
  a.status = st->status;
  a.wait_limit_ns = g_wait_limit_ns.load();
  a.M = M; a.N = N; a.K = K; a.gs = gs;
  a.tiles_n = N / 128;
  a.n_full = static_cast<int>(plan.n_full);
  a.split = plan.split;
  a.stall = g_inject_stall.exchange(0);
  const flexq::LayerTable tab = single_layer_table(map_sw, Wp, Y, N, plan);
  if (layout == 1)
    rc = launch_gemm_t<16, false, true, 1>(st, map_x, map_sa, tab, a, plan.ctas,
                                           static_cast<cudaStream_t>(stream));
  else
    rc = launch_gemm_t<16, false, true>(st, map_x, map_sa, tab, a, plan.ctas,
                                        static_cast<cudaStream_t>(stream));
  return rc ? rc : ok();
}

// ------------------------------------------------------ grouped launches --
// Layers that read the same activations (the q, k and v projections, or gate
// and up) in one launch of the decode kernel: one set of CTAs for all of
// them, so that a layer's set-up, first-byte latency and split-K tail overlap
// the other layers' streaming instead of following it.  Each layer keeps its
// own packed weights, scales and output.  The token tile follows M as for a
// single layer; with fewer output tiles in all layers than CTA slots every
// tile is split along K by the same factor, otherwise nothing is split.
// Batches that take 128-token tiles run the layers one launch after another.
struct GroupPlan {
  int T = 0, split = 1, n = 0;
  long long tiles[flexq::kMaxLayers] = {};
  long long n_split[flexq::kMaxLayers] = {};
  long long ctas = 0;
  size_t ws_bytes = 0;
};

GroupPlan make_group_plan(int M, const int* N, int n, int K, int gs, int sms,
                          bool allow_split = true) {
  GroupPlan g;
  g.n = n;
  long long n_sum = 0;
  for (int l = 0; l < n; ++l) n_sum += N[l];
  g.T = make_plan(M, static_cast<int>(std::min<long long>(n_sum, 1 << 30)), K, gs, sms, false).T;
  const long long mtiles = (M + g.T - 1) / g.T;
  long long total = 0;
  for (int l = 0; l < n; ++l) total += (g.tiles[l] = static_cast<long long>(N[l] / 128) * mtiles);
  const long long slots = static_cast<long long>(sms) * min_blocks_for(g.T);
  const long long max_s = std::min<long long>(max_split_for(g.T), K / 256);
  long long s = total < slots ? slots / total : 1;
  const int fS = g_force_split.load();
  if (fS >= 1 && fS <= max_split_for(g.T) && fS <= K / 256) s = fS;
  s = std::max<long long>(1, std::min(s, max_s));
  if (!allow_split || (s > 1 && total > kMaxSplitTiles)) s = 1;
  g.split = static_cast<int>(s);
  size_t part = 0;
  for (int l = 0; l < n; ++l) {
    g.n_split[l] = s > 1 ? g.tiles[l] : 0;
    g.ctas += (g.tiles[l] - g.n_split[l]) + g.n_split[l] * s;
    part += static_cast<size_t>(g.n_split[l]) * s * g.T * 128 * sizeof(float);
  }
  g.ws_bytes = s > 1 ? kCounterBytes + part : 0;
  return g;
}

int check_group(int M, int K, int gs, int bits, int n_layers, const flexq_layer_t* layers,
                int* N) {
  if (bits != 6 && bits != 8) return fail(FLEXQ_ERR_INVALID_ARG, "act_bits=%d is not 6 or 8", bits);
  if (n_layers < 1 || n_layers > flexq::kMaxLayers)
    return fail(FLEXQ_ERR_INVALID_ARG, "n_layers=%d not in 1..%d", n_layers, flexq::kMaxLayers);
  if (!layers) return fail(FLEXQ_ERR_INVALID_ARG, "layers is NULL");
  for (int l = 0; l < n_layers; ++l) {
    int rc = check_gemm_shape(M, layers[l].N, K, gs);
    if (rc) return rc;
    N[l] = layers[l].N;
  }
  return FLEXQ_OK;
}

int check_group_ptrs(int n_layers, const flexq_layer_t* layers) {
  for (int l = 0; l < n_layers; ++l) {
    const void* ptrs[] = {layers[l].Wq_packed, layers[l].W_scales, layers[l].Y_fp16};
    const char* names[] = {"layers[].Wq_packed", "layers[].W_scales", "layers[].Y_fp16"};
    int rc = check_ptrs(3, ptrs, names);
    if (rc) return rc;
  }
  return FLEXQ_OK;
}

// The grouped launch itself (plan.T <= 64): X is int8 codes with their
// scales, or (fused) the FP16 activations quantized inside the kernel.
int launch_group(DeviceState* st, const GroupPlan& g, int M, int K, int gs, int bits, const void* X,
                 const void* Xs, bool fused, const flexq_layer_t* layers, void* workspace,
                 cudaStream_t stream) {
  flexq::LayerTable tab;
  memset(&tab, 0, sizeof(tab));
  tab.n_layers = g.n;
  long long unit = 0, tile0 = 0, part0 = 0;
  for (int l = 0; l < g.n; ++l) {
    int rc = encode_scale_map(&tab.sw[l], layers[l].W_scales, layers[l].N, layers[l].N, K / gs, 128);
    if (rc) return rc;
    tab.wp[l] = static_cast<const uint8_t*>(layers[l].Wq_packed);
    tab.y[l] = static_cast<__half*>(layers[l].Y_fp16);
    tab.N[l] = layers[l].N;
    tab.unit0[l] = static_cast<int>(unit);
    tab.n_full[l] = static_cast<int>(g.tiles[l] - g.n_split[l]);
    tab.split[l] = g.split;
    tab.tile0[l] = static_cast<int>(tile0);
    tab.part0[l] = part0;
    unit += (g.tiles[l] - g.n_split[l]) + g.n_split[l] * g.split;
    tile0 += g.n_split[l];
    part0 += g.n_split[l] * g.split * g.T * 128;
  }
  tab.unit0[g.n] = static_cast<int>(unit);
  CUtensorMap map_x, map_sa;
  memset(&map_x, 0, sizeof(map_x));
  memset(&map_sa, 0, sizeof(map_sa));
  int rc = FLEXQ_OK;
  if (!fused) {
    if ((rc = encode_x_map(&map_x, X, M, K, g.T))) return rc;
    if ((rc = encode_scale_map(&map_sa, Xs, M, act_scales_ld(M), K / gs, g.T))) return rc;
  }
  flexq::GemmArgs a = {};
  a.x = fused ? static_cast<const __half*>(X) : nullptr;
  a.qmax = bits == 6 ? 31 : 127;
  if (g.split > 1) {
    a.ws_cnt = static_cast<unsigned int*>(workspace);
    a.ws_part = reinterpret_cast<float*>(static_cast<char*>(workspace) + kCounterBytes);
  }
  a.status = st->status;
  a.wait_limit_ns = g_wait_limit_ns.load();
  a.M = M; a.K = K; a.gs = gs;
  a.stall = g_inject_stall.exchange(0);
  if (fused) return launch_gemm_t<16, false, true>(st, map_x, map_sa, tab, a, g.ctas, stream);
  switch (g.T) {
    case 16: return launch_gemm_t<16, false>(st, map_x, map_sa, tab, a, g.ctas, stream);
    case 32: return launch_gemm_t<32, false>(st, map_x, map_sa, tab, a, g.ctas, stream);
    default: return launch_gemm_t<64, false>(st, map_x, map_sa, tab, a, g.ctas, stream);
  }
}

// Workspace of a grouped GEMM: the grouped plan's split-K region, or for
// 128-token tiles the largest single layer's (they run one after another).
size_t group_gemm_bytes(int M, const int* N, int n, int K, int gs, int sms, GroupPlan* out) {
  GroupPlan g = make_group_plan(M, N, n, K, gs, sms);
  if (out) *out = g;
  if (g.T <= 64) return g.ws_bytes;
  size_t need = 0;
  for (int l = 0; l < n; ++l)
    need = std::max(need, workspace_bytes_for(make_plan(M, N[l], K, gs, sms, false), M, N[l]));
  return need;
}

int gemm_group_common(int M, int K, int gs, int bits, const int8_t* Xq, const void* Xs,
                      int n_layers, const flexq_layer_t* layers, void* workspace,
                      size_t workspace_bytes, void* stream) {
  int N[flexq::kMaxLayers];
  int rc = check_group(M, K, gs, bits, n_layers, layers, N);
  if (rc) return rc;
  if (M == 0) return ok();
  const void* ptrs[] = {Xq, Xs};
  const char* names[] = {"Xq", "X_scales"};
  if ((rc = check_ptrs(2, ptrs, names)) || (rc = check_group_ptrs(n_layers, layers))) return rc;
  DeviceState* st = nullptr;
  if ((rc = device_state(&st))) return rc;
  GroupPlan g;
  const size_t need = group_gemm_bytes(M, N, n_layers, K, gs, st->sms, &g);
  if (g.T > 64) {
    for (int l = 0; l < n_layers; ++l) {
      rc = gemm_common(M, layers[l].N, K, gs, Xq, Xs, layers[l].Wq_packed, layers[l].W_scales,
                       layers[l].Y_fp16, nullptr, false, workspace, workspace_bytes, stream);
      if (rc) return rc;
    }
    return ok();
  }
  if (need > 0) {
    if (workspace == nullptr && workspace_bytes == 0) {
      g = make_group_plan(M, N, n_layers, K, gs, st->sms, false);   // no workspace: no K split
    } else if (workspace == nullptr || workspace_bytes < need) {
      return fail(FLEXQ_ERR_INVALID_ARG, "workspace of %zu bytes at %p, the grouped plan needs %zu",
                  workspace_bytes, workspace, need);
    } else if (!aligned16(workspace)) {
      return fail(FLEXQ_ERR_MISALIGNED, "workspace is not 16-byte aligned");
    }
  }
  rc = launch_group(st, g, M, K, gs, bits, Xq, Xs, false, layers, workspace,
                    static_cast<cudaStream_t>(stream));
  return rc ? rc : ok();
}

// A grouped linear call quantizes inside the GEMM under the same rule as a
// single layer (16-token tiles, few tokens times stages of K per CTA); else
// the activation quantizer writes codes and scales after the GEMM's region
// of the workspace and the grouped GEMM reads them.
struct GroupLinearLayout {
  bool fused;
  GroupPlan plan;
  size_t gemm_bytes, xq_off, xs_off, total;
};

GroupLinearLayout group_linear_layout(int M, const int* N, int n, int K, int gs, int sms) {
  GroupLinearLayout L = {};
  L.gemm_bytes = group_gemm_bytes(M, N, n, K, gs, sms, &L.plan);
  L.fused = fused_by_shape(L.plan.T, M, K, L.plan.split);
  if (L.fused) {
    L.total = L.gemm_bytes;
    return L;
  }
  const size_t head = std::max(L.gemm_bytes, kCounterBytes);
  L.xq_off = (head + 255) & ~static_cast<size_t>(255);
  L.xs_off = (L.xq_off + static_cast<size_t>(M) * K + 255) & ~static_cast<size_t>(255);
  L.total = L.xs_off + static_cast<size_t>(K / gs) * act_scales_ld(M) * sizeof(__half);
  return L;
}

int linear_group_common(int M, int K, int gs, int bits, const void* X, int n_layers,
                        const flexq_layer_t* layers, void* workspace, size_t workspace_bytes,
                        void* stream) {
  int N[flexq::kMaxLayers];
  int rc = check_group(M, K, gs, bits, n_layers, layers, N);
  if (rc) return rc;
  if (M == 0) return ok();
  const void* ptrs[] = {X};
  const char* names[] = {"X_fp16"};
  if ((rc = check_ptrs(1, ptrs, names)) || (rc = check_group_ptrs(n_layers, layers))) return rc;
  DeviceState* st = nullptr;
  if ((rc = device_state(&st))) return rc;
  const GroupLinearLayout L = group_linear_layout(M, N, n_layers, K, gs, st->sms);
  if (workspace == nullptr || workspace_bytes < L.total) {
    if (!(L.total == 0 && workspace == nullptr))
      return fail(FLEXQ_ERR_INVALID_ARG, "workspace of %zu bytes at %p, the grouped layer needs %zu",
                  workspace_bytes, workspace, L.total);
  }
  if (workspace && !aligned16(workspace)) return fail(FLEXQ_ERR_MISALIGNED, "workspace is not 16-byte aligned");
  if (L.fused) {
    rc = launch_group(st, L.plan, M, K, gs, bits, X, nullptr, true, layers, workspace,
                      static_cast<cudaStream_t>(stream));
    return rc ? rc : ok();
  }
  int8_t* xq = reinterpret_cast<int8_t*>(static_cast<char*>(workspace) + L.xq_off);
  void* xs = static_cast<char*>(workspace) + L.xs_off;
  if ((rc = flexq_quantize_act(M, K, gs, bits, X, xq, xs, stream))) return rc;
  return gemm_group_common(M, K, gs, bits, xq, xs, n_layers, layers, workspace, L.xq_off, stream);
}

// --------------------------------------------------- static GEMM scratch --
// Scratch of flexq_gemm_static_scratch, for callers that may not allocate
// device memory: the same layout as a caller workspace (arrival counters,
// then FP32 partial tiles), fixed at 16 MiB.  Every device that loads the
// library holds it until the process exits.
constexpr size_t kStaticScratchBytes = static_cast<size_t>(16) << 20;
static __device__ __align__(256) unsigned char g_flexq_static_scratch[kStaticScratchBytes];

// Device address of the scratch on each device, looked up once per device
// with that device current (host code may not use the symbol itself: in host
// code it names a host-side stand-in, not device memory).
void* g_static_scratch_ptr[kMaxDevices] = {};
std::mutex g_static_scratch_mutex;

int static_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(FLEXQ_ERR_UNSUPPORTED, "device index %d", dev);
  std::lock_guard<std::mutex> lock(g_static_scratch_mutex);
  if (g_static_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_flexq_static_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(static scratch)");
    g_static_scratch_ptr[dev] = p;
  }
  *out = g_static_scratch_ptr[dev];
  return FLEXQ_OK;
}

}  // namespace

// ===================================================================== ABI ==
extern "C" {

const char* flexq_status_string(int status) {
  switch (status) {
    case FLEXQ_OK: return "FLEXQ_OK";
    case FLEXQ_ERR_INVALID_ARG: return "FLEXQ_ERR_INVALID_ARG";
    case FLEXQ_ERR_UNSUPPORTED: return "FLEXQ_ERR_UNSUPPORTED";
    case FLEXQ_ERR_MISALIGNED: return "FLEXQ_ERR_MISALIGNED";
    case FLEXQ_ERR_CUDA: return "FLEXQ_ERR_CUDA";
    case FLEXQ_ERR_DEVICE_TIMEOUT: return "FLEXQ_ERR_DEVICE_TIMEOUT";
    default: return "FLEXQ_ERR_UNKNOWN";
  }
}

const char* flexq_last_error_message(void) { return t_last_error.c_str(); }

size_t flexq_act_scales_ld(int M) { return M > 0 ? static_cast<size_t>(act_scales_ld(M)) : 0; }

size_t flexq_weight_packed_bytes(int N, int K, int group_size) {
  if (N <= 0 || K <= 0 || N % 128 || K % 256 || !valid_gs(group_size) || K % group_size) return 0;
  return static_cast<size_t>(N) * static_cast<size_t>(K) / 4 * 3;
}

int flexq_quantize_weight(int N, int K, int group_size, const void* W_fp16, void* Wq_packed,
                          void* W_scales_fp16, void* stream) {
  return flexq_quantize_weight_layout(N, K, group_size, FLEXQ_LAYOUT_BYTE_ALIGNED, W_fp16,
                                      Wq_packed, W_scales_fp16, stream);
}

int flexq_quantize_weight_layout(int N, int K, int group_size, int layout, const void* W_fp16,
                                 void* Wq_packed, void* W_scales_fp16, void* stream) {
  if (layout != FLEXQ_LAYOUT_BYTE_ALIGNED && layout != FLEXQ_LAYOUT_4_2)
    return fail(FLEXQ_ERR_INVALID_ARG, "layout=%d is not a weight layout", layout);
  int rc = check_gemm_shape(1, N, K, group_size);
  if (rc) return rc;
  const void* ptrs[] = {W_fp16, Wq_packed, W_scales_fp16};
  const char* names[] = {"W_fp16", "Wq_packed", "W_scales_fp16"};
  if ((rc = check_ptrs(3, ptrs, names))) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const long long G = K / group_size;
  const long long n1 = static_cast<long long>(N) * G;
  flexq::weight_scale_kernel<<<static_cast<unsigned>((n1 + 255) / 256), 256, 0, s>>>(
      static_cast<const __half*>(W_fp16), static_cast<__half*>(W_scales_fp16), N, K, group_size);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "weight_scale_kernel launch");
  const long long n2 = static_cast<long long>(N) * (K / 128) * 2;
  if (layout == FLEXQ_LAYOUT_4_2)
    flexq::weight_pack42_kernel<<<static_cast<unsigned>((n2 + 255) / 256), 256, 0, s>>>(
        static_cast<const __half*>(W_fp16), static_cast<const __half*>(W_scales_fp16),
        static_cast<uint8_t*>(Wq_packed), N, K, group_size);
  else
    flexq::weight_pack_kernel<<<static_cast<unsigned>((n2 + 255) / 256), 256, 0, s>>>(
        static_cast<const __half*>(W_fp16), static_cast<const __half*>(W_scales_fp16),
        static_cast<uint8_t*>(Wq_packed), N, K, group_size);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "weight_pack_kernel launch");
  return ok();
}

int flexq_debug_export_canonical(int N, int K, int layout, const void* Wq_packed,
                                 void* W_canonical, void* stream) {
  if (layout != FLEXQ_LAYOUT_BYTE_ALIGNED && layout != FLEXQ_LAYOUT_4_2)
    return fail(FLEXQ_ERR_INVALID_ARG, "layout=%d is not a weight layout", layout);
  int rc = check_gemm_shape(1, N, K, 128);
  if (rc) return rc;
  const void* ptrs[] = {Wq_packed, W_canonical};
  const char* names[] = {"Wq_packed", "W_canonical"};
  if ((rc = check_ptrs(2, ptrs, names))) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const dim3 grid(static_cast<unsigned>(K / 128), static_cast<unsigned>(N / 128));
  const uint8_t* wp = static_cast<const uint8_t*>(Wq_packed);
  uint8_t* out = static_cast<uint8_t*>(W_canonical);
  if (layout == FLEXQ_LAYOUT_4_2)
    flexq::export_canonical_kernel<1><<<grid, flexq::kTileRows, 0, s>>>(wp, out, K);
  else
    flexq::export_canonical_kernel<0><<<grid, flexq::kTileRows, 0, s>>>(wp, out, K);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "export_canonical_kernel launch");
  return ok();
}

int flexq_quantize_act(int M, int K, int group_size, int bits, const void* X_fp16, int8_t* Xq,
                       void* X_scales_fp16, void* stream) {
  if (M < 0 || K <= 0) return fail(FLEXQ_ERR_INVALID_ARG, "sizes must be M >= 0, K > 0 (M=%d K=%d)", M, K);
  if (bits != 6 && bits != 8) return fail(FLEXQ_ERR_INVALID_ARG, "bits=%d is not 6 or 8", bits);
  if (!valid_gs(group_size)) return fail(FLEXQ_ERR_UNSUPPORTED, "group_size %d not in {32,64,128,256}", group_size);
  if (K % group_size) return fail(FLEXQ_ERR_UNSUPPORTED, "K=%d is not a multiple of group_size %d", K, group_size);
  if (M == 0) return ok();               // empty batch: nothing to read or write
  const void* ptrs[] = {X_fp16, Xq, X_scales_fp16};
  const char* names[] = {"X_fp16", "Xq", "X_scales_fp16"};
  int rc = check_ptrs(3, ptrs, names);
  if (rc) return rc;
  DeviceState* st = nullptr;
  if ((rc = device_state(&st))) return rc;
  // Grid: whole rows per step (the thread count a multiple of the row length
  // in 16-byte chunks, cpr = K/8), at most one resident wave; each thread
  // keeps four loads in flight and strides over the remaining rows.
  const int cpr = K / 8;
  if (static_cast<long long>(M) * cpr >= (1ll << 31))
    return fail(FLEXQ_ERR_UNSUPPORTED, "M*K/8 = %lld chunks exceeds 2^31", static_cast<long long>(M) * cpr);
  int per_sm = 0;
  cudaError_t oe = cudaSuccess;
  switch (group_size) {
    case 32: oe = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, flexq::quant_act_kernel<32>, 256, 0); break;
    case 64: oe = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, flexq::quant_act_kernel<64>, 256, 0); break;
    case 128: oe = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, flexq::quant_act_kernel<128>, 256, 0); break;
    default: oe = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, flexq::quant_act_kernel<256>, 256, 0); break;
  }
  if (oe != cudaSuccess || per_sm < 1) per_sm = 4;
  // blocks per group of whole rows: the smallest b with b*256 a multiple of cpr
  long long g = cpr, h = 256;                 // gcd(cpr, 256)
  while (h) { const long long r = g % h; g = h; h = r; }
  const long long unit_blocks = cpr / g;       // blocks that hold whole rows
  const long long unit_rows = unit_blocks * 256 / cpr;
  long long units = static_cast<long long>(st->sms) * per_sm / unit_blocks;
  if (units < 1) units = 1;
  const long long need_units = (M + unit_rows - 1) / unit_rows;
  if (units > need_units) units = need_units;
  const long long blocks = units * unit_blocks;
  const int rows_per_step = static_cast<int>(units * unit_rows);
  const int qmax = bits == 6 ? 31 : 127;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const uint4* x = static_cast<const uint4*>(X_fp16);
  uint2* q = reinterpret_cast<uint2*>(Xq);
  __half* xs = static_cast<__half*>(X_scales_fp16);
  const int ld = act_scales_ld(M);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(blocks), 1, 1);
  cfg.blockDim = dim3(256, 1, 1);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e;
  switch (group_size) {
    case 32: e = cudaLaunchKernelEx(&cfg, flexq::quant_act_kernel<32>, x, q, xs, M, cpr, rows_per_step, ld, qmax); break;
    case 64: e = cudaLaunchKernelEx(&cfg, flexq::quant_act_kernel<64>, x, q, xs, M, cpr, rows_per_step, ld, qmax); break;
    case 128: e = cudaLaunchKernelEx(&cfg, flexq::quant_act_kernel<128>, x, q, xs, M, cpr, rows_per_step, ld, qmax); break;
    default: e = cudaLaunchKernelEx(&cfg, flexq::quant_act_kernel<256>, x, q, xs, M, cpr, rows_per_step, ld, qmax); break;
  }
  if (e != cudaSuccess) return cuda_fail(e, "quant_act_kernel launch");
  return ok();
}

size_t flexq_gemm_workspace_bytes(int M, int N, int K, int group_size) {
  if (M <= 0 || N <= 0 || K <= 0 || N % 128 || K % 256 || !valid_gs(group_size) || K % group_size)
    return 0;
  const Plan p = make_plan(M, N, K, group_size, sm_count_or_default(), false);
  return workspace_bytes_for(p, M, N);
}

int flexq_gemm_w6a6(int M, int N, int K, int group_size, const int8_t* Xq, const void* X_scales,
                    const void* Wq_packed, const void* W_scales, void* Y_fp16, void* workspace,
                    size_t workspace_bytes, void* stream) {
  return gemm_common(M, N, K, group_size, Xq, X_scales, Wq_packed, W_scales, Y_fp16, nullptr,
                     false, workspace, workspace_bytes, stream);
}

int flexq_gemm_w6a8(int M, int N, int K, int group_size, const int8_t* Xq, const void* X_scales,
                    const void* Wq_packed, const void* W_scales, void* Y_fp16, void* workspace,
                    size_t workspace_bytes, void* stream) {
  return gemm_common(M, N, K, group_size, Xq, X_scales, Wq_packed, W_scales, Y_fp16, nullptr,
                     false, workspace, workspace_bytes, stream);
}

int flexq_gemm_static_scratch(int M, int N, int K, int group_size, int act_bits,
                              const int8_t* Xq, const void* X_scales, const void* Wq_packed,
                              const void* W_scales, void* Y_fp16, void* stream) {
  if (act_bits != 6 && act_bits != 8)
    return fail(FLEXQ_ERR_INVALID_ARG, "act_bits=%d is not 6 or 8", act_bits);
  int rc = check_gemm_shape(M, N, K, group_size);
  if (rc) return rc;
  if (M == 0) return ok();
  // every pointer is checked before anything is enqueued (the counter clear
  // below is the first work on the stream)
  const void* ptrs[] = {Xq, X_scales, Wq_packed, W_scales, Y_fp16};
  const char* names[] = {"Xq", "X_scales", "Wq_packed", "W_scales", "Y"};
  if ((rc = check_ptrs(5, ptrs, names))) return rc;
  DeviceState* st = nullptr;
  if ((rc = device_state(&st))) return rc;
  const size_t need = workspace_bytes_for(make_plan(M, N, K, group_size, st->sms, false), M, N);
  if (need > kStaticScratchBytes)
    return fail(FLEXQ_ERR_UNSUPPORTED,
                "this shape needs %zu bytes of split-K scratch, more than the %zu of the "
                "static scratch; use flexq_gemm_w6a6/w6a8 with a workspace", need,
                kStaticScratchBytes);
  void* scratch = nullptr;
  if ((rc = static_scratch(&scratch))) return rc;
  if (need > 0) {
    // the arrival counters must start at zero; earlier calls leave them zero
    // unless one of them gave up on a wait, so clear them every time
    cudaError_t e = cudaMemsetAsync(scratch, 0, kCounterBytes, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "clearing the static scratch counters");
  }
  return gemm_common(M, N, K, group_size, Xq, X_scales, Wq_packed, W_scales, Y_fp16, nullptr,
                     false, scratch, kStaticScratchBytes, stream);
}

size_t flexq_linear_workspace_bytes(int M, int N, int K, int group_size) {
  if (M <= 0 || N <= 0 || K <= 0 || N % 128 || K % 256 || !valid_gs(group_size) || K % group_size)
    return 0;
  const Plan p = make_plan(M, N, K, group_size, sm_count_or_default(), false);
  return linear_layout(p, M, N, K, group_size).total;
}

int flexq_linear_launches(int M, int N, int K, int group_size) {
  if (M <= 0 || N <= 0 || K <= 0 || N % 128 || K % 256 || !valid_gs(group_size) || K % group_size)
    return 0;
  const Plan p = make_plan(M, N, K, group_size, sm_count_or_default(), false);
  return linear_layout(p, M, N, K, group_size).fused ? 1 : 2;
}

int flexq_debug_force_linear_route(int route) {
  if (route < 0 || route > 2) return fail(FLEXQ_ERR_INVALID_ARG, "route %d not in {0, 1, 2}", route);
  g_force_linear_route.store(route);
  return ok();
}

int flexq_linear_w6a6(int M, int N, int K, int group_size, const void* X_fp16,
                      const void* Wq_packed, const void* W_scales, void* Y_fp16, void* workspace,
                      size_t workspace_bytes, void* stream) {
  return linear_common(M, N, K, group_size, 6, X_fp16, Wq_packed, W_scales, Y_fp16, workspace,
                       workspace_bytes, stream);
}

int flexq_linear_w6a8(int M, int N, int K, int group_size, const void* X_fp16,
                      const void* Wq_packed, const void* W_scales, void* Y_fp16, void* workspace,
                      size_t workspace_bytes, void* stream) {
  return linear_common(M, N, K, group_size, 8, X_fp16, Wq_packed, W_scales, Y_fp16, workspace,
                       workspace_bytes, stream);
}

int flexq_gemm_layout(int M, int N, int K, int group_size, int act_bits, int layout,
                      const int8_t* Xq, const void* X_scales, const void* Wq_packed,
                      const void* W_scales, void* Y_fp16, void* workspace, size_t workspace_bytes,
                      void* stream) {
  if (act_bits != 6 && act_bits != 8)
    return fail(FLEXQ_ERR_INVALID_ARG, "act_bits=%d is not 6 or 8", act_bits);
  if (layout != FLEXQ_LAYOUT_BYTE_ALIGNED && layout != FLEXQ_LAYOUT_4_2)
    return fail(FLEXQ_ERR_INVALID_ARG, "layout=%d is not a weight layout", layout);
  return gemm_common(M, N, K, group_size, Xq, X_scales, Wq_packed, W_scales, Y_fp16, nullptr,
                     false, workspace, workspace_bytes, stream, layout);
}

int flexq_linear_layout(int M, int N, int K, int group_size, int act_bits, int layout,
                        const void* X_fp16, const void* Wq_packed, const void* W_scales,
                        void* Y_fp16, void* workspace, size_t workspace_bytes, void* stream) {
  if (layout != FLEXQ_LAYOUT_BYTE_ALIGNED && layout != FLEXQ_LAYOUT_4_2)
    return fail(FLEXQ_ERR_INVALID_ARG, "layout=%d is not a weight layout", layout);
  return linear_common(M, N, K, group_size, act_bits, X_fp16, Wq_packed, W_scales, Y_fp16,
                       workspace, workspace_bytes, stream, layout);
}

int flexq_debug_check_quantizer(unsigned long long* mismatches, unsigned int* first_mismatch) {
  if (!mismatches || !first_mismatch)
    return fail(FLEXQ_ERR_INVALID_ARG, "mismatches and first_mismatch must not be NULL");
  unsigned long long* d_count = nullptr;
  unsigned* d_first = nullptr;
  // test hook only: the library's product entry points never allocate
  cudaError_t e = cudaMalloc(&d_count, sizeof(unsigned long long) + 4 * sizeof(unsigned));
  if (e != cudaSuccess) return cuda_fail(e, "cudaMalloc");
  d_first = reinterpret_cast<unsigned*>(d_count + 1);
  e = cudaMemset(d_count, 0, sizeof(unsigned long long) + 4 * sizeof(unsigned));
  // every positive finite FP16 scale (0x0001 .. 0x7BFF), 1024 scales per launch
  for (unsigned s0 = 1; e == cudaSuccess && s0 <= 0x7BFFu; s0 += 1024) {
    const unsigned n_s = (0x7BFFu - s0 + 1 < 1024u) ? 0x7BFFu - s0 + 1 : 1024u;
    const unsigned long long threads = static_cast<unsigned long long>(n_s) * 65536ull;
    flexq::check_quantizer_kernel<<<static_cast<unsigned>((threads + 255) / 256), 256>>>(
        s0, n_s, d_count, d_first);
    e = cudaGetLastError();
  }
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  if (e == cudaSuccess) e = cudaMemcpy(mismatches, d_count, sizeof(unsigned long long), cudaMemcpyDeviceToHost);
  if (e == cudaSuccess) e = cudaMemcpy(first_mismatch, d_first, 3 * sizeof(unsigned), cudaMemcpyDeviceToHost);
  cudaFree(d_count);
  if (e != cudaSuccess) return cuda_fail(e, "quantizer check");
  return ok();
}

int flexq_debug_group_partials(int M, int N, int K, int group_size, const int8_t* Xq,
                               const void* Wq_packed, int32_t* P, void* stream) {
  return gemm_common(M, N, K, group_size, Xq, nullptr, Wq_packed, nullptr, nullptr, P, true,
                     nullptr, 0, stream);
}

int flexq_gemm_plan(int M, int N, int K, int group_size, int* tile_tokens, int* k_split,
                    int* ctas) {
  int rc = check_gemm_shape(M, N, K, group_size);
  if (rc) return rc;
  if (M == 0) {
    if (tile_tokens) *tile_tokens = 0;
    if (k_split) *k_split = 0;
    if (ctas) *ctas = 0;
    return ok();
  }
  const Plan p = make_plan(M, N, K, group_size, sm_count_or_default(), false);
  if (tile_tokens) *tile_tokens = p.T;
  if (k_split) *k_split = p.split;
  if (ctas) *ctas = static_cast<int>(p.ctas);
  return ok();
}

int flexq_debug_force_plan(int tile_tokens, int k_split) {
  if (!(tile_tokens == 0 || tile_tokens == 16 || tile_tokens == 32 || tile_tokens == 64 ||
        tile_tokens == 128))
    return fail(FLEXQ_ERR_INVALID_ARG, "tile_tokens %d not in {0,16,32,64,128}", tile_tokens);
  if (k_split < 0 || k_split > 8) return fail(FLEXQ_ERR_INVALID_ARG, "k_split %d not in 0..8", k_split);
  g_force_tokens.store(tile_tokens);
  g_force_split.store(k_split);
  return ok();
}

int flexq_set_wait_limit_ns(uint64_t limit_ns) {
  if (limit_ns == 0) return fail(FLEXQ_ERR_INVALID_ARG, "wait limit must be > 0");
  g_wait_limit_ns.store(limit_ns);
  return ok();
}

int flexq_debug_inject_stall(int enable) {
  g_inject_stall.store(enable ? 1 : 0);
  return ok();
}

int flexq_get_device_status(void* stream) {
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  DeviceState* st = nullptr;
  int rc = device_state(&st);
  if (rc) return rc;
  unsigned int h[4] = {0, 0, 0, 0};
  e = cudaMemcpy(h, st->status, sizeof(h), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "reading the device status word");
  if (h[0] == 0) return ok();
  e = cudaMemset(st->status, 0, sizeof(h));
  if (e != cudaSuccess) return cuda_fail(e, "clearing the device status word");
  static const char* roles[] = {"producer", "mma", "unpack", "?", "epilogue (partials)",
                                "epilogue (scales)"};
  return fail(static_cast<int>(h[0]), "device wait timed out in the %s role of block %u",
              h[1] < 6 ? roles[h[1]] : "?", h[2]);
}

size_t flexq_gemm_group_workspace_bytes(int M, int K, int group_size, int n_layers,
                                        const int* N) {
  if (M <= 0 || K <= 0 || n_layers < 1 || n_layers > flexq::kMaxLayers || !N) return 0;
  for (int l = 0; l < n_layers; ++l)
    if (N[l] <= 0 || N[l] % 128 || K % 256 || !valid_gs(group_size) || K % group_size) return 0;
  return group_gemm_bytes(M, N, n_layers, K, group_size, sm_count_or_default(), nullptr);
}

size_t flexq_linear_group_workspace_bytes(int M, int K, int group_size, int n_layers,
                                          const int* N) {
  if (M <= 0 || K <= 0 || n_layers < 1 || n_layers > flexq::kMaxLayers || !N) return 0;
  for (int l = 0; l < n_layers; ++l)
    if (N[l] <= 0 || N[l] % 128 || K % 256 || !valid_gs(group_size) || K % group_size) return 0;
  return group_linear_layout(M, N, n_layers, K, group_size, sm_count_or_default()).total;
}

int flexq_group_plan(int M, int K, int group_size, int n_layers, const int* N, int* tile_tokens,
                     int* k_split, int* ctas, int* launches) {
  if (M <= 0 || K <= 0 || n_layers < 1 || n_layers > flexq::kMaxLayers || !N)
    return fail(FLEXQ_ERR_INVALID_ARG, "M=%d K=%d n_layers=%d", M, K, n_layers);
  for (int l = 0; l < n_layers; ++l) {
    int rc = check_gemm_shape(M, N[l], K, group_size);
    if (rc) return rc;
  }
  const GroupLinearLayout L = group_linear_layout(M, N, n_layers, K, group_size, sm_count_or_default());
  if (tile_tokens) *tile_tokens = L.plan.T;
  if (k_split) *k_split = L.plan.T <= 64 ? L.plan.split : 0;
  if (ctas) *ctas = L.plan.T <= 64 ? static_cast<int>(L.plan.ctas) : 0;
  if (launches) *launches = L.fused ? 1 : 1 + (L.plan.T <= 64 ? 1 : n_layers);
  return ok();
}

int flexq_gemm_group(int M, int K, int group_size, int act_bits, const int8_t* Xq,
                     const void* X_scales, int n_layers, const flexq_layer_t* layers,
                     void* workspace, size_t workspace_bytes, void* stream) {
  return gemm_group_common(M, K, group_size, act_bits, Xq, X_scales, n_layers, layers, workspace,
                           workspace_bytes, stream);
}

int flexq_linear_group(int M, int K, int group_size, int act_bits, const void* X_fp16,
                       int n_layers, const flexq_layer_t* layers, void* workspace,
                       size_t workspace_bytes, void* stream) {
  return linear_group_common(M, K, group_size, act_bits, X_fp16, n_layers, layers, workspace,
                             workspace_bytes, stream);
}

#ifdef FLEXQ_TRACE
// Trace builds only: per-role loop/wait cycles of CTA 0 and of the middle CTA
// ([2][4][4]) and the per-CTA timeline ([8192][8]) of the last launch.
int flexq_debug_read_roles(long long* host, size_t count) {
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceSynchronize");
  const size_t n = sizeof(flexq::g_flexq_role) / sizeof(long long);
  e = cudaMemcpyFromSymbol(host, flexq::g_flexq_role, (count < n ? count : n) * sizeof(long long));
  if (e != cudaSuccess) return cuda_fail(e, "reading the role trace");
  return ok();
}

int flexq_debug_read_cta_times(unsigned long long* host, size_t count) {
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceSynchronize");
  const size_t n = sizeof(flexq::g_flexq_cta_times) / sizeof(unsigned long long);
  e = cudaMemcpyFromSymbol(host, flexq::g_flexq_cta_times,
                           (count < n ? count : n) * sizeof(unsigned long long));
  if (e != cudaSuccess) return cuda_fail(e, "reading the CTA timeline");
  return ok();
}
#endif

}  // extern "C"
