// flexq_gemm.cuh -- the W6A6 / W6A8 group GEMM on tcgen05 tensor cores.
//
// What it computes (FlexQ paper, arXiv abstract; drgamma blog, "Bridging
// Software and Hardware with BTC"): for every K-group g the exact integer
// partial P_g[m,n] = sum_{k in g} qa[m,k] * qw[n,k], recombined with the
// group scales, Y[m,n] = sum_g P_g[m,n] * sa[m,g] * sw[n,g], dequantization
// fused into the GEMM.  The pages' kernel decomposes 6-bit operands into
// 1-bit planes for binary tensor cores; on sm_100a one exact int8 MMA
// replaces all plane products, so here the 6-bit weight codes are unpacked
// losslessly to int8 and multiplied with tcgen05.mma.kind::i8.
//
// Orientation ("swap AB"): the MMA's M side is 128 weight rows, its N side
// is T tokens.  Per CTA: one 128-row weight tile, one T-token tile and a
// contiguous, group-aligned range of K.  With a K split, the `split` CTAs of
// an output tile write FP32 partial tiles to a workspace and the last one to
// finish adds them in split order (see the teardown).
//
// The pipeline advances in stages of 256 codes of K (two 128 x 128 weight
// tiles).
//
// Warp roles (all pipeline waits are bounded, see mbar_wait):
//   warp 0      producer: per stage, one 24576-byte bulk copy of two
//               consecutive packed weight tiles into a STAGES-deep weight
//               ring (a stage is free again once the unpack warps hold its
//               bytes) and two TMA boxes of the int8 activations (T rows x
//               128 B each, 128-byte swizzle) into an activation ring of
//               kXSlots slots (free again after the MMAs that read it); per
//               8 groups, the group scales;
//   warp 1      TMEM allocator and MMA issuer: 8 MMAs (K = 32 each) per
//               stage into the int32 partial buffer of the current group
//               (kPBufs buffers of T columns), one commit per group;
//   warps 2..5  unpack: each thread owns one weight row, turns its 192 packed
//               bytes into 256 int8 codes (code * 4: the 6-bit field in the
//               top of each byte) and stores them into a TMEM "A" slot
//               (kASlots slots of 64 columns);
//   warps 6..   epilogue: per group, load the int32 partials from TMEM,
//               release the buffer, and accumulate
//               acc += float(P) * (sw[n,g]/4 * sa[m,g]) in FP32 registers;
//               at the end store FP16 (or hand the partial tile to the
//               split-K reduction).
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <cstdint>
#include <type_traits>

#include "flexq_ptx.cuh"
#include "flexq_quant.cuh"

namespace flexq {

constexpr int kTileRows = 128;        // weight rows per tile (MMA M)
constexpr int kKBlock = 128;          // codes per K block
constexpr int kWTileBytes = 12288;    // packed bytes of a 128 x 128 tile
constexpr int kStatusTimeout = 5;     // == FLEXQ_ERR_DEVICE_TIMEOUT

struct GemmArgs {
  const uint8_t* wp;       // packed weights, device form
  __half* y;               // [M, N] output (GEMM mode)
  int32_t* p;              // [G, M, N] partials (debug mode)
  const __half* x;         // [M, K] FP16 activations (fused quantization only)
  const __half* sa;        // activation scales [G][sa_ld] (wide kernel)
  const __half* sw;        // weight scales [G][N] (wide kernel)
  int sa_ld;
  int qmax;                // activation code range Q (fused quantization only)
  int fq_offset;           // byte offset of the fused quantizer's smem block
  float* ws_part;          // split-K partial tiles [tiles][split][T][128] (split > 1)
  unsigned int* ws_cnt;    // split-K arrival counters [tiles], zero between calls
  unsigned int* status;    // device status word [4]
  unsigned long long wait_limit_ns;
  int M, N, K, gs;
  int tiles_n;             // weight tiles along N (N / 128)
  int n_full;              // output tiles 0 .. n_full-1 run whole (no K split) ...
  int split;               // ... the later ones are split `split` ways along K
  int ctrl_offset;         // byte offset of the control block in smem
  int stall;               // test hook: withhold the first stage
};

// The layers of one launch of gemm_w6ax_kernel: one, or up to kMaxLayers
// layers that read the same activations (a grouped launch: the q, k and v
// projections, or gate and up), each with its own packed weights, scales,
// output and K-split plan.  Work units are numbered layer after layer.
constexpr int kMaxLayers = 4;
struct LayerTable {
  CUtensorMap sw[kMaxLayers];      // weight scales [G][N_l], box 128 rows x 8 groups
  const uint8_t* wp[kMaxLayers];   // packed weights, device form
  __half* y[kMaxLayers];           // [M, N_l] FP16 outputs
  long long part0[kMaxLayers];     // first float of the layer's split-K partial tiles
  int N[kMaxLayers];
  int unit0[kMaxLayers + 1];       // first work unit of each layer; unit0[n] = all units
  int n_full[kMaxLayers];          // output tiles run whole (the rest split `split` ways)
  int split[kMaxLayers];
  int tile0[kMaxLayers];           // first split-K arrival counter of each layer
  int n_layers;
};

template <int T>
struct GemmCfg {
  // each epilogue warp owns one TMEM lane quarter (32 weight rows) and kCols
  // tokens; T = 128 uses 16 epilogue warps so that four warps per scheduler
  // hide the latency of the TMEM loads and conversions
  static constexpr int kCols = T < 32 ? T : 32;
  static constexpr int kEpiWarps = 4 * (T / kCols);
  static constexpr int kThreads = (6 + kEpiWarps) * 32;
  static constexpr int kStages = (T == 64) ? 2 : 3;
  static constexpr int kMinBlocks = (T <= 64) ? 2 : 1;
  static constexpr int kMaxSplit = (T == 16) ? 8 : (T == 32) ? 6 : 4;
  static constexpr int kKStage = 2 * kKBlock;            // codes of K per stage
  static constexpr int kXsHalf = T * 128;                // one activation box
  static constexpr int kXsBytes = 2 * kXsHalf;
  static constexpr int kWStageBytes = 2 * kWTileBytes;
  static constexpr int kStageBytes = kXsBytes + kWStageBytes;
  // activation boxes have a ring of their own, released by the MMA commit,
  // while a weight stage is free once the unpack warps hold its bytes in
  // registers; with more activation slots than stages (16-token tiles, whose
  // boxes are small) a weight stage is refilled without waiting for the MMA
  // of the stage that last used it
  static constexpr int kXSlots = (T == 16) ? 6 : kStages;
  // scale ring: one slot holds 8 groups ("octet") of activation scales for
  // the T tokens ([8][T] fp16) and of weight scales for the 128 rows
  // ([8][128] fp16), each brought by one TMA box
  static constexpr int kScSlots = 3;
  static constexpr int kScSaBytes = 8 * T * 2;
  static constexpr int kScSlotBytes = kScSaBytes + 8 * 128 * 2;
  static constexpr int kMainBytes =
      kXSlots * kXsBytes + kStages * kWStageBytes + kScSlots * kScSlotBytes;
  // TMEM: int32 partial buffers (one per group in flight), then the A slots
  // (64 columns = 256 int8 codes per row each).  Two CTAs share an SM for
  // T <= 64, so those stay within 256 columns; T = 128 takes all 512 for
  // three partial buffers and two A slots.
  static constexpr int kPBufs = (T == 16) ? 4 : (T == 128) ? 3 : 2;
  static constexpr int kASlots = (T == 128) ? 2 : kStages;
  static constexpr int kPCol0 = 0;
  static constexpr int kACol0 = kPBufs * T;
  static constexpr int kACols = 64;
  static constexpr int kTmemCols = (kACol0 + kACols * kASlots <= 256) ? 256 : 512;
  static_assert(kACol0 + kACols * kASlots <= kTmemCols, "TMEM budget");
  static_assert(kMinBlocks == 1 || kTmemCols <= 256, "two CTAs per SM share 512 columns");
};

template <int T>
struct GemmCtrl {
  uint64_t full[GemmCfg<T>::kStages];
  uint64_t empty[GemmCfg<T>::kStages];
  uint64_t x_empty[GemmCfg<T>::kXSlots];
  uint64_t a_full[GemmCfg<T>::kASlots];
  uint64_t a_empty[GemmCfg<T>::kASlots];
  uint64_t p_full[GemmCfg<T>::kPBufs];
  uint64_t p_empty[GemmCfg<T>::kPBufs];
  uint64_t s_full[GemmCfg<T>::kScSlots];
  uint64_t s_empty[GemmCfg<T>::kScSlots];
  uint64_t done;
  uint32_t tmem_base;
  uint32_t is_last;        // split-K: this CTA reduces the output tile
  // per epilogue warp: its tokens' activation scales of the current octet, FP32
  alignas(16) float sa[GemmCfg<T>::kEpiWarps][8][GemmCfg<T>::kCols];
};

// A ring position: index into a ring of R slots and the parity of the
// current round; advancing past the last slot flips the parity.
template <int R>
struct RingPos {
  uint32_t idx = 0, phase = 0;
  __device__ __forceinline__ void next() {
    const uint32_t n = idx + 1;
    const uint32_t wrap = (n == static_cast<uint32_t>(R)) ? 1u : 0u;
    idx = wrap ? 0u : n;
    phase ^= wrap;
  }
};

// Optional pipeline trace (compile with -DFLEXQ_TRACE).  Every CTA records
// %globaltimer at entry (0), after set-up (1), after its roles' loops (2), at
// exit (3), after the TMEM release (5), after the split-K partial store (6)
// and before the output store (7), with its SM id in slot 4.  CTA 0 and the
// CTA in the middle of the grid also record, per role (producer, MMA, unpack
// warp of lane quarter 0, first epilogue warp), the cycles spent in the role
// loop, the cycles spent waiting on barriers and the iteration count:
// g_flexq_role[which CTA][role][0..2].
#ifdef FLEXQ_TRACE
__device__ unsigned long long g_flexq_cta_times[8192][8];
__device__ long long g_flexq_role[2][4][4];
#define FLEXQ_CTA_TIME(slot)                                                   \
  do {                                                                         \
    const unsigned cta_ = blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z); \
    if (threadIdx.x == 0 && cta_ < 8192) {                                     \
      g_flexq_cta_times[cta_][slot] = global_timer_ns();                       \
      unsigned smid_;                                                          \
      asm volatile("mov.u32 %0, %%smid;" : "=r"(smid_));                       \
      g_flexq_cta_times[cta_][4] = smid_;                                      \
    }                                                                          \
  } while (0)
#define FLEXQ_ROLE_CLOCK long long fx_wait_ = 0, fx_t0_ = clock64()
#define FLEXQ_WAIT(expr)                       \
  ({                                           \
    const long long fx_w0_ = clock64();        \
    const bool fx_r_ = (expr);                 \
    fx_wait_ += clock64() - fx_w0_;            \
    fx_r_;                                     \
  })
#define FLEXQ_ROLE_DONE(role, iters)                                             \
  do {                                                                           \
    const unsigned cta_ = blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z); \
    const unsigned mid_ = (gridDim.x * gridDim.y * gridDim.z) / 2;              \
    if (cta_ == 0 || cta_ == mid_) {                                             \
      const int w_ = cta_ == 0 ? 0 : 1;                                          \
      g_flexq_role[w_][role][0] = clock64() - fx_t0_;                            \
      g_flexq_role[w_][role][1] = fx_wait_;                                      \
      g_flexq_role[w_][role][2] = (iters);                                       \
    }                                                                            \
  } while (0)
#else
#define FLEXQ_CTA_TIME(slot) \
  do {                       \
  } while (0)
#define FLEXQ_ROLE_CLOCK
#define FLEXQ_WAIT(expr) (expr)
#define FLEXQ_ROLE_DONE(role, iters) \
  do {                               \
  } while (0)
#endif

__device__ __forceinline__ void record_status(unsigned int* status, int code,
                                              int where) {
  if (atomicCAS(status, 0u, static_cast<unsigned>(code)) == 0u) {
    status[1] = static_cast<unsigned>(where);
    status[2] = blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z);
  }
}

// Otherwise lane 0 waits (the other lanes park at the warp barrier instead of
// polling the mbarrier); the warp agrees on the outcome.  The warp barrier
// orders the waiting lane's acquire before every lane's subsequent reads.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity,
                                          uint64_t limit) {
  // fast path: the phase is usually complete already; every lane probes it
  // (each probe acquires for its own lane) and one vote settles it
  if (__all_sync(0xffffffffu, mbar_test_wait(smem_u32(bar), parity))) return true;
  bool ok = true;
  if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, limit);
  ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
  __syncwarp();
  return ok;
}

// One 16-code block of the device form (three words, see weight_pack_kernel)
// -> four int8x4 words in k order, each byte code * 4.  Bytes of w0..w2 hold
// codes 0..11 in their bits [7:2]; their bits [1:0] hold the 2-bit pieces of
// codes 12..15 (w0: bits 1:0 of the code, w1: bits 3:2, w2: bits 5:4).  The
// pieces occupy disjoint bits of each byte, so adding them cannot carry.
__device__ __forceinline__ void unpack_block(uint32_t w0, uint32_t w1, uint32_t w2,
                                             uint32_t* out) {
  out[0] = w0 & 0xFCFCFCFCu;
  out[1] = w1 & 0xFCFCFCFCu;
  out[2] = w2 & 0xFCFCFCFCu;
  const uint32_t p0 = w0 & 0x03030303u, p1 = w1 & 0x03030303u, p2 = w2 & 0x03030303u;
  out[3] = ((p2 * 4u + p1) * 4u + p0) * 4u;
}

// One 16-code block of the "4+2" form (nibble words n0, n1 and the 2-bit
// word l, see weight_pack42_kernel) -> four int8x4 words in k order, each
// byte code * 4 = h << 4 | l << 2: the nibbles in bits 7:4, the 2-bit pieces
// shifted into bits 3:2.
__device__ __forceinline__ void unpack_block42(uint32_t n0, uint32_t n1, uint32_t l,
                                               uint32_t* out) {
  out[0] = (n0 & 0xF0F0F0F0u) | ((l << 2) & 0x0C0C0C0Cu);
  out[1] = ((n0 << 4) & 0xF0F0F0F0u) | (l & 0x0C0C0C0Cu);
  out[2] = (n1 & 0xF0F0F0F0u) | ((l >> 2) & 0x0C0C0C0Cu);
  out[3] = ((n1 << 4) & 0xF0F0F0F0u) | ((l >> 4) & 0x0C0C0C0Cu);
}

// The 24 words of one row's 96 packed bytes of a 128-code tile (six 16-byte
// chunks) -> its 128 int8 codes * 4, in k order, for either weight layout.
template <int LAYOUT>
__device__ __forceinline__ void unpack_row_tile(const uint32_t (&w)[24], uint32_t (&out)[32]) {
#pragma unroll
  for (int b = 0; b < 8; ++b) {
    if (LAYOUT == 0)
      unpack_block(w[3 * b], w[3 * b + 1], w[3 * b + 2], &out[4 * b]);
    else
      unpack_block42(w[2 * b], w[2 * b + 1], w[16 + b], &out[4 * b]);
  }
}

// The device form of packed weights (either layout) -> the canonical form:
// row-major, codes 4j .. 4j+3 of a row as the 24-bit word
// u0 | u1 << 6 | u2 << 12 | u3 << 18 (u_i = code_i & 0x3F) in bytes 3j .. 3j+2,
// little endian.  One thread per weight row of a 128 x 128 tile: it reads the
// row's six 16-byte chunks, unpacks them as the GEMM does (code * 4 per byte)
// and writes the row's 96 canonical bytes of the tile.
template <int LAYOUT>
__global__ void __launch_bounds__(kTileRows) export_canonical_kernel(
    const uint8_t* __restrict__ wp, uint8_t* __restrict__ out, int K) {
  const int kb = blockIdx.x, nt = blockIdx.y, r = threadIdx.x;
  const int KB = K / kKBlock;
  const uint4* tile =
      reinterpret_cast<const uint4*>(wp + (static_cast<size_t>(nt) * KB + kb) * kWTileBytes);
  uint32_t w[24];
#pragma unroll
  for (int j = 0; j < 6; ++j) {
    const uint4 v = __ldg(tile + j * kTileRows + r);
    w[4 * j] = v.x; w[4 * j + 1] = v.y; w[4 * j + 2] = v.z; w[4 * j + 3] = v.w;
  }
  uint32_t c[32];
  unpack_row_tile<LAYOUT>(w, c);
  uint32_t o[24];
#pragma unroll
  for (int q4 = 0; q4 < 8; ++q4) {
    uint32_t t[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t v = c[4 * q4 + i];                // four codes * 4, one per byte
      t[i] = ((v >> 2) & 0x3Fu) | (((v >> 10) & 0x3Fu) << 6) | (((v >> 18) & 0x3Fu) << 12) |
             (((v >> 26) & 0x3Fu) << 18);
    }
    o[3 * q4] = t[0] | (t[1] << 24);
    o[3 * q4 + 1] = (t[1] >> 8) | (t[2] << 16);
    o[3 * q4 + 2] = (t[2] >> 16) | (t[3] << 8);
  }
  uint4* dst = reinterpret_cast<uint4*>(out + (static_cast<size_t>(nt) * kTileRows + r) *
                                                  (static_cast<size_t>(K) * 3 / 4) +
                                        static_cast<size_t>(kb) * 96);
#pragma unroll
  for (int j = 0; j < 6; ++j) dst[j] = make_uint4(o[4 * j], o[4 * j + 1], o[4 * j + 2], o[4 * j + 3]);
}

// ---------------------------------------------------------------------------
// Fused activation quantization (FUSEDQ, token tiles of 16 rows): the kernel
// reads the FP16 activations itself.  At stage i unpack warp q quantizes rows
// m0, m0 + 4, ... with m0 = (q - i * Mt) mod 4 (fq_row0) of the stage's 256
// codes of K -- lane l owns codes
// 8l .. 8l+7, a group is gs/8 lanes -- by the code rule of the activation
// quantizer (flexq_quant.cuh), and stores
//   * the int8 codes into the stage's activation tile, in the layout the TMA
//     would have written: row r of a 128-code block at r * 128 bytes, its
//     16-byte chunk c at position c ^ (r % 8) (128-byte swizzle);
//   * the FP16 group scales into a ring of per-stage scale slots ([8][T],
//     group within the stage x token), read by the epilogue.
// Rows past Mt are never written: their codes multiply a zero scale.
// ---------------------------------------------------------------------------
constexpr int kQaSlots = 8;           // per-stage activation-scale slots
constexpr int kQaRowsTogether = 1;    // rows whose arithmetic interleaves

template <int T>
struct FusedQLayout {
  static constexpr int kSlotHalves = 8 * T;
  static constexpr int kBytes = 2 * kQaSlots * 8 + kQaSlots * kSlotHalves * 2;
};

// First row of unpack warp q at stage i: the stage's (stage, row) pairs are
// dealt to the four warps in turn, so a batch of one or two rows spreads its
// quantization over all four warps across consecutive stages instead of
// loading one warp with every stage.
__device__ __forceinline__ int fq_row0(int q, int i, int Mt) {
  return (q - (i * Mt) % 4 + 4) & 3;
}

// FP16 rows m0 + 4r (r < R, below Mt) of codes k0 .. k0+255, 16 bytes per lane.
template <int R>
__device__ __forceinline__ void load_act_rows(uint4 (&xv)[R], const __half* __restrict__ xt,
                                              int Mt, int K, int m0, int k0, int lane) {
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const int m = m0 + 4 * r;
    xv[r] = make_uint4(0u, 0u, 0u, 0u);
    if (m < Mt)
      xv[r] = __ldg(reinterpret_cast<const uint4*>(xt + static_cast<size_t>(m) * K + k0) + lane);
  }
}

// RG rows m0, m0 + 4, ... at once, by the activation quantizer's route
// (group_scale_fast, quantize8).
template <int T, int RG>
__device__ __forceinline__ void quantize_act_group(const uint4* raw, int Mt, int m0, int lanes,
                                                   int grp, int qmax, uint8_t* xs,
                                                   __half* qa_slot, int lane) {
  const float fq = static_cast<float>(qmax);
  const float rq = __frcp_rn(fq);
  const int kb = lane >> 4;                              // 128-code block of the stage
  const int chunk = (lane & 15) >> 1;                    // 16-byte chunk in the block
  const int half8 = (lane & 1) * 8;                      // byte offset in the chunk
  float v[RG][8], amax[RG];
#pragma unroll
  for (int r = 0; r < RG; ++r) {
    const __half2* h2 = reinterpret_cast<const __half2*>(&raw[r]);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __half22float2(h2[i]);
      v[r][2 * i] = f.x;
      v[r][2 * i + 1] = f.y;
    }
    amax[r] = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) amax[r] = fmaxf(amax[r], fabsf(v[r][i]));
  }
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
#pragma unroll
    for (int r = 0; r < RG; ++r) {
      const float o = __shfl_xor_sync(0xffffffffu, amax[r], off);
      if (off < lanes) amax[r] = fmaxf(amax[r], o);
    }
  }
#pragma unroll
  for (int r = 0; r < RG; ++r) {
    const int m = m0 + 4 * r;
    const __half s16 = group_scale_fast(amax[r], fq, rq);
    const float sc = __half2float(s16);
    const uint2 codes = quantize8(v[r], sc, rcp_estimate(sc), qmax);
    if (m < Mt) {
      *reinterpret_cast<uint2*>(xs + kb * (T * 128) + m * 128 + ((chunk ^ (m & 7)) << 4) + half8) =
          codes;
      if ((lane & (lanes - 1)) == 0) qa_slot[grp * T + m] = s16;
    }
  }
}

// This warp's R rows of one stage (m0 + 4r), RG at a time.
template <int T, int R, int RG>
__device__ __forceinline__ void quantize_act_rows(uint4 (&xv)[R], int Mt, int m0, int gs_log2,
                                                  int qmax, uint8_t* xs, __half* qa_slot,
                                                  int lane) {
  static_assert(R % RG == 0, "row groups");
  const int lanes = (1 << gs_log2) >> 3;                 // lanes per group (4..32)
  const int grp = (lane * 8) >> gs_log2;                 // group within the stage
#pragma unroll
  for (int r = 0; r < R; r += RG) {
    if (m0 + 4 * r >= Mt) break;                         // uniform across the warp
    quantize_act_group<T, RG>(&xv[r], Mt, m0 + 4 * r, lanes, grp, qmax, xs, qa_slot, lane);
  }
}

template <int T, bool PARTIALS, bool FUSEDQ = false, int LAYOUT = 0>
__global__ void __launch_bounds__(GemmCfg<T>::kThreads, GemmCfg<T>::kMinBlocks)
    gemm_w6ax_kernel(const __grid_constant__ CUtensorMap tmap_x,
                     const __grid_constant__ CUtensorMap tmap_sa,
                     const __grid_constant__ LayerTable tab, const GemmArgs args) {
  using Cfg = GemmCfg<T>;
  constexpr int STAGES = Cfg::kStages;
  constexpr int ASLOTS = Cfg::kASlots;
  constexpr int NB = Cfg::kPBufs;
  // With fused quantization the unpack warps run the quantizer's code too:
  // the unpack loop over a stage's two weight tiles and the epilogue loop
  // over an octet's groups stay rolled, so that the code every warp of a
  // scheduler runs stays in its instruction cache (measured on the LLaMA-2
  // layers: unrolled, the instruction-fetch stalls made the in-kernel
  // quantization cost more than the separate quantizer's launch).
  constexpr int kTileUnroll = FUSEDQ ? 1 : 2;
  constexpr int kGroupUnroll = FUSEDQ ? 1 : 8;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  // activation slots: the TMA's ring, or with fused quantization one slot
  // per stage written by the unpack warps (its reuse is ordered by the A
  // slot's release, the same MMA commit)
  constexpr int XSL = FUSEDQ ? STAGES : Cfg::kXSlots;
  uint8_t* xs_ring = base;                                  // kXSlots * kXsBytes
  uint8_t* w_ring = base + Cfg::kXSlots * Cfg::kXsBytes;    // STAGES * 24576
  uint8_t* sc_ring = w_ring + STAGES * Cfg::kWStageBytes;   // kScSlots slots
  GemmCtrl<T>* ctrl = reinterpret_cast<GemmCtrl<T>*>(base + args.ctrl_offset);
  // fused quantization: per-stage activation-scale slots and their barriers
  static_assert(!FUSEDQ || (T == 16 && !PARTIALS && ASLOTS == STAGES), "fused quantization");
  uint64_t* qa_full = reinterpret_cast<uint64_t*>(base + args.fq_offset);   // 4 unpack warps
  uint64_t* qa_empty = qa_full + kQaSlots;                                   // epilogue warps
  __half* qa_ring = reinterpret_cast<__half*>(qa_empty + kQaSlots);          // [slot][8][T]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint64_t lim = args.wait_limit_ns;
  FLEXQ_CTA_TIME(0);
  // the next kernel of the stream may start its own prologue now; it waits
  // for this grid before it reads anything this grid writes
  if (threadIdx.x == 0) grid_launch_dependents();

  // work unit -> output tile and K range: the first n_full units are whole
  // tiles; after them every tile takes `split` consecutive units, one per K
  // range (the plan splits only what would otherwise run as a partial last
  // wave, or everything when there are fewer tiles than SMs)
  // the unit's layer, then its output tile and K range within the layer
  int layer = 0;
  while (layer + 1 < tab.n_layers && static_cast<int>(blockIdx.x) >= tab.unit0[layer + 1]) ++layer;
  const int unit = blockIdx.x - tab.unit0[layer];
  const int n_full = tab.n_full[layer];
  int tile, ks, S;
  if (unit < n_full) {
    tile = unit;
    ks = 0;
    S = 1;
  } else {
    const int split = tab.split[layer];
    const int u = unit - n_full;
    tile = n_full + u / split;
    ks = u - (u / split) * split;
    S = split;
  }
  const int N = tab.N[layer];
  const int tiles_n = N / kTileRows;
  const uint8_t* __restrict__ wp = tab.wp[layer];
  const CUtensorMap* tmap_sw = &tab.sw[layer];
  const int nt = tile % tiles_n;        // weight tile (fastest: neighbours share the tokens)
  const int mt = tile / tiles_n;        // token tile
  const int M = args.M, K = args.K, gs = args.gs;
  const int KB = K / kKBlock;                         // 128-wide weight tiles
  const int units = K / Cfg::kKStage;                 // stages along K (gs | 256)
  const int u0 = static_cast<int>((static_cast<long long>(ks) * units) / S);
  const int u1 = static_cast<int>((static_cast<long long>(ks + 1) * units) / S);
  const int kb0 = 2 * u0;                             // first weight tile
  const int nst = u1 - u0;                            // stages of this CTA
  // gs is a power of two (32..256): group arithmetic uses masks and shifts
  const int gs_log2 = __ffs(gs) - 1;
  const int g0 = (u0 * Cfg::kKStage) >> gs_log2;
  const int ngroups = (nst * Cfg::kKStage) >> gs_log2;

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&ctrl->full[s], 1);
      mbar_init(&ctrl->empty[s], 4);         // 4 unpack warps (weights read)
    }
    for (int x = 0; x < Cfg::kXSlots; ++x) mbar_init(&ctrl->x_empty[x], 1);   // MMA commit
    for (int a = 0; a < ASLOTS; ++a) {
      mbar_init(&ctrl->a_full[a], 4);        // 4 unpack warps
      mbar_init(&ctrl->a_empty[a], 1);       // MMA commit
    }
    for (int b = 0; b < NB; ++b) {
      mbar_init(&ctrl->p_full[b], 1);
      mbar_init(&ctrl->p_empty[b], Cfg::kEpiWarps);
    }
    for (int s = 0; s < Cfg::kScSlots; ++s) {
      mbar_init(&ctrl->s_full[s], 1);
      mbar_init(&ctrl->s_empty[s], Cfg::kEpiWarps);
    }
    mbar_init(&ctrl->done, 1);
    if (FUSEDQ) {
      for (int s = 0; s < kQaSlots; ++s) {
        mbar_init(&qa_full[s], 4);
        mbar_init(&qa_empty[s], Cfg::kEpiWarps);
      }
    }
    fence_barrier_init();
    // The packed weights are read-only inputs: the first ring's worth is
    // requested at once, before the TMEM allocation and the CTA barrier, and
    // before waiting for the kernels this one depends on (whose outputs may
    // be this kernel's activations and their scales).  With fused
    // quantization a stage's copy is the weights alone.
    constexpr uint32_t kStageTx0 = FUSEDQ ? Cfg::kWStageBytes : Cfg::kStageBytes;
    const int n_pre = nst < STAGES ? nst : STAGES;
    for (int i = 0; i < n_pre; ++i) {
      if (args.stall && i == 0) continue;
      mbar_arrive_expect_tx(&ctrl->full[i], kStageTx0);
      bulk_load(w_ring + i * Cfg::kWStageBytes,
                wp + (static_cast<size_t>(nt) * KB + kb0 + 2 * i) * kWTileBytes,
                Cfg::kWStageBytes, &ctrl->full[i]);
    }
    if (!FUSEDQ) prefetch_tensormap(&tmap_x);
    if (!PARTIALS) {
      if (!FUSEDQ) prefetch_tensormap(&tmap_sa);
      prefetch_tensormap(tmap_sw);
    }
  }
  if (FUSEDQ) {
    // tokens past M keep a zero scale in every slot
    for (int i = threadIdx.x; i < kQaSlots * 8 * T / 8; i += blockDim.x)
      reinterpret_cast<uint4*>(qa_ring)[i] = make_uint4(0u, 0u, 0u, 0u);
  }
  if (warp == 1) tmem_alloc(&ctrl->tmem_base, Cfg::kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctrl->tmem_base;
  FLEXQ_CTA_TIME(1);

  // epilogue state lives across the role switch below
  // FP32 accumulators as pairs (packed f32x2 arithmetic: sm_100 FFMA2/FMUL2)
  float2 acc[Cfg::kCols / 2];
#pragma unroll
  for (int j = 0; j < Cfg::kCols / 2; ++j) acc[j] = make_float2(0.0f, 0.0f);

  if (warp == 0) {
    // ------------------------------------------------------- producer ----
    if (lane == 0) {
      FLEXQ_ROLE_CLOCK;
      uint32_t issued = 0, parity = 0, sc_issued = 0, sc_parity = 0;
      const int n_oct = PARTIALS ? 0 : (ngroups + 7) / 8;
      int next_oct = 0;
      bool ok = true;
      // the first ring's weights were requested during set-up; with fused
      // quantization the stage's copy is the weights alone, and the scale
      // slots receive the weight scales only
      const int n_pre = nst < STAGES ? nst : STAGES;
      constexpr uint32_t kStageTx = FUSEDQ ? Cfg::kWStageBytes : Cfg::kStageBytes;
      constexpr uint32_t kScTx = FUSEDQ ? Cfg::kScSlotBytes - Cfg::kScSaBytes : Cfg::kScSlotBytes;
      grid_wait_dependencies();
      for (int i = 0; i < nst && ok; ++i) {
        // scales: issue octet o at the first stage that touches group 8*o
        const int lg_first = (i * Cfg::kKStage) >> gs_log2;
        while (next_oct < n_oct && next_oct * 8 <= lg_first) {
          const int o = next_oct, slot = o % Cfg::kScSlots;
          if (o >= Cfg::kScSlots &&
              !FLEXQ_WAIT(mbar_wait(&ctrl->s_empty[slot], ((o / Cfg::kScSlots) - 1) & 1, lim))) {
            ok = false;
            break;
          }
          uint8_t* dst = sc_ring + slot * Cfg::kScSlotBytes;
          mbar_arrive_expect_tx(&ctrl->s_full[slot], kScTx);
          if (!FUSEDQ) tma_load_2d(dst, &tmap_sa, &ctrl->s_full[slot], mt * T, g0 + 8 * o);
          tma_load_2d(dst + Cfg::kScSaBytes, tmap_sw, &ctrl->s_full[slot], nt * kTileRows,
                      g0 + 8 * o);
          sc_issued |= 1u << slot;
          sc_parity = (sc_parity & ~(1u << slot)) |
                      (static_cast<uint32_t>((o / Cfg::kScSlots) & 1) << slot);
          ++next_oct;
        }
        if (!ok) break;
        const int s = i % STAGES;
        if (i >= STAGES &&
            !FLEXQ_WAIT(mbar_wait(&ctrl->empty[s], ((i / STAGES) - 1) & 1, lim))) {
          ok = false;
          break;
        }
        if (args.stall && i == 0) continue;
        const int kb = kb0 + 2 * i;
        const int xsl = i % XSL;
        uint8_t* xs = xs_ring + xsl * Cfg::kXsBytes;
        if (i >= n_pre) {
          mbar_arrive_expect_tx(&ctrl->full[s], kStageTx);
          // tiles (nt, kb) and (nt, kb + 1) are adjacent in the device form
          bulk_load(w_ring + s * Cfg::kWStageBytes,
                    wp + (static_cast<size_t>(nt) * KB + kb) * kWTileBytes,
                    Cfg::kWStageBytes, &ctrl->full[s]);
        }
        // recorded before any further wait, so that a timeout below still
        // waits (bounded) for the copy in flight
        issued |= 1u << s;
        parity = (parity & ~(1u << s)) | (static_cast<uint32_t>((i / STAGES) & 1) << s);
        if (!FUSEDQ) {
          // the activation slot's previous box is free once the MMA that
          // read it has completed
          if (i >= XSL &&
              !FLEXQ_WAIT(mbar_wait(&ctrl->x_empty[xsl], ((i / XSL) - 1) & 1, lim))) {
            ok = false;
            break;
          }
          tma_load_2d(xs, &tmap_x, &ctrl->full[s], kb * kKBlock, mt * T);
          tma_load_2d(xs + Cfg::kXsHalf, &tmap_x, &ctrl->full[s], (kb + 1) * kKBlock, mt * T);
        }
      }
      if (!ok) record_status(args.status, kStatusTimeout, 0);
      FLEXQ_ROLE_DONE(0, nst);
      // every issued copy must land before the CTA may finish
      for (int s = 0; s < STAGES; ++s)
        if ((issued >> s) & 1u) mbar_wait(&ctrl->full[s], (parity >> s) & 1u, lim);
      for (int s = 0; s < Cfg::kScSlots; ++s)
        if ((sc_issued >> s) & 1u) mbar_wait(&ctrl->s_full[s], (sc_parity >> s) & 1u, lim);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ----------------------------------------------------------- MMA -----
    // On the issuing thread a tcgen05.mma is cheap only inside a straight
    // run of MMAs: any branch, predicated tcgen05 op or commit between two
    // MMAs waits for the previous one to be taken by the tensor pipe.  So the
    // MMAs of a group are one straight run (the group size is a compile-time
    // constant here), and the waits sit before a group's first MMA:
    //   a_full[a]  the unpack warps stored the stage's weights in A slot a;
    //              they do so after observing full[s], so the activations
    //              the TMA brought into shared memory are in place too;
    //   p_empty    with at least twice as many partial buffers as groups
    //              per stage, one wait at the stage start for the buffer of
    //              the stage's last group (the epilogue releases buffers in
    //              order, so the earlier ones are free too, and it still has
    //              a whole stage of groups to work on meanwhile); otherwise
    //              each group waits for its own buffer.
    if (lane == 0) {
      FLEXQ_ROLE_CLOCK;
      const uint64_t desc0 = smem_desc_k_sw128(smem_u32(xs_ring));
      auto run = [&](auto gs_c) -> bool {
        constexpr int GS = decltype(gs_c)::value;
        constexpr int G = Cfg::kKStage / GS;            // groups per stage
        constexpr int SPG = GS / 32;                     // MMAs per group
        constexpr bool kBatch = NB >= 2 * G;
        constexpr uint32_t idesc = idesc_i8(kTileRows, T);
        RingPos<XSL> xp;
        RingPos<ASLOTS> as;
        RingPos<NB> pb;                                  // buffer of the next group
        for (int i = 0; i < nst; ++i) {
          if (!FLEXQ_WAIT(mbar_wait(&ctrl->a_full[as.idx], as.phase, lim))) return false;
          if constexpr (kBatch) {
            RingPos<NB> last = pb;
#pragma unroll
            for (int j = 1; j < G; ++j) last.next();
            // use u of a buffer waits for the release of use u - 1: parity
            // (u & 1) ^ 1, which a fresh barrier reports complete for u = 0
            if (!FLEXQ_WAIT(mbar_wait(&ctrl->p_empty[last.idx], last.phase ^ 1u, lim)))
              return false;
          }
          tc_fence_after();
          const uint32_t a_col = tmem + Cfg::kACol0 + as.idx * Cfg::kACols;
          const uint64_t b_desc = desc0 + ((xp.idx * Cfg::kXsBytes) >> 4);
#pragma unroll
          for (int j = 0; j < G; ++j) {
            if constexpr (!kBatch) {
              if (!FLEXQ_WAIT(mbar_wait(&ctrl->p_empty[pb.idx], pb.phase ^ 1u, lim)))
                return false;
              tc_fence_after();
            }
            const uint32_t d_col = tmem + Cfg::kPCol0 + pb.idx * T;
#pragma unroll
            for (int k = 0; k < SPG; ++k) {
              const int sub = j * SPG + k;
              // A: weights of this stage in TMEM (8 columns per 32 codes);
              // B: activation box (sub / 4), 32-byte K step (sub % 4)
              mma_i8_tmem_a(d_col, a_col + sub * 8,
                            b_desc + (((sub >> 2) * Cfg::kXsHalf + (sub & 3) * 32) >> 4), idesc,
                            k == 0 ? 0u : 1u);
            }
            mma_commit(&ctrl->p_full[pb.idx]);
            pb.next();
          }
          if (!FUSEDQ) mma_commit(&ctrl->x_empty[xp.idx]);   // frees the activation slot
          mma_commit(&ctrl->a_empty[as.idx]);   // frees the A slot
          xp.next();
          as.next();
        }
        return true;
      };
      bool ok;
      switch (gs) {
        case 32: ok = run(std::integral_constant<int, 32>{}); break;
        case 64: ok = run(std::integral_constant<int, 64>{}); break;
        case 128: ok = run(std::integral_constant<int, 128>{}); break;
        default: ok = run(std::integral_constant<int, 256>{}); break;
      }
      if (!ok) record_status(args.status, kStatusTimeout, 1);
      FLEXQ_ROLE_DONE(1, nst);
      // all issued MMAs must finish before TMEM is released
      mma_commit(&ctrl->done);
      mbar_wait(&ctrl->done, 0, lim);
    }
    __syncwarp();
  } else if (warp < 6) {
    // -------------------------------------------------------- unpack -----
    const int q = warp & 3;                       // TMEM lane quarter
    const int row = q * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    FLEXQ_ROLE_CLOCK;
    RingPos<STAGES> st;
    RingPos<ASLOTS> as;
    // fused quantization: this warp's activation rows, loaded during the
    // previous stage
    constexpr int R = FUSEDQ ? T / 4 : 1;
    uint4 xv[R];
    RingPos<kQaSlots> qp;
    const __half* xt = args.x + static_cast<size_t>(mt) * T * K;   // the token tile's rows
    const int Mt = min(T, M - mt * T);
    if constexpr (FUSEDQ) {
      grid_wait_dependencies();                   // the activations may come from the previous kernel
      load_act_rows<R>(xv, xt, Mt, K, fq_row0(q, 0, Mt), kb0 * kKBlock, lane);
    }
    for (int i = 0; i < nst; ++i) {
      if constexpr (FUSEDQ) {
        // the stage's activation tile is free once its A slot is: the same
        // MMA commit releases both (as many A slots as stages)
        if (!FLEXQ_WAIT(warp_wait(&ctrl->a_empty[as.idx], as.phase ^ 1u, lim)) ||
            !FLEXQ_WAIT(warp_wait(&qa_empty[qp.idx], qp.phase ^ 1u, lim))) {
          if (lane == 0) record_status(args.status, kStatusTimeout, 2);
          break;
        }
        uint4 cur[R];
#pragma unroll
        for (int r = 0; r < R; ++r) cur[r] = xv[r];
        quantize_act_rows<T, R, kQaRowsTogether>(cur, Mt, fq_row0(q, i, Mt), gs_log2, args.qmax,
                                                 xs_ring + st.idx * Cfg::kXsBytes,
                                                 qa_ring + qp.idx * FusedQLayout<T>::kSlotHalves,
                                                 lane);
        fence_proxy_async_smem();                 // codes -> the MMA's operand reads
        __syncwarp();
        if (lane == 0) mbar_arrive(&qa_full[qp.idx]);
        qp.next();
        if (!FLEXQ_WAIT(warp_wait(&ctrl->full[st.idx], st.phase, lim))) {
          if (lane == 0) record_status(args.status, kStatusTimeout, 2);
          break;
        }
      } else {
        if (!FLEXQ_WAIT(warp_wait(&ctrl->full[st.idx], st.phase, lim)) ||
            !FLEXQ_WAIT(warp_wait(&ctrl->a_empty[as.idx], as.phase ^ 1u, lim))) {
          if (lane == 0) record_status(args.status, kStatusTimeout, 2);
          break;
        }
      }
      tc_fence_after();                           // the MMAs that read slot a are done
      // this row's packed bytes: tile t, chunk j at t*12288 + (j*128 + row)*16
      const uint4* src = reinterpret_cast<const uint4*>(w_ring + st.idx * Cfg::kWStageBytes) + row;
      const uint32_t col = tmem + lane_base + Cfg::kACol0 + as.idx * Cfg::kACols;
#pragma unroll kTileUnroll
      for (int t = 0; t < 2; ++t) {
        uint32_t w[24];
#pragma unroll
        for (int j = 0; j < 6; ++j) {
          const uint4 v = src[t * (kWTileBytes / 16) + j * 128];
          w[4 * j] = v.x; w[4 * j + 1] = v.y; w[4 * j + 2] = v.z; w[4 * j + 3] = v.w;
        }
        if (t == 1) {
          __syncwarp();
          if (lane == 0) mbar_arrive(&ctrl->empty[st.idx]);
        }
        uint32_t out[32];
        unpack_row_tile<LAYOUT>(w, out);
        tmem_st32(col + 32 * t, out);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctrl->a_full[as.idx]);
      // fused quantization: the next stage's rows, requested once this
      // stage's weights are out of the registers
      if (FUSEDQ && i + 1 < nst)
        load_act_rows<R>(xv, xt, Mt, K, fq_row0(q, i + 1, Mt), (kb0 + 2 * i + 2) * kKBlock, lane);
      st.next();
      as.next();
    }
    if (q == 0 && lane == 0) FLEXQ_ROLE_DONE(2, nst);
  } else {
    // ------------------------------------------------------ epilogue -----
    const int e = warp - 6;
    const int q = warp & 3;
    const int c = e >> 2;
    const int row = q * 32 + lane;
    const int n = nt * kTileRows + row;
    const int col0 = c * Cfg::kCols;
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    const int m_base = mt * T + col0;
    FLEXQ_ROLE_CLOCK;
    // groups in octets (the scale ring's unit): the eight groups of an octet
    // are unrolled, so their scale offsets are compile-time constants and the
    // ring slot and its release happen once per octet
    RingPos<NB> pb;
    RingPos<Cfg::kScSlots> sp;                       // scale-ring slot of the octet
    RingPos<kQaSlots> qp;                            // fused quantization: stage scale slot
    const int G_st = Cfg::kKStage >> gs_log2;        // groups per stage
    bool failed = false;
    for (int lo = 0; lo < ngroups && !failed; lo += 8) {
      const uint8_t* sc = sc_ring + sp.idx * Cfg::kScSlotBytes;
      const __half* sw_h = reinterpret_cast<const __half*>(sc + Cfg::kScSaBytes);
      if (!PARTIALS) {
        if (!FLEXQ_WAIT(warp_wait(&ctrl->s_full[sp.idx], sp.phase, lim))) {
          if (lane == 0) record_status(args.status, kStatusTimeout, 5);
          break;
        }
        if (!FUSEDQ) {
          // this warp's tokens of the octet, FP16 -> FP32, into its own buffer
          const __half* sa_h = reinterpret_cast<const __half*>(sc);
#pragma unroll
          for (int idx = lane; idx < 8 * Cfg::kCols; idx += 32) {
            const int gg = idx / Cfg::kCols, j = idx - gg * Cfg::kCols;
            ctrl->sa[e][gg][j] = __half2float(sa_h[gg * T + col0 + j]);
          }
          __syncwarp();
        }
      }
#pragma unroll kGroupUnroll
      for (int gi = 0; gi < 8; ++gi) {
      const int lg = lo + gi;
      if (lg >= ngroups) break;
      const int g = g0 + lg;
      if (FUSEDQ && (lg & (G_st - 1)) == 0) {
        // first group of a stage: its activation scales, from the unpack warps
        if (!FLEXQ_WAIT(warp_wait(&qa_full[qp.idx], qp.phase, lim))) {
          if (lane == 0) record_status(args.status, kStatusTimeout, 6);
          failed = true;
          break;
        }
        const __half* qa = qa_ring + qp.idx * FusedQLayout<T>::kSlotHalves;
        for (int idx = lane; idx < G_st * Cfg::kCols; idx += 32) {
          const int j = idx / Cfg::kCols, t = idx - j * Cfg::kCols;
          ctrl->sa[e][gi + j][t] = __half2float(qa[j * T + col0 + t]);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&qa_empty[qp.idx]);
        qp.next();
      }
      float swn = 0.0f;
      if (!PARTIALS) swn = __half2float(sw_h[gi * kTileRows + row]) * 0.25f;
      const float* sa_w = ctrl->sa[e][gi];
      if (!FLEXQ_WAIT(warp_wait(&ctrl->p_full[pb.idx], pb.phase, lim))) {
        if (lane == 0) record_status(args.status, kStatusTimeout, 4);
        failed = true;
        break;
      }
      tc_fence_after();
      // two 16-column loads: the second is issued before the first chunk's
      // arithmetic, so its latency hides behind it; the buffer is released
      // once both have landed
      static_assert(Cfg::kCols == 32 || Cfg::kCols == 16, "chunking");
      constexpr int NC = Cfg::kCols / 16;
      const uint32_t pcol = tmem + lane_base + Cfg::kPCol0 + pb.idx * T + col0;
      uint32_t pv[NC][16];
      tmem_ld16(pcol, pv[0]);
      tmem_wait_ld();
      if (NC == 2) tmem_ld16(pcol + 16, pv[NC - 1]);
#pragma unroll
      for (int ch = 0; ch < NC; ++ch) {
        if (ch == NC - 1) {
          if (NC == 2) tmem_wait_ld();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&ctrl->p_empty[pb.idx]);
        }
        if (PARTIALS) {
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int m = m_base + ch * 16 + j;
            if (m < M)
              args.p[(static_cast<size_t>(g) * M + m) * N + n] = static_cast<int32_t>(pv[ch][j]) >> 2;
          }
        } else {
          const float2 swn2 = make_float2(swn, swn);
          const float4* sa4 = reinterpret_cast<const float4*>(sa_w + ch * 16);
#pragma unroll
          for (int j = 0; j < 16; j += 4) {
            const float4 s4 = sa4[j / 4];
            const float2 s_lo = __fmul2_rn(swn2, make_float2(s4.x, s4.y));
            const float2 s_hi = __fmul2_rn(swn2, make_float2(s4.z, s4.w));
            const float2 p_lo = make_float2(__int2float_rn(static_cast<int32_t>(pv[ch][j])),
                                            __int2float_rn(static_cast<int32_t>(pv[ch][j + 1])));
            const float2 p_hi = make_float2(__int2float_rn(static_cast<int32_t>(pv[ch][j + 2])),
                                            __int2float_rn(static_cast<int32_t>(pv[ch][j + 3])));
            acc[(ch * 16 + j) / 2] = __ffma2_rn(p_lo, s_lo, acc[(ch * 16 + j) / 2]);
            acc[(ch * 16 + j) / 2 + 1] = __ffma2_rn(p_hi, s_hi, acc[(ch * 16 + j) / 2 + 1]);
          }
        }
      }
      pb.next();
      }
      if (!PARTIALS && !failed) {
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctrl->s_empty[sp.idx]);
      }
      sp.next();
    }
    if (e == 0 && lane == 0) FLEXQ_ROLE_DONE(3, ngroups);
  }

  // ------------------------------------------------------------ teardown --
  tc_fence_before();
  __syncthreads();
  FLEXQ_CTA_TIME(2);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, Cfg::kTmemCols);
  }
  FLEXQ_CTA_TIME(5);
  if (PARTIALS) {
    FLEXQ_CTA_TIME(3);
    return;
  }

  const bool is_epi = warp >= 6;
  const int e = warp - 6;
  const int row = (warp & 3) * 32 + lane;
  const int col0 = (e >> 2) * Cfg::kCols;
  if (S > 1) {
    // split-K: every CTA writes its FP32 partial tile to the workspace; the
    // last CTA of the output tile to arrive adds the `split` partials in
    // split order (the same order whichever CTA arrives last, so the result
    // is deterministic), writes the FP16 output and resets the counter.
    const size_t st_idx = static_cast<size_t>(tab.tile0[layer] + tile - n_full);   // counter
    float* part = args.ws_part + tab.part0[layer] +
                  static_cast<size_t>(tile - n_full) * S * T * kTileRows;
    if (is_epi) {
#pragma unroll
      for (int j = 0; j < Cfg::kCols; ++j)
        part[(static_cast<size_t>(ks) * T + col0 + j) * kTileRows + row] =
            (j & 1) ? acc[j / 2].y : acc[j / 2].x;
    }
    __syncthreads();
    FLEXQ_CTA_TIME(6);
    if (threadIdx.x == 0) {
      // the barrier orders the CTA's partial stores before this thread's
      // acquire-release add, which releases them with the count; the last
      // CTA's add acquires the other CTAs' partials before the barrier below
      const unsigned old = atom_add_acq_rel_gpu(&args.ws_cnt[st_idx], 1u);
      const bool last = old == static_cast<unsigned>(S - 1);
      if (last) args.ws_cnt[st_idx] = 0u;    // for the next launch (ordered by the kernel boundary)
      ctrl->is_last = last ? 1u : 0u;
    }
    __syncthreads();
    if (!ctrl->is_last) {
      FLEXQ_CTA_TIME(3);
      return;
    }
    if (is_epi) {
      float2 sum[Cfg::kCols / 2];
#pragma unroll
      for (int j = 0; j < Cfg::kCols / 2; ++j) sum[j] = make_float2(0.0f, 0.0f);
      for (int r = 0; r < S; ++r) {
        const float* pr = part + (static_cast<size_t>(r) * T + col0) * kTileRows + row;
#pragma unroll
        for (int j = 0; j < Cfg::kCols; j += 2) {
          // this CTA's own partial from registers, the others from L2
          const float x0 = (r == ks) ? acc[j / 2].x : __ldcg(pr + j * kTileRows);
          const float x1 = (r == ks) ? acc[j / 2].y : __ldcg(pr + (j + 1) * kTileRows);
          sum[j / 2].x += x0;
          sum[j / 2].y += x1;
        }
      }
#pragma unroll
      for (int j = 0; j < Cfg::kCols / 2; ++j) acc[j] = sum[j];
    }
  }
  FLEXQ_CTA_TIME(7);
  if (is_epi) {
    const int n = nt * kTileRows + row;
#pragma unroll
    for (int j = 0; j < Cfg::kCols; ++j) {
      const int m = mt * T + col0 + j;
      if (m < M)
        tab.y[layer][static_cast<size_t>(m) * N + n] =
            __float2half_rn((j & 1) ? acc[j / 2].y : acc[j / 2].x);
    }
  }
  FLEXQ_CTA_TIME(3);
}

}  // namespace flexq
