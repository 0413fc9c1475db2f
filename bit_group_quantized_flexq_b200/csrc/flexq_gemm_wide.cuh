// flexq_gemm_wide.cuh -- the W6A6 / W6A8 group GEMM for batches of more than
// 64 tokens: 128 weight rows x 128 tokens per CTA, warp roles aligned to
// warpgroups so that each warpgroup gets the registers its role needs.
//
// What it computes is the same as gemm_w6ax_kernel (flexq_gemm.cuh): the exact
// integer partial of every K-group, P_g[m,n] = sum_{k in g} qa[m,k] * qw[n,k],
// recombined with the group scales, Y[m,n] = sum_g P_g[m,n] * sa[m,g] *
// sw[n,g] (FlexQ paper, arXiv abstract; drgamma blog, "Bridging Software and
// Hardware with BTC": integer products summed, then recombined with the
// scales, dequantization fused into the GEMM).  Weight codes are unpacked
// losslessly to int8 (code * 4) into tensor memory and multiplied with
// tcgen05.mma.kind::i8, one fresh int32 accumulator per group.
//
// At 128 x 128 outputs per group of 128 codes the per-group rescale is as
// much work for the CUDA cores as the MMA is for the tensor core, so the
// layout below is built around the epilogue:
//   * the group scales are converted once per CTA into FP32 tables (sa / 4:
//     the factor 4 of the int8 weight codes folded in), read with 128-bit
//     broadcast loads;
//   * eight epilogue warps of 64 tokens each, tensor-memory loads issued one
//     32-column chunk ahead of the arithmetic, each partial converted with
//     one int -> float conversion (an exact one: |P| < 2^24) and rescaled
//     with packed FP32 multiplies and FMAs.
// (Measured alternatives, all slower at group 128: partial buffers pre-filled
// with the bits of 1.5 * 2^23 so that a packed subtraction replaces the
// conversion -- the refill stores cost more than the conversions save; the
// 16x256b load layout with per-thread scale pairs; sixteen 32-token epilogue
// warps; a 7-deep ring of 128-code stages.)
//
// Warpgroup 0  warp 0  producer: per stage of 256 codes, two TMA boxes of the
//                      int8 activations (128 rows x 128 B, 128-byte swizzle)
//                      and one 24576-byte bulk copy of two packed weight
//                      tiles into a 3-deep shared-memory ring;
//              warp 1  TMEM allocator and MMA issuer;
//              warps 2-3  scale converters: per 8 groups ("octet"), the FP16
//                      activation and weight scales of the tile from global
//                      memory into FP32 tables (a 3-deep ring);
// Warpgroup 1  warps 4-7  unpack: one weight row per thread, 192 packed bytes
//                      per stage -> 256 int8 codes in a TMEM "A" slot;
// Warpgroups 2-3  warps 8-15  epilogue: lane quarter q = warp % 4, tokens
//                      64 h .. 64 h + 63 with h = (warp - 8) / 4.
// Every pipeline wait is bounded (mbar_wait / warp_wait): a wait that runs
// out records FLEXQ_ERR_DEVICE_TIMEOUT and the role gives up.
#pragma once

#include "flexq_gemm.cuh"

namespace flexq {

struct WideCfg {
  static constexpr int T = 128;                       // tokens per tile (MMA N)
  static constexpr int kBandN = 32;                   // weight tiles per raster band
  static constexpr int kThreads = 512;
  static constexpr int kStages = 3;
  static constexpr int kKStage = 2 * kKBlock;         // codes of K per stage
  static constexpr int kXsHalf = T * 128;             // one activation box
  static constexpr int kXsBytes = 2 * kXsHalf;
  static constexpr int kWStageBytes = 2 * kWTileBytes;
  static constexpr int kStageBytes = kXsBytes + kWStageBytes;
  static constexpr int kScSlots = 3;
  static constexpr int kScFloats = 8 * 128;           // one FP32 table: 8 groups x 128
  static constexpr int kScSlotBytes = 2 * kScFloats * 4;   // activation + weight table
  static constexpr int kMainBytes = kStages * kStageBytes + kScSlots * kScSlotBytes;
  static constexpr int kPBufs = 3;                    // int32 partial buffers of T columns
  static constexpr int kASlots = 2;                   // A slots of 64 columns
  static constexpr int kACols = 64;
  static constexpr int kPCol0 = 0;
  static constexpr int kACol0 = kPBufs * T;
  static constexpr int kTmemCols = 512;
  static constexpr int kEpiWarps = 8;
  static constexpr int kMaxSplit = 4;
  // register budgets per warpgroup after the role split (launch: 128 each)
  static constexpr uint32_t kRegsCtl = 40, kRegsUnpack = 96, kRegsEpi = 184;
  static_assert(kACol0 + kACols * kASlots <= kTmemCols, "TMEM budget");
  static_assert(128 * kRegsCtl + 128 * kRegsUnpack + 256 * kRegsEpi <= 65536,
                "register split exceeds the launch's registers");
};

struct WideCtrl {
  uint64_t full[WideCfg::kStages];
  uint64_t empty[WideCfg::kStages];
  uint64_t a_full[WideCfg::kASlots];
  uint64_t a_empty[WideCfg::kASlots];
  uint64_t p_full[WideCfg::kPBufs];
  uint64_t p_empty[WideCfg::kPBufs];
  uint64_t sc_full[WideCfg::kScSlots];
  uint64_t sc_empty[WideCfg::kScSlots];
  uint64_t done;
  uint32_t tmem_base;
  uint32_t is_last;        // split-K: this CTA reduces the output tile
};

// The partial's 32 columns of one chunk into the FP32 accumulators:
// acc[j] += P'[j] * sa4[j] * sw (P' = 4 P from the code * 4 weights, sa4 =
// sa / 4 from the table); |P'| <= 2^22, so the conversion is exact.
__device__ __forceinline__ void wide_rescale_chunk(const uint32_t (&pv)[32], const float* sa,
                                                   float sw, float2* acc) {
  const float2 sw2 = make_float2(sw, sw);
  const float4* sa4 = reinterpret_cast<const float4*>(sa);
#pragma unroll
  for (int j = 0; j < 32; j += 4) {
    const float4 s4 = sa4[j / 4];
    const float2 s_lo = __fmul2_rn(sw2, make_float2(s4.x, s4.y));
    const float2 s_hi = __fmul2_rn(sw2, make_float2(s4.z, s4.w));
    const float2 p_lo = make_float2(__int2float_rn(static_cast<int32_t>(pv[j])),
                                    __int2float_rn(static_cast<int32_t>(pv[j + 1])));
    const float2 p_hi = make_float2(__int2float_rn(static_cast<int32_t>(pv[j + 2])),
                                    __int2float_rn(static_cast<int32_t>(pv[j + 3])));
    acc[j / 2] = __ffma2_rn(p_lo, s_lo, acc[j / 2]);
    acc[j / 2 + 1] = __ffma2_rn(p_hi, s_hi, acc[j / 2 + 1]);
  }
}

// Debug export: the chunk's exact int32 partials P = P' / 4.
__device__ __forceinline__ void wide_store_partials(const uint32_t (&pv)[32], int32_t* p, int g,
                                                    int M, int N, int m0, int n) {
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    const int m = m0 + j;
    if (m < M)
      p[(static_cast<size_t>(g) * M + m) * N + n] =
          static_cast<int32_t>(pv[j]) >> 2;
  }
}

template <bool PARTIALS, int LAYOUT = 0>
__global__ void __launch_bounds__(WideCfg::kThreads, 1)
    gemm_w6ax_wide_kernel(const __grid_constant__ CUtensorMap tmap_x, const GemmArgs args) {
  using Cfg = WideCfg;
  constexpr int T = Cfg::T;
  constexpr int STAGES = Cfg::kStages;
  constexpr int NB = Cfg::kPBufs;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* xs_ring = base;                                  // STAGES * kXsBytes
  uint8_t* w_ring = base + STAGES * Cfg::kXsBytes;          // STAGES * 24576
  float* sc_tab = reinterpret_cast<float*>(w_ring + STAGES * Cfg::kWStageBytes);
  WideCtrl* ctrl = reinterpret_cast<WideCtrl*>(base + args.ctrl_offset);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint64_t lim = args.wait_limit_ns;
  if (threadIdx.x == 0) grid_launch_dependents();

  // work unit -> output tile and K range (as gemm_w6ax_kernel)
  const int unit = blockIdx.x;
  int tile, ks, S;
  if (unit < args.n_full) {
    tile = unit;
    ks = 0;
    S = 1;
  } else {
    const int u = unit - args.n_full;
    tile = args.n_full + u / args.split;
    ks = u - (u / args.split) * args.split;
    S = args.split;
  }
  const int M = args.M, N = args.N, K = args.K, gs = args.gs;
  // output tile -> (weight tile nt, token tile mt) in bands of kBandN weight
  // tiles: inside a band the weight tile varies fastest and every token tile
  // passes the band's weight rows, so the CTAs in flight share a few weight
  // strips, which stay in L2 while the band lasts, and the packed weights are
  // read from DRAM about once (the activations once per band) instead of once
  // per token tile.
  const int tiles_m = (M + T - 1) / T;
  constexpr int kBandN = Cfg::kBandN;
  const int band = tile / (kBandN * tiles_m);
  const int n_band0 = band * kBandN;
  const int band_n = min(kBandN, args.tiles_n - n_band0);
  const int in_band = tile - band * kBandN * tiles_m;
  const int nt = n_band0 + in_band % band_n;
  const int mt = in_band / band_n;
  const int KB = K / kKBlock;
  const int units = K / Cfg::kKStage;
  const int u0 = static_cast<int>((static_cast<long long>(ks) * units) / S);
  const int u1 = static_cast<int>((static_cast<long long>(ks + 1) * units) / S);
  const int kb0 = 2 * u0;
  const int nst = u1 - u0;
  const int gs_log2 = __ffs(gs) - 1;
  const int g0 = (u0 * Cfg::kKStage) >> gs_log2;
  const int ngroups = (nst * Cfg::kKStage) >> gs_log2;
  const int n_oct = (ngroups + 7) / 8;

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&ctrl->full[s], 1);
      mbar_init(&ctrl->empty[s], 4 + 1);     // 4 unpack warps + MMA commit
    }
    for (int a = 0; a < Cfg::kASlots; ++a) {
      mbar_init(&ctrl->a_full[a], 4);
      mbar_init(&ctrl->a_empty[a], 1);
    }
    for (int b = 0; b < NB; ++b) {
      mbar_init(&ctrl->p_full[b], 1);
      mbar_init(&ctrl->p_empty[b], Cfg::kEpiWarps);
    }
    for (int s = 0; s < Cfg::kScSlots; ++s) {
      mbar_init(&ctrl->sc_full[s], 2);       // 2 converter warps
      mbar_init(&ctrl->sc_empty[s], Cfg::kEpiWarps);
    }
    mbar_init(&ctrl->done, 1);
    fence_barrier_init();
    // weights are read-only inputs: the first ring's worth is requested at
    // once, before the TMEM allocation and before waiting for the kernel
    // that produced the activations
    const int n_pre = nst < STAGES ? nst : STAGES;
    for (int i = 0; i < n_pre; ++i) {
      if (args.stall && i == 0) continue;
      mbar_arrive_expect_tx(&ctrl->full[i], Cfg::kStageBytes);
      bulk_load(w_ring + i * Cfg::kWStageBytes,
                args.wp + (static_cast<size_t>(nt) * KB + kb0 + 2 * i) * kWTileBytes,
                Cfg::kWStageBytes, &ctrl->full[i]);
    }
    prefetch_tensormap(&tmap_x);
  }
  if (warp == 1) tmem_alloc(&ctrl->tmem_base, Cfg::kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctrl->tmem_base;

  // Teardown, in every warp, on named barriers 1-3 (512 threads each):
  //   1: all roles done (TMEM freed after it);
  //   2: split-K partial tiles written (thread 0 then counts the arrival);
  //   3: the arrival count published (the last CTA reduces).
  // The epilogue warps hold the accumulators and run their own copy of it.
  auto teardown_ctl = [&]() {
    tc_fence_before();
    named_bar_sync(1, Cfg::kThreads);
    if (warp == 1) {
      tc_fence_after();
      tmem_dealloc(tmem, Cfg::kTmemCols);
    }
    if (!PARTIALS && S > 1) {
      named_bar_sync(2, Cfg::kThreads);
      if (threadIdx.x == 0) {
        // the barrier orders the CTA's partial stores before this
        // acquire-release add, which releases them with the count; the last
        // CTA's add acquires the other CTAs' partial tiles before barrier 3
        const size_t st_idx = static_cast<size_t>(tile - args.n_full);
        const unsigned old = atom_add_acq_rel_gpu(&args.ws_cnt[st_idx], 1u);
        const bool last = old == static_cast<unsigned>(S - 1);
        if (last) args.ws_cnt[st_idx] = 0u;  // for the next launch (ordered by the kernel boundary)
        ctrl->is_last = last ? 1u : 0u;
      }
      named_bar_sync(3, Cfg::kThreads);
    }
  };

  if (warp < 4) {
    regs_decrease<Cfg::kRegsCtl>();
    if (warp == 0) {
      // ----------------------------------------------------- producer ----
      if (lane == 0) {
        uint32_t issued = 0, parity = 0;
        bool ok = true;
        // the first ring's weights were requested during set-up
        const int n_pre = nst < STAGES ? nst : STAGES;
        grid_wait_dependencies();
        for (int i = 0; i < nst; ++i) {
          const int s = i % STAGES;
          if (i >= STAGES && !mbar_wait(&ctrl->empty[s], ((i / STAGES) - 1) & 1, lim)) {
            ok = false;
            break;
          }
          if (args.stall && i == 0) continue;
          const int kb = kb0 + 2 * i;
          uint8_t* xs = xs_ring + s * Cfg::kXsBytes;
          if (i >= n_pre) {
            mbar_arrive_expect_tx(&ctrl->full[s], Cfg::kStageBytes);
            bulk_load(w_ring + s * Cfg::kWStageBytes,
                      args.wp + (static_cast<size_t>(nt) * KB + kb) * kWTileBytes,
                      Cfg::kWStageBytes, &ctrl->full[s]);
          }
          tma_load_2d(xs, &tmap_x, &ctrl->full[s], kb * kKBlock, mt * T);
          tma_load_2d(xs + Cfg::kXsHalf, &tmap_x, &ctrl->full[s], (kb + 1) * kKBlock, mt * T);
          issued |= 1u << s;
          parity = (parity & ~(1u << s)) | (static_cast<uint32_t>((i / STAGES) & 1) << s);
        }
        if (!ok) record_status(args.status, kStatusTimeout, 0);
        // every issued copy must land before the CTA may finish
        for (int s = 0; s < STAGES; ++s)
          if ((issued >> s) & 1u) mbar_wait(&ctrl->full[s], (parity >> s) & 1u, lim);
      }
      __syncwarp();
    } else if (warp == 1) {
      // ---------------------------------------------------------- MMA ----
      // The MMAs of a group form one straight run (the group size is a
      // compile-time constant); the waits sit before a group's first MMA,
      // whose first K slice starts a fresh accumulator.
      if (lane == 0) {
        const uint64_t desc0 = smem_desc_k_sw128(smem_u32(xs_ring));
        auto run = [&](auto gs_c) -> bool {
          constexpr int GS = decltype(gs_c)::value;
          constexpr int G = Cfg::kKStage / GS;
          constexpr int SPG = GS / 32;
          constexpr uint32_t idesc = idesc_i8(kTileRows, T);
          RingPos<STAGES> st;
          RingPos<Cfg::kASlots> as;
          RingPos<NB> pb;
          for (int i = 0; i < nst; ++i) {
            if (!mbar_wait(&ctrl->a_full[as.idx], as.phase, lim)) return false;
            const uint32_t a_col = tmem + Cfg::kACol0 + as.idx * Cfg::kACols;
            const uint64_t b_desc = desc0 + ((st.idx * Cfg::kXsBytes) >> 4);
#pragma unroll
            for (int j = 0; j < G; ++j) {
              // use u of a buffer follows phase u of its release barrier
              // (phase 0: the epilogue's start)
              if (!mbar_wait(&ctrl->p_empty[pb.idx], pb.phase, lim)) return false;
              tc_fence_after();
              const uint32_t d_col = tmem + Cfg::kPCol0 + pb.idx * T;
#pragma unroll
              for (int k = 0; k < SPG; ++k) {
                const int sub = j * SPG + k;
                mma_i8_tmem_a(d_col, a_col + sub * 8,
                              b_desc + (((sub >> 2) * Cfg::kXsHalf + (sub & 3) * 32) >> 4), idesc,
                              k == 0 ? 0u : 1u);
              }
              mma_commit(&ctrl->p_full[pb.idx]);
              pb.next();
            }
            mma_commit(&ctrl->empty[st.idx]);
            mma_commit(&ctrl->a_empty[as.idx]);
            st.next();
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
        mma_commit(&ctrl->done);
        mbar_wait(&ctrl->done, 0, lim);
      }
      __syncwarp();
    } else {
      // ------------------------------------------- scale converters ------
      // 64 threads; thread c covers tokens (and weight rows) 2c, 2c + 1 of
      // the tile.  Activation scales may come from the previous kernel.
      if (!PARTIALS) {
        const int c = threadIdx.x - 64;
        const int m = mt * T + 2 * c;
        const int n = nt * kTileRows + 2 * c;
        const int ld = args.sa_ld;
        grid_wait_dependencies();
        RingPos<Cfg::kScSlots> sp;
        for (int o = 0; o < n_oct; ++o) {
          if (o >= Cfg::kScSlots &&
              !warp_wait(&ctrl->sc_empty[sp.idx], sp.phase ^ 1u, lim)) {
            if (lane == 0) record_status(args.status, kStatusTimeout, 5);
            break;
          }
          __half2 a2[8], w2[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const int lg = 8 * o + j;
            const int g = g0 + lg;
            a2[j] = __floats2half2_rn(0.0f, 0.0f);
            w2[j] = a2[j];
            if (lg < ngroups) {
              // a pair of tokens inside the scale rows' padded length (a
              // multiple of 8 >= M) is in bounds; tokens past M are never stored
              if (m < ld)
                a2[j] = __ldg(reinterpret_cast<const __half2*>(args.sa + static_cast<size_t>(g) * ld + m));
              w2[j] = __ldg(reinterpret_cast<const __half2*>(args.sw + static_cast<size_t>(g) * N + n));
            }
          }
          float* tab = sc_tab + sp.idx * (2 * Cfg::kScFloats);
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const float2 a = __half22float2(a2[j]);
            reinterpret_cast<float2*>(tab + j * 128)[c] = make_float2(a.x * 0.25f, a.y * 0.25f);
            reinterpret_cast<float2*>(tab + Cfg::kScFloats + j * 128)[c] = __half22float2(w2[j]);
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(&ctrl->sc_full[sp.idx]);
          sp.next();
        }
      }
    }
    teardown_ctl();
  } else if (warp < 8) {
    // ------------------------------------------------------- unpack ------
    regs_decrease<Cfg::kRegsUnpack>();
    const int q = warp & 3;
    const int row = q * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    RingPos<STAGES> st;
    RingPos<Cfg::kASlots> as;
    for (int i = 0; i < nst; ++i) {
      if (!warp_wait(&ctrl->full[st.idx], st.phase, lim) ||
          !warp_wait(&ctrl->a_empty[as.idx], as.phase ^ 1u, lim)) {
        if (lane == 0) record_status(args.status, kStatusTimeout, 2);
        break;
      }
      tc_fence_after();
      const uint4* src = reinterpret_cast<const uint4*>(w_ring + st.idx * Cfg::kWStageBytes) + row;
      const uint32_t col = tmem + lane_base + Cfg::kACol0 + as.idx * Cfg::kACols;
#pragma unroll
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
      st.next();
      as.next();
    }
    teardown_ctl();
  } else {
    // ----------------------------------------------------- epilogue ------
    regs_increase<Cfg::kRegsEpi>();
    // FP32 accumulators: tokens 64 h + 2 i and 64 h + 2 i + 1 of the tile
    float2 acc[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) acc[j] = make_float2(0.0f, 0.0f);
    const int q = warp & 3;
    const int h = (warp - 8) >> 2;
    const int row = q * 32 + lane;
    const int n = nt * kTileRows + row;
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    const int col_h = 64 * h;                        // this warp's tokens in the tile
    auto pcol = [&](int b, int c) -> uint32_t {
      return tmem + lane_base + Cfg::kPCol0 + b * T + col_h + 32 * c;
    };
    // phase 0 of every release barrier: every buffer is free at the start
    __syncwarp();
    if (lane == 0)
      for (int b = 0; b < NB; ++b) mbar_arrive(&ctrl->p_empty[b]);

    RingPos<NB> pb;
    RingPos<Cfg::kScSlots> sp;
    bool failed = false;
    uint32_t pa[32], pc[32];                         // chunk 0 / chunk 1 of a group
    if (ngroups > 0) {
      if (!warp_wait(&ctrl->p_full[0], 0, lim)) {
        failed = true;
      } else {
        tc_fence_after();
        tmem_ld32(pcol(0, 0), pa);
      }
    }
    for (int lg = 0; lg < ngroups && !failed; ++lg) {
      const int gi = lg & 7;
      const int g = g0 + lg;
      if (!PARTIALS && gi == 0 && !warp_wait(&ctrl->sc_full[sp.idx], sp.phase, lim)) {
        if (lane == 0) record_status(args.status, kStatusTimeout, 5);
        break;
      }
      const float* tab = sc_tab + sp.idx * (2 * Cfg::kScFloats);
      const float* sa_g = tab + gi * 128 + col_h;
      const float sw = PARTIALS ? 0.0f : tab[Cfg::kScFloats + gi * 128 + row];
      const int b = pb.idx;
      // chunk 0 has landed (issued one chunk ago); request chunk 1, then
      // rescale chunk 0 while chunk 1 loads
      tmem_wait_ld();
      tmem_ld32(pcol(b, 1), pc);
      if (PARTIALS)
        wide_store_partials(pa, args.p, g, M, N, mt * T + col_h, n);
      else
        wide_rescale_chunk(pa, sa_g, sw, acc);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctrl->p_empty[b]);
      pb.next();
      // the next group's chunk 0: requested before this group's chunk 1 is
      // rescaled when its MMAs are already done, else after
      bool ahead = false;
      const bool more = lg + 1 < ngroups;
      if (more && __all_sync(0xffffffffu, mbar_test_wait(smem_u32(&ctrl->p_full[pb.idx]), pb.phase))) {
        tc_fence_after();
        tmem_ld32(pcol(pb.idx, 0), pa);
        ahead = true;
      }
      if (PARTIALS)
        wide_store_partials(pc, args.p, g, M, N, mt * T + col_h + 32, n);
      else
        wide_rescale_chunk(pc, sa_g + 32, sw, acc + 16);
      if (!PARTIALS && (gi == 7 || !more)) {
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctrl->sc_empty[sp.idx]);
        sp.next();
      }
      if (more && !ahead) {
        if (!warp_wait(&ctrl->p_full[pb.idx], pb.phase, lim)) {
          if (lane == 0) record_status(args.status, kStatusTimeout, 4);
          failed = true;
          break;
        }
        tc_fence_after();
        tmem_ld32(pcol(pb.idx, 0), pa);
      }
    }
    if (failed && lane == 0) record_status(args.status, kStatusTimeout, 4);
    tmem_wait_ld();

    // -------------------------------------------------- teardown ----
    tc_fence_before();
    named_bar_sync(1, Cfg::kThreads);
    if (PARTIALS) return;
    const int col0 = col_h;
    if (S > 1) {
      // split-K: every CTA writes its FP32 partial tile to the workspace; the
      // last CTA of the output tile to arrive adds the `split` partials in
      // split order (deterministic whatever the arrival order), writes the
      // FP16 output; thread 0 (teardown_ctl) counts the arrivals
      const size_t st_idx = static_cast<size_t>(tile - args.n_full);
      float* part = args.ws_part + st_idx * static_cast<size_t>(S) * T * kTileRows;
#pragma unroll
      for (int j = 0; j < 64; ++j)
        part[(static_cast<size_t>(ks) * T + col0 + j) * kTileRows + row] =
            (j & 1) ? acc[j / 2].y : acc[j / 2].x;
      named_bar_sync(2, Cfg::kThreads);
      named_bar_sync(3, Cfg::kThreads);
      if (!ctrl->is_last) return;
      float2 sum[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) sum[j] = make_float2(0.0f, 0.0f);
      for (int r = 0; r < S; ++r) {
        const float* pr = part + (static_cast<size_t>(r) * T + col0) * kTileRows + row;
#pragma unroll
        for (int j = 0; j < 64; j += 2) {
          const float x0 = (r == ks) ? acc[j / 2].x : __ldcg(pr + j * kTileRows);
          const float x1 = (r == ks) ? acc[j / 2].y : __ldcg(pr + (j + 1) * kTileRows);
          sum[j / 2].x += x0;
          sum[j / 2].y += x1;
        }
      }
#pragma unroll
      for (int j = 0; j < 32; ++j) acc[j] = sum[j];
    }
#pragma unroll
    for (int j = 0; j < 64; ++j) {
      const int m = mt * T + col0 + j;
      if (m < M)
        args.y[static_cast<size_t>(m) * N + n] =
            __float2half_rn((j & 1) ? acc[j / 2].y : acc[j / 2].x);
    }
  }
}

}  // namespace flexq
