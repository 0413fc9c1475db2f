/*
 * flexq.h -- C ABI of the B200 (sm_100a) library for FlexQ's group-quantized
 * W6A6 / W6A8 linear layer.
 *
 * The method (FlexQ: Efficient Post-training INT6 Quantization for LLM
 * Serving via Algorithm-System Co-Design): weights are quantized uniformly to
 * 6 bits, activations to 6 bits or, in sensitive layers, 8 bits (arXiv
 * abstract); both use fine-grained groups along K that share one scale
 * (drgamma blog, "Fine-Grained Quantization and Layer Sensitivity" and
 * "Bridging Software and Hardware with BTC"); the GEMM sums integer products
 * per group and recombines them with the scales, with dequantization fused
 * into the GEMM (blog, "Bridging Software and Hardware with BTC").
 *
 * Conventions shared by every entry point
 *   - All buffers are DEVICE memory owned by the caller; the library never
 *     allocates, frees or retains them.  FP16 buffers are IEEE binary16.
 *   - Matrices are row-major.  M = tokens, N = output channels, K = input
 *     channels, gs = group size along K, G = K / gs.
 *   - Supported shapes: M >= 0 (M == 0 is a no-op), N % 128 == 0, K % 256 == 0,
 *     gs in {32, 64, 128, 256} (K % gs == 0 follows).  Activation
 *     quantization alone only needs K % gs == 0.
 *   - Every device pointer must be 16-byte aligned.  With M == 0 the
 *     activation-side pointers are not read and may be NULL.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Calls
 *     are asynchronous: they validate their arguments, enqueue the work on
 *     `stream` and return.  Invalid arguments are reported before anything
 *     is enqueued.
 *   - Return value: a flexq_status_t.  flexq_last_error_message() gives a
 *     human-readable detail for the calling thread's last failure.
 *   - Device-side failures (a pipeline wait that exceeded its time limit) do
 *     not trap: the kernel records them in a device status word and returns;
 *     flexq_get_device_status() reads and clears that word.
 */
#ifndef FLEXQ_H_
#define FLEXQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FLEXQ_OK = 0,
  FLEXQ_ERR_INVALID_ARG = 1,     /* null pointer, negative size, bad bits     */
  FLEXQ_ERR_UNSUPPORTED = 2,     /* shape outside the supported set above     */
  FLEXQ_ERR_MISALIGNED = 3,      /* a device pointer is not 16-byte aligned   */
  FLEXQ_ERR_CUDA = 4,            /* a CUDA runtime call or launch failed      */
  FLEXQ_ERR_DEVICE_TIMEOUT = 5   /* a kernel's bounded wait gave up           */
} flexq_status_t;

/* Name of a status code (static string, never NULL). */
const char* flexq_status_string(int status);

/* Detail of the calling thread's most recent failure ("" if none). */
const char* flexq_last_error_message(void);

/*
 * Leading dimension (in elements) of the group-major activation scales for a
 * batch of M tokens: M rounded up to a multiple of 8, so that every group's
 * row starts on a 16-byte boundary.  0 for M <= 0.
 */
size_t flexq_act_scales_ld(int M);

/*
 * Size in bytes of the packed 6-bit weight buffer for an [N, K] layer:
 * 3*N*K/4 (four codes in three bytes).  Returns 0 for unsupported shapes.
 */
size_t flexq_weight_packed_bytes(int N, int K, int group_size);

/*
 * flexq_quantize_weight -- offline 6-bit weight quantization and packing.
 * Passage: uniform 6-bit weights (arXiv abstract); groups along K sharing a
 * scale (blog, "Fine-Grained Quantization and Layer Sensitivity";
 * "Bridging Software and Hardware with BTC").
 *
 *   W_fp16        [N, K] FP16, finite values.
 *   Wq_packed     out, flexq_weight_packed_bytes(N, K, gs) bytes: the device
 *                 form of the 6-bit codes, four codes per three bytes.  Each
 *                 row is cut into blocks of 16 consecutive codes c0..c15
 *                 (u_j = c_j & 63); a block is three little-endian 32-bit
 *                 words w0, w1, w2 in which byte t of word i holds u_{4i+t}
 *                 in its bits [7:2] and bits [2i+1:2i] of u_{12+t} in its
 *                 bits [1:0].  The row's 96 bytes of codes kb*128 ..
 *                 kb*128+127 (eight blocks) are cut into six 16-byte chunks;
 *                 tile (nt, kb) (rows nt*128 .. nt*128+127) is 12288
 *                 contiguous bytes at offset (nt*(K/128) + kb)*12288, and
 *                 chunk j of row r sits at offset (j*128 + r)*16 inside it.
 *   W_scales_fp16 out, N*G FP16 values stored group-major: the scale of row
 *                 n, group g is element g*N + n.  s = fp16_rne(absmax / 31)
 *                 with absmax/31 computed as an IEEE FP32 division.
 * Codes: clamp(round_half_even(w / s), -31, 31) with an IEEE FP32 division by
 * the stored FP16 scale; a group whose FP16 scale is 0 gets all-zero codes.
 */
int flexq_quantize_weight(int N, int K, int group_size, const void* W_fp16,
                          void* Wq_packed, void* W_scales_fp16, void* stream);

/*
 * Weight layouts of the packed buffer.  FLEXQ_LAYOUT_BYTE_ALIGNED is the
 * device form above (the default everywhere).  FLEXQ_LAYOUT_4_2 is the
 * "4+2" bit-plane form, after the split storage of 6-bit values into a 4-bit
 * and a 2-bit part (ZeroQuant(4+2) abstract): with h_j = u_j >> 2 and
 * l_j = u_j & 3, a 16-code block is an 8-byte 4-bit plane (byte t = h_t << 4
 * | h_{4+t}, byte 4+t = h_{8+t} << 4 | h_{12+t}) and a 4-byte 2-bit plane
 * (byte t = l_t | l_{4+t} << 2 | l_{8+t} << 4 | l_{12+t} << 6); tiles as
 * above, and inside a tile chunks 0..3 of each row hold its eight blocks'
 * 4-bit planes, chunks 4 and 5 their 2-bit planes, so that each plane is one
 * contiguous 16-byte aligned region (8192 and 4096 bytes) of the tile.  Same
 * size, same codes and scales; only the bit placement differs.
 */
#define FLEXQ_LAYOUT_BYTE_ALIGNED 0
#define FLEXQ_LAYOUT_4_2 1

/* flexq_quantize_weight with an explicit layout (FLEXQ_ERR_INVALID_ARG for
 * any other value). */
int flexq_quantize_weight_layout(int N, int K, int group_size, int layout, const void* W_fp16,
                                 void* Wq_packed, void* W_scales_fp16, void* stream);

/*
 * flexq_quantize_act -- per-forward activation quantization, 6 or 8 bits.
 * Passage: 6-bit activations, 8-bit ones kept in sensitive layers (arXiv
 * abstract; blog, "Fine-Grained Quantization and Layer Sensitivity").
 *
 *   X_fp16        [M, K] FP16, finite values.
 *   bits          6 (codes in [-31, 31], Q = 31) or 8 (codes in [-127, 127],
 *                 Q = 127).
 *   Xq            out, [M, K] int8, one code per byte for both widths.
 *   X_scales_fp16 out, G * flexq_act_scales_ld(M) FP16 values stored
 *                 group-major: the scale of token m, group g is element
 *                 g*ld + m with ld = flexq_act_scales_ld(M) (M rounded up to
 *                 a multiple of 8); entries m >= M are not written.
 *                 s = fp16_rne(absmax / Q).
 * Same rounding rules as flexq_quantize_weight.
 */
int flexq_quantize_act(int M, int K, int group_size, int bits,
                       const void* X_fp16, int8_t* Xq, void* X_scales_fp16,
                       void* stream);

/*
 * flexq_gemm_workspace_bytes -- device workspace the GEMM entry points need
 * for a shape: 0 when the launch plan does not split K, otherwise 4096 bytes
 * of arrival counters (one per output tile, always at the start, so calls of
 * different shapes can share one workspace) followed by the FP32 partial
 * tiles of the K split.  Pure host computation; 0 for unsupported shapes and
 * M <= 0.  Plans with more than 1024 output tiles never split K.
 */
size_t flexq_gemm_workspace_bytes(int M, int N, int K, int group_size);

/*
 * flexq_gemm_w6a6 / flexq_gemm_w6a8 -- Y = dequant(Xq) . dequant(Wq)^T.
 * Passage: the W6A6 / W6A8 GEMM whose integer products are summed per group
 * and recombined with the scales, dequantization fused into the GEMM (arXiv
 * abstract; blog, "Bridging Software and Hardware with BTC").
 *
 *   Xq, X_scales     activation codes [M, K] int8 and FP16 scales in the
 *                    group-major layout of flexq_quantize_act.
 *   Wq_packed,       weight codes in the device form above and FP16 scales
 *   W_scales         (group-major, g*N + n), as written by
 *                    flexq_quantize_weight.
 *   Y_fp16           out, [M, N] FP16.
 *   workspace,       device scratch of flexq_gemm_workspace_bytes(M, N, K, gs)
 *   workspace_bytes  bytes or more, owned by the caller, 16-byte aligned.  It
 *                    must be zero-filled before its first use; every call
 *                    that completes leaves it zero-filled again (re-zero it
 *                    after a call that reported FLEXQ_ERR_DEVICE_TIMEOUT).
 *                    Calls that share a workspace must not overlap on the
 *                    GPU.  NULL with 0 bytes runs the GEMM without a K split
 *                    (correct, slower at small M); a smaller non-zero size is
 *                    FLEXQ_ERR_INVALID_ARG.
 * For each group g the integer partial P_g[m,n] = sum_{k in g} Xq[m,k]*Wq[n,k]
 * is formed exactly (int32), then Y[m,n] = fp16_rne(sum_g P_g[m,n] *
 * sa[m,g] * sw[n,g]) with the sum over groups accumulated in FP32 (per
 * output, |Y - Y_exact| <= 5e-4 * max|Y| on the benchmark distributions).
 * A K split adds the FP32 partial sums of its ranges in a fixed order, so the
 * output does not depend on the order in which the CTAs finish.
 * The two entry points run the same kernel: they differ only in the code
 * range the caller's activations are expected to use ([-31, 31] vs
 * [-127, 127]); neither checks the range, and any int8 activation code and
 * any 6-bit weight code (including -32) are multiplied exactly.
 */
int flexq_gemm_w6a6(int M, int N, int K, int group_size, const int8_t* Xq,
                    const void* X_scales, const void* Wq_packed,
                    const void* W_scales, void* Y_fp16, void* workspace,
                    size_t workspace_bytes, void* stream);
int flexq_gemm_w6a8(int M, int N, int K, int group_size, const int8_t* Xq,
                    const void* X_scales, const void* Wq_packed,
                    const void* W_scales, void* Y_fp16, void* workspace,
                    size_t workspace_bytes, void* stream);

/*
 * flexq_linear_workspace_bytes -- device workspace the linear entry points
 * need for a shape.  Shapes that quantize inside the GEMM (see
 * flexq_linear_launches) need exactly flexq_gemm_workspace_bytes; the others
 * also hold the quantized activations: 4096 bytes of arrival counters (or the
 * GEMM workspace if larger), then the [M, K] int8 codes and the FP16 scales
 * (G * flexq_act_scales_ld(M) values), each starting on a 256-byte boundary.
 * Pure host computation; 0 for unsupported shapes and M <= 0.
 */
size_t flexq_linear_workspace_bytes(int M, int N, int K, int group_size);

/*
 * flexq_linear_launches -- kernel launches of one linear call for a shape:
 * 1 where the activations are quantized inside the GEMM, 2 otherwise
 * (quantizer, GEMM).  The GEMM quantizes on 16-token tiles where
 * (M + 2) * stages <= 28, stages being the stages of 256 codes of K that each
 * CTA streams (where that is faster than a separate quantizer).
 * 0 for unsupported shapes and M <= 0.  Pure host computation.
 */
int flexq_linear_launches(int M, int N, int K, int group_size);

/*
 * flexq_linear_w6a6 / flexq_linear_w6a8 -- a quantized linear layer from
 * FP16 activations: Y = dequant(quant_a(X)) . dequant(Wq)^T with quant_a the
 * 6-bit (w6a6) or 8-bit (w6a8) activation quantizer of flexq_quantize_act.
 * Passage: activations quantized per group at run time and multiplied with
 * the 6-bit weights, dequantization fused into the GEMM (arXiv abstract;
 * blog, "Fine-Grained Quantization and Layer Sensitivity" and "Bridging
 * Software and Hardware with BTC").
 *
 *   X_fp16           [M, K] FP16 activations, finite values, 16-byte aligned.
 *   Wq_packed,       as for flexq_gemm_w6a6.
 *   W_scales
 *   Y_fp16           out, [M, N] FP16.
 *   workspace,       device scratch of flexq_linear_workspace_bytes(M, N, K,
 *   workspace_bytes  gs) bytes or more, owned by the caller, 16-byte
 *                    aligned, zero-filled before its first use (completed
 *                    calls leave its counters zero again).  Where the
 *                    quantization runs inside the GEMM, NULL with 0 bytes
 *                    runs without a K split, as for the GEMM; elsewhere the
 *                    workspace is required (FLEXQ_ERR_INVALID_ARG).
 * Small batches on short K ranges (flexq_linear_launches) quantize the
 * activations inside the GEMM kernel (one launch, no quantized copy in device
 * memory); the others launch the activation quantizer into the workspace and
 * then the GEMM.  Both routes
 * compute the same codes and scales as flexq_quantize_act, and the result is
 * bit-identical to flexq_quantize_act followed by flexq_gemm_w6a6/w6a8 under
 * the same plan.
 */
int flexq_linear_w6a6(int M, int N, int K, int group_size, const void* X_fp16,
                      const void* Wq_packed, const void* W_scales, void* Y_fp16,
                      void* workspace, size_t workspace_bytes, void* stream);
int flexq_linear_w6a8(int M, int N, int K, int group_size, const void* X_fp16,
                      const void* Wq_packed, const void* W_scales, void* Y_fp16,
                      void* workspace, size_t workspace_bytes, void* stream);

/*
 * flexq_gemm_static_scratch -- the GEMM of flexq_gemm_w6a6 (act_bits 6) or
 * flexq_gemm_w6a8 (act_bits 8) for callers that cannot allocate device
 * memory when they call it: an engine plugin whose enqueue step may not
 * allocate, or a serving process that reserves all device memory for its own
 * pool at start-up.  The paper has no counterpart; this is an interface
 * convenience of this library.
 *   Same arguments, layouts and results as flexq_gemm_w6a6/w6a8 without the
 *   workspace: the split-K scratch is a 16 MiB array the library keeps in
 *   each device's global memory for the life of the process.  The call
 *   allocates nothing (no cudaMalloc, cudaFree or allocating library call).
 *   Shapes whose plan needs more split-K scratch than 16 MiB are rejected
 *   with FLEXQ_ERR_UNSUPPORTED (no plan the library picks by itself does).
 *   Shapes and pointers are checked first; an invalid argument returns its
 *   status with nothing enqueued.  The first call on a device looks up the
 *   scratch's device address; make that first call before capturing a
 *   stream.  Each call then clears the scratch's arrival counters on
 *   `stream` (a 4 KB memset) and launches.
 *   All calls on a device share the one scratch, which keeps the last call's
 *   partial tiles: two calls that overlap on the GPU (different streams, or
 *   concurrently running graphs) race on it and give wrong results.
 */
int flexq_gemm_static_scratch(int M, int N, int K, int group_size, int act_bits,
                              const int8_t* Xq, const void* X_scales,
                              const void* Wq_packed, const void* W_scales,
                              void* Y_fp16, void* stream);

/*
 * flexq_gemm_layout / flexq_linear_layout -- flexq_gemm_w6a6/w6a8 and
 * flexq_linear_w6a6/w6a8 (act_bits 6 or 8) on packed weights of either
 * layout (the weights must have been packed with the same layout).  Same
 * arguments, plans, workspaces and results otherwise; FLEXQ_ERR_INVALID_ARG
 * for an unknown layout or act_bits.
 */
int flexq_gemm_layout(int M, int N, int K, int group_size, int act_bits, int layout,
                      const int8_t* Xq, const void* X_scales, const void* Wq_packed,
                      const void* W_scales, void* Y_fp16, void* workspace, size_t workspace_bytes,
                      void* stream);
int flexq_linear_layout(int M, int N, int K, int group_size, int act_bits, int layout,
                        const void* X_fp16, const void* Wq_packed, const void* W_scales,
                        void* Y_fp16, void* workspace, size_t workspace_bytes, void* stream);

/*
 * One layer of a grouped call: layers that read the same activations (the
 * q, k and v projections of attention, or the gate and up projections of an
 * MLP), each with its own weights and output.
 *   N          output channels of this layer (N % 128 == 0);
 *   Wq_packed  its packed 6-bit weights (device form, flexq_quantize_weight);
 *   W_scales   its FP16 weight scales, group-major [K/gs, N];
 *   Y_fp16     its FP16 output [M, N] (written, not read).
 */
typedef struct flexq_layer {
  int N;
  const void* Wq_packed;
  const void* W_scales;
  void* Y_fp16;
} flexq_layer_t;

#define FLEXQ_MAX_GROUP_LAYERS 4

/*
 * flexq_gemm_group -- the GEMM of flexq_gemm_w6a6 / w6a8 for 1 to 4 layers
 * that share their quantized activations (Xq, X_scales as for those calls;
 * act_bits 6 or 8 only names the code range), in one kernel launch for
 * batches of at most 64 tokens and one launch per layer above.  The method
 * is per layer exactly that of flexq_gemm_w6a6/w6a8 (FlexQ arXiv abstract;
 * drgamma blog, "Bridging Software and Hardware with BTC"); grouping the
 * layers is this library's launch strategy: one set of CTAs streams every
 * layer's weights, so that one layer's set-up and split-K tail overlap the
 * others' streaming.  The plan is shared: the token tile follows M, and when
 * all layers together have fewer output tiles than CTA slots every tile is
 * split along K by one factor (split-K partials in the workspace, added in
 * split order: results are deterministic, and equal to a single-layer call
 * with the same split).
 *   workspace  zero-filled device buffer of flexq_gemm_group_workspace_bytes
 *              bytes (NULL and 0 run without a K split), left zero.
 * Errors: FLEXQ_ERR_INVALID_ARG for n_layers outside 1..4, a NULL `layers`,
 * bad act_bits or a short workspace; the shape and pointer rules of
 * flexq_gemm_w6a6 per layer.
 */
int flexq_gemm_group(int M, int K, int group_size, int act_bits, const int8_t* Xq,
                     const void* X_scales, int n_layers, const flexq_layer_t* layers,
                     void* workspace, size_t workspace_bytes, void* stream);

/* Workspace bytes of flexq_gemm_group (0 for invalid arguments). */
size_t flexq_gemm_group_workspace_bytes(int M, int K, int group_size, int n_layers,
                                        const int* N);

/*
 * flexq_linear_group -- flexq_linear_w6a6 / w6a8 (act_bits 6 or 8) for 1 to
 * 4 layers that read the same FP16 activations X [M, K]: the activations are
 * quantized once, inside the grouped GEMM launch where a single layer would
 * be (16-token tiles, few K stages per CTA, a few tokens), else by one
 * activation-quantizer launch into the workspace, followed by
 * flexq_gemm_group on those codes.  Every output equals flexq_linear_* on
 * that layer alone up to the FP32 summation order of the K split.
 *   workspace  zero-filled device buffer of flexq_linear_group_workspace_bytes
 *              bytes (may be NULL when that is 0).
 */
int flexq_linear_group(int M, int K, int group_size, int act_bits, const void* X_fp16,
                       int n_layers, const flexq_layer_t* layers, void* workspace,
                       size_t workspace_bytes, void* stream);

/* Workspace bytes of flexq_linear_group (0 for invalid arguments). */
size_t flexq_linear_group_workspace_bytes(int M, int K, int group_size, int n_layers,
                                          const int* N);

/*
 * flexq_group_plan -- host only: the grouped plan for these layers: tokens
 * per tile, K split and CTAs of the grouped launch (0 and 0 when the batch
 * takes 128-token tiles and the layers run one launch each), and the kernel
 * launches of flexq_linear_group.
 */
int flexq_group_plan(int M, int K, int group_size, int n_layers, const int* N, int* tile_tokens,
                     int* k_split, int* ctas, int* launches);

/*
 * flexq_debug_check_quantizer -- test hook: runs the GPU quantizer's
 * division-free code rule against the IEEE-division rule (FP32 division by
 * the stored FP16 scale, round half to even, clamp) on every pair of a
 * finite FP16 value and a positive finite FP16 scale, for Q = 31 and
 * Q = 127.  Writes the number of differing (x, s, Q) cases to *mismatches
 * and the first one found ({x bits, s bits, Q}) to first_mismatch[0..2].
 * Synchronous; allocates and frees its own small device buffer.
 */
int flexq_debug_check_quantizer(unsigned long long* mismatches,
                                unsigned int* first_mismatch);

/*
 * flexq_debug_force_linear_route -- test hook: 0 picks the linear route by
 * shape (flexq_linear_launches), 1 quantizes inside the GEMM whenever the
 * plan's token tile is 16 rows, 2 always runs the separate quantizer.
 * Process-wide; FLEXQ_ERR_INVALID_ARG for other values.
 */
int flexq_debug_force_linear_route(int route);

/*
 * flexq_debug_group_partials -- exports the per-group int32 partials of the
 * GEMM above, computed by the same kernel mainloop (test hook).
 *   P  out, int32 [G, M, N]: P[g][m][n] = sum_{k in g} Xq[m,k] * Wq[n,k].
 */
int flexq_debug_group_partials(int M, int N, int K, int group_size,
                               const int8_t* Xq, const void* Wq_packed,
                               int32_t* P, void* stream);

/*
 * flexq_debug_export_canonical -- the packed weights in the canonical 6-bit
 * form, for tests and for interchange with other tools.  Passage: uniform
 * 6-bit weights stored four codes to three bytes (arXiv abstract; blog,
 * "Bridging Software and Hardware with BTC").
 *   layout       FLEXQ_LAYOUT_BYTE_ALIGNED or FLEXQ_LAYOUT_4_2: the form of
 *                Wq_packed (as written by flexq_quantize_weight_layout).
 *   Wq_packed    in, device, flexq_weight_packed_bytes(N, K, 128) bytes.
 *   W_canonical  out, device, 3*N*K/4 bytes, row-major: for codes c0..c3 at
 *                k = 4j..4j+3 of row n (u_i = c_i & 63) the 24-bit word
 *                u0 | u1<<6 | u2<<12 | u3<<18, little endian, at bytes
 *                n*(3K/4) + 3j .. +2.  Owned by the caller.
 * Shapes as for the GEMM (N % 128 == 0, K % 256 == 0); both pointers 16-byte
 * aligned (FLEXQ_ERR_MISALIGNED), checked before anything is enqueued.
 * Asynchronous on `stream`.
 */
int flexq_debug_export_canonical(int N, int K, int layout, const void* Wq_packed,
                                 void* W_canonical, void* stream);

/*
 * flexq_gemm_plan -- the launch the GEMM entry points would use for a shape
 * given enough workspace: tokens per tile (16, 32, 64 or 128), K-split factor
 * (CTAs that share an output tile, each over its own range of K) and the
 * number of CTAs.  Tokens per tile follow M (16 up to 16 tokens, 32 up to 32,
 * 128 above 64; 33..64 tokens take two 32-token tiles while those fit one
 * wave of CTA slots, else one 64-token tile).  With fewer output tiles than
 * CTA slots every tile is split (128-token tiles keep at least 8 stages of
 * 256 codes per CTA); otherwise the whole waves of tiles run unsplit and only
 * the tiles of a partial last wave are split (k_split is then their split, 1
 * if none).  Any output pointer may be NULL.  Pure host computation.
 */
int flexq_gemm_plan(int M, int N, int K, int group_size, int* tile_tokens,
                    int* k_split, int* ctas);

/*
 * flexq_debug_force_plan -- test hook: make subsequent GEMM launches on the
 * calling process use tile_tokens (16/32/64/128) and k_split (1..8) when the
 * shape allows it.  (0, 0) restores the automatic choice.
 */
int flexq_debug_force_plan(int tile_tokens, int k_split);

/*
 * flexq_set_wait_limit_ns -- time limit of every bounded pipeline wait in the
 * GEMM kernel (default 2e9 ns).  A wait that exceeds it records
 * FLEXQ_ERR_DEVICE_TIMEOUT in the device status word and the kernel returns.
 */
int flexq_set_wait_limit_ns(uint64_t limit_ns);

/*
 * flexq_debug_inject_stall -- test hook: when enabled, the next GEMM launch's
 * producer warp withholds its first stage, so every consumer's bounded wait
 * runs out.  The kernel must then report FLEXQ_ERR_DEVICE_TIMEOUT through
 * flexq_get_device_status() and leave the context usable.  One-shot.
 */
int flexq_debug_inject_stall(int enable);

/*
 * flexq_get_device_status -- synchronizes `stream`, reads the current
 * device's status word, clears it and returns FLEXQ_OK or the recorded error
 * (FLEXQ_ERR_DEVICE_TIMEOUT).  A failing CUDA call returns FLEXQ_ERR_CUDA.
 */
int flexq_get_device_status(void* stream);

#ifdef __cplusplus
}
#endif

#endif /* FLEXQ_H_ */
