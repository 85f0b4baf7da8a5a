/*
 * apex_w4a4.h -- C ABI of the B200 (sm_100a) pure W4A4 group-quantized GEMM library.
 *
 * The operation: "APEX4: Efficient Pure W4A4 LLM Inference via Intra-SM Compute
 * Rebalancing" (abstract) -- both GEMM operands are 4-bit integers with one fp16 scale per
 * 128-wide K-group (the "W4A4-g128 kernel"); the INT4 tensor-core products of each group
 * are dequantised with the group scales and summed.  Its "mixed-granularity mode" keeps
 * 128-wide activation groups and uses coarser weight groups (here 512, or the whole row).
 *
 *   Y[m,n] = sum_g ( sum_{k in group g} qa[m,k] * qw[n,k] ) * sa[m,g] * sw[n, g*128/gw]
 *
 * Conventions shared by every entry point:
 *   - All tensor pointers are DEVICE pointers owned by the caller.  The library never
 *     allocates device memory.
 *   - Layouts are row-major with K contiguous.  Packed int4 rows: byte j of a row holds
 *     element k = 2j in bits 0..3 and k = 2j+1 in bits 4..7, as two's-complement nibbles.
 *     Scales are IEEE fp16, one per (row, group), row-major [rows][K/group].
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).  Every call
 *     only enqueues work: it returns once the kernels are launched.
 *   - Argument errors are detected on the host before anything is launched; nothing is
 *     enqueued and the call returns APEX_ERR_INVALID_ARG / _UNSUPPORTED / _ALIGNMENT.
 *     A failed launch returns APEX_ERR_CUDA.  Device-side problems (a pipeline wait that
 *     ran out of time) are recorded in a status word read by apex_get_device_status().
 */
#ifndef APEX_W4A4_H
#define APEX_W4A4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  APEX_OK = 0,
  APEX_ERR_INVALID_ARG = 1,  /* null pointer, non-positive size, K not a multiple of group */
  APEX_ERR_UNSUPPORTED = 2,  /* a group configuration this build does not implement */
  APEX_ERR_ALIGNMENT = 3,    /* a pointer without the alignment stated for it */
  APEX_ERR_CUDA = 4,         /* a CUDA runtime error (launch failure, no device, ...) */
  APEX_ERR_TIMEOUT = 5       /* a device-side pipeline wait gave up (see apex_get_device_status) */
} apex_status_t;

/*
 * Offline weight quantization and packing (per row, per K-group, symmetric).
 * Rule (the plainest reading of the method's "W4", with fp16 scales):
 *   s = fp16_rne(fp32(max_k |w[n,k]|) / 7)  (IEEE fp32 division),
 *   q = clamp(round_half_even(fp32(w) / fp32(s)), -8, 7), q = 0 when s == 0.
 *   w_f16        [N][K] fp16 (read)
 *   w_packed_u8  [N][K/2] bytes (written)
 *   w_scales_f16 [N][K/group_w] fp16 (written)
 * group_w: a multiple of 128 that divides K (128, 512, ..., K).  K % 128 == 0.
 * Alignment: w_f16 16 bytes, w_packed_u8 4 bytes, w_scales_f16 2 bytes.
 */
apex_status_t apex_pack_weights_int4(const void *w_f16, int64_t N, int64_t K, int32_t group_w,
                                     void *w_packed_u8, void *w_scales_f16, void *stream);

/*
 * Online per-token, per-group activation quantization and packing: the same rule as
 * apex_pack_weights_int4, applied to x_f16 [M][K] with group_a (128 for the GEMM).
 *   x_packed_u8 [M][K/2], x_scales_f16 [M][K/group_a].
 */
apex_status_t apex_quantize_act_int4(const void *x_f16, int64_t M, int64_t K, int32_t group_a,
                                     void *x_packed_u8, void *x_scales_f16, void *stream);

/*
 * Online activation quantization into the GEMM's expanded operand form (same rule and the
 * same q and scales as apex_quantize_act_int4; group_a must be 128).  x_q8 [M][K] bytes:
 * for every 8 consecutive elements k0..k7 of a row, bytes 0..3 hold 16*q(k0), 16*q(k2),
 * 16*q(k4), 16*q(k6) and bytes 4..7 hold 16*q(k1), 16*q(k3), 16*q(k5), 16*q(k7), as signed
 * 8-bit integers -- the values are still 4-bit; this is the order the tensor-core path
 * consumes, so the GEMM need not unpack activations.  Twice the bytes of the packed form;
 * worth it when M is large (prefill), where activation traffic is small next to the math.
 * x_q8 8-byte aligned (16 for the GEMM), x_scales_f16 [M][K/128].
 */
apex_status_t apex_quantize_act_int4_expanded(const void *x_f16, int64_t M, int64_t K,
                                              int32_t group_a, void *x_q8, void *x_scales_f16,
                                              void *stream);

/*
 * The W4A4 GEMM on expanded activations (from apex_quantize_act_int4_expanded): the same
 * result, arguments and rules as apex_w4a4_gemm, with a_q8 [M][K] in place of a_packed.
 */
apex_status_t apex_w4a4_gemm_expanded(int64_t M, int64_t N, int64_t K, int32_t group_a,
                                      int32_t group_w, const void *a_q8, const void *a_scales,
                                      const void *w_packed, const void *w_scales, void *y_f16,
                                      void *workspace, size_t workspace_bytes, void *stream);

/*
 * The W4A4 GEMM: y_f16[M][N] = fp16_rne(sum_g P_g * sa * sw), accumulated in fp32.
 *   a_packed [M][K/2], a_scales [M][K/group_a]   (from apex_quantize_act_int4)
 *   w_packed [N][K/2], w_scales [N][K/group_w]   (from apex_pack_weights_int4)
 * Supported: group_a == 128; group_w a multiple of 128 dividing K; K % 128 == 0;
 * M, N >= 1 (ragged tiles are handled).  a_packed / w_packed 16-byte aligned, scales and
 * y 2-byte aligned.
 * workspace: device scratch for split-K partial sums, may be NULL (then no split-K).
 *   Its size should be apex_w4a4_gemm_workspace_size(...); a smaller one limits the
 *   split.  Its first bytes hold per-tile arrival counters that must be zero before the
 *   first use (e.g. cudaMemset); every call that completes leaves them zero again.  Calls
 *   that share a workspace must not run concurrently, and a workspace used for one shape
 *   (M, N, K, group sizes) must be zeroed again before it serves another.
 */
apex_status_t apex_w4a4_gemm(int64_t M, int64_t N, int64_t K, int32_t group_a, int32_t group_w,
                             const void *a_packed, const void *a_scales, const void *w_packed,
                             const void *w_scales, void *y_f16, void *workspace,
                             size_t workspace_bytes, void *stream);

/*
 * The W4A4 GEMM whose output is also quantized as the next layer's activations (a chain of
 * W4A4 layers without a separate quantizer pass): the same computation and rules as
 * apex_w4a4_gemm, and additionally
 *   yq [M][N/2] packed int4 (yq_expanded == 0) or [M][N] 16*q bytes in the GEMM's
 *      expanded operand order (yq_expanded != 0), with yq_scales [M][N/128] fp16:
 * exactly what apex_quantize_act_int4 (or _expanded) would make, with group_a = 128, from
 * the fp16 Y this call computes -- every tile of 128 outputs is one K-group of the next
 * layer, so its scale and codes are made in the GEMM's epilogue.
 *   y_f16 may be NULL (then only yq and yq_scales are written).  Requires N % 128 == 0
 *   (APEX_ERR_UNSUPPORTED otherwise); yq 16-byte (as the next GEMM's operand needs) and
 *   yq_scales 2-byte aligned.
 */
apex_status_t apex_w4a4_gemm_quant(int64_t M, int64_t N, int64_t K, int32_t group_a,
                                   int32_t group_w, const void *a_packed, const void *a_scales,
                                   const void *w_packed, const void *w_scales, void *y_f16,
                                   void *yq, void *yq_scales, int32_t yq_expanded,
                                   void *workspace, size_t workspace_bytes, void *stream);

/* As apex_w4a4_gemm_quant, reading expanded activations (see apex_w4a4_gemm_expanded). */
apex_status_t apex_w4a4_gemm_expanded_quant(int64_t M, int64_t N, int64_t K, int32_t group_a,
                                            int32_t group_w, const void *a_q8,
                                            const void *a_scales, const void *w_packed,
                                            const void *w_scales, void *y_f16, void *yq,
                                            void *yq_scales, int32_t yq_expanded,
                                            void *workspace, size_t workspace_bytes,
                                            void *stream);

/*
 * Allocation-free variant of apex_w4a4_gemm.  The paper has no counterpart: this entry
 * point exists for callers that cannot allocate device memory while they run -- serving
 * runtimes that budget every device byte up front and hand out no scratch, plugin hosts
 * whose allocator the plugin may not call, and latency-critical paths that must avoid
 * cudaMalloc/cudaFree because those can stall or synchronize the device.
 * It computes exactly what apex_w4a4_gemm computes, with the same operand rules, but takes
 * no workspace: its split-K scratch is a fixed array of APEX_STATIC_SCRATCH_BYTES inside
 * the library, reserved on every GPU that loads the library until the process exits.  It
 * calls no allocator.  A problem whose scratch would exceed that size is refused with
 * APEX_ERR_UNSUPPORTED.
 * The first call on each device looks the array's device address up (with that device
 * current), so make that first call before any stream capture.  The address is kept for
 * the rest of the process: resetting the device (cudaDeviceReset) or destroying and
 * re-creating its primary context afterwards is not supported.  All calls on a device
 * share the one array and it keeps the previous call's contents (each call clears the
 * parts that must start at zero), so calls that overlap on the GPU -- on different
 * streams, or from different host threads -- race and must be ordered by the caller.
 */
#define APEX_STATIC_SCRATCH_BYTES (8u << 20)
apex_status_t apex_w4a4_gemm_noalloc(int64_t M, int64_t N, int64_t K, int32_t group_a,
                                     int32_t group_w, const void *a_packed, const void *a_scales,
                                     const void *w_packed, const void *w_scales, void *y_f16,
                                     void *stream);

/*
 * Online quantization and the W4A4 GEMM in one call: y_f16[M][N] from fp16 activations
 * x_f16 [M][K] (row-major, 16-byte aligned) and packed weights.  The activations are
 * quantized with exactly the rule of apex_quantize_act_int4 (group_a = 128) into the
 * workspace (packed below 128 tokens, the expanded form from 128 tokens on), then the GEMM
 * runs on them: the result equals apex_quantize_act_int4 followed by apex_w4a4_gemm.
 * workspace: at least apex_w4a4_linear_workspace_size(...) bytes (else
 *   APEX_ERR_INVALID_ARG), 256-byte aligned; its tail is the GEMM's split-K scratch, with
 *   apex_w4a4_gemm's zero-counter contract (zero it once before the first call).
 * The same group rules, alignment rules and errors as apex_w4a4_gemm otherwise.
 */
apex_status_t apex_w4a4_linear(int64_t M, int64_t N, int64_t K, int32_t group_a,
                               int32_t group_w, const void *x_f16, const void *w_packed,
                               const void *w_scales, void *y_f16, void *workspace,
                               size_t workspace_bytes, void *stream);

/* Workspace bytes apex_w4a4_linear needs for this problem (0 when it needs none). */
size_t apex_w4a4_linear_workspace_size(int64_t M, int64_t N, int64_t K, int32_t group_a,
                                       int32_t group_w);

/* Workspace bytes apex_w4a4_gemm would use for this problem (0 when it needs none). */
size_t apex_w4a4_gemm_workspace_size(int64_t M, int64_t N, int64_t K, int32_t group_a,
                                     int32_t group_w);

/*
 * ---- The E4M3-carrier forms, for compute-bound shapes (many tokens).
 *
 * The same 4-bit values q, one byte per element in element order, each byte the E4M3 code
 * of q (1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits; every q in [-8, 7] is an
 * E4M3 value).  The tensor cores multiply such operands with an fp32 accumulator
 * (kind::f8f6f4), which holds every group's integer partial exactly, so the GEMM below
 * computes exactly what apex_w4a4_gemm computes while the per-group dequantisation needs
 * no int-to-float conversion ("APEX4: Efficient Pure W4A4 LLM Inference via Intra-SM
 * Compute Rebalancing", abstract: the group dequantisation on the CUDA cores is the
 * bottleneck of the W4A4 GEMM).  Twice the bytes of the packed form: worth it where the
 * math, not memory traffic, bounds the GEMM.
 */

/*
 * Online activation quantization into E4M3 codes: the rule of apex_quantize_act_int4
 * (group_a must be 128), x_codes [M][K] bytes (8-byte aligned; 16 for the GEMM), x_scales_f16
 * [M][K/128] -- the same q and the same scales as the packed form.
 */
apex_status_t apex_quantize_act_int4_fp8(const void *x_f16, int64_t M, int64_t K,
                                         int32_t group_a, void *x_codes, void *x_scales_f16,
                                         void *stream);

/*
 * Offline weight quantization into E4M3 codes: the rule of apex_pack_weights_int4 (any
 * group_w it accepts), w_codes [N][K] bytes (8-byte aligned; 16 for the GEMM), w_scales_f16
 * [N][K/group_w] -- the same q and the same scales as the packed form.
 */
apex_status_t apex_pack_weights_int4_fp8(const void *w_f16, int64_t N, int64_t K,
                                         int32_t group_w, void *w_codes, void *w_scales_f16,
                                         void *stream);

/*
 * Packed int4 [rows][K/2] (the format of apex_pack_weights_int4) -> E4M3 codes of the same
 * values [rows][K].  K % 16 == 0; packed 8-byte and codes 16-byte aligned.
 */
apex_status_t apex_unpack_int4_fp8(const void *packed, int64_t rows, int64_t K, void *codes,
                                   void *stream);

/*
 * The W4A4 GEMM on E4M3-coded operands: y_f16 [M][N] = fp16_rne(sum_g P_g * sa * sw),
 * accumulated in fp32, the same result rule as apex_w4a4_gemm.
 *   a_codes [M][K], a_scales [M][K/128]       (from apex_quantize_act_int4_fp8)
 *   w_codes [N][K], w_scales [N][K/group_w]   (apex_pack_weights_int4_fp8 or
 *                                              apex_unpack_int4_fp8 + the packed scales)
 * group_a == 128, group_w a multiple of 128 dividing K, K % 128 == 0, M, N >= 1 (ragged tiles
 * handled).  a_codes / w_codes 16-byte aligned, scales and y 2-byte aligned.  No workspace:
 * tiles of 128 tokens x 256 outputs are never split.  Codes that are not E4M3 values of
 * integers in [-8, 7] give undefined results.
 */
apex_status_t apex_w4a4_gemm_fp8(int64_t M, int64_t N, int64_t K, int32_t group_a,
                                 int32_t group_w, const void *a_codes, const void *a_scales,
                                 const void *w_codes, const void *w_scales, void *y_f16,
                                 void *stream);

/*
 * The E4M3-carrier GEMM whose output is also quantized as the next layer's activations (a
 * chain of W4A4 layers without a separate quantizer pass): the computation and rules of
 * apex_w4a4_gemm_fp8, and additionally
 *   yq_codes [M][N] E4M3 codes, yq_scales [M][N/128] fp16:
 * exactly what apex_quantize_act_int4_fp8 (group_a = 128) would make from the fp16 Y this
 * call computes -- each tile holds every 128 outputs of a token that form one K-group of the
 * next layer.  y_f16 may be NULL (then only the quantized output is written).  N % 128 == 0
 * (APEX_ERR_UNSUPPORTED otherwise); yq_codes 16-byte, yq_scales 2-byte aligned.
 */
apex_status_t apex_w4a4_gemm_fp8_quant(int64_t M, int64_t N, int64_t K, int32_t group_a,
                                       int32_t group_w, const void *a_codes,
                                       const void *a_scales, const void *w_codes,
                                       const void *w_scales, void *y_f16, void *yq_codes,
                                       void *yq_scales, void *stream);

/*
 * Parity export of the E4M3-carrier GEMM: every exact per-group partial, as
 * apex_w4a4_group_partials, computed by the same tensor-core path as apex_w4a4_gemm_fp8
 * (its fp32 partials stored as int32).
 */
apex_status_t apex_w4a4_group_partials_fp8(int64_t M, int64_t N, int64_t K,
                                           const void *a_codes, const void *w_codes,
                                           int32_t *partials_i32, void *stream);

/*
 * Debug / parity export: the exact integer partial of every 128-wide K-group,
 *   partials_i32[g][m][n] = sum_{k in group g} qa[m,k] * qw[n,k],  g < K/128,
 * computed by the same tensor-core path as apex_w4a4_gemm (its epilogue replaced by a
 * store).  Same operand rules as apex_w4a4_gemm; partials_i32 4-byte aligned.
 */
apex_status_t apex_w4a4_group_partials(int64_t M, int64_t N, int64_t K, const void *a_packed,
                                       const void *w_packed, int32_t *partials_i32,
                                       void *stream);

/*
 * Synchronizes `stream`, then reads and clears the library's device status word.
 * Returns APEX_ERR_TIMEOUT if a kernel since the last call gave up waiting on its own
 * pipeline (its outputs are then undefined and a split-K workspace must be re-zeroed),
 * APEX_ERR_CUDA on a CUDA error, else APEX_OK.
 */
apex_status_t apex_get_device_status(void *stream);

/* Time limit, in nanoseconds, of every device-side pipeline wait (default 2e9). */
void apex_set_wait_limit_ns(uint64_t ns);

/* Static description of a status code (never NULL). */
const char *apex_status_string(apex_status_t status);

/*
 * Introspection: the work plan apex_w4a4_gemm would use for an M x N x K problem on a GPU
 * with `sms` SMs (with_workspace != 0: a large enough workspace is given).  Writes
 * plan[0..5] = { token tile BT, tiles, K-stages per tile, persistent CTAs, split-K (0/1),
 * CTAs per cluster (1: the parts of split tiles go through global memory) }.  Host only;
 * nothing is launched.  APEX_ERR_INVALID_ARG for a NULL plan, sms <= 0 or a bad shape.
 * The launch itself may still fall back from clusters to global memory when the clusters
 * would not all be resident at once on the actual device.
 */
apex_status_t apex_debug_gemm_plan(int64_t M, int64_t N, int64_t K, int32_t sms,
                                   int32_t with_workspace, int32_t *plan);

/*
 * The speed side of the APEX4 page's "rho-aware granularity adaptation" ("APEX4: Efficient
 * Pure W4A4 LLM Inference via Intra-SM Compute Rebalancing", abstract: the tensor-core to
 * CUDA-core throughput ratio rho governs the group-dequantisation bottleneck; the
 * mixed-granularity mode recovers the high-rho GPU).  Host only, no device work.
 *   rho:    dense integer tensor-core operations per second / fp32 CUDA-core operations per
 *           second (the page: 8 L40S, 16 RTX 3090 and A40, 64 A100; B200: about 60-64)
 *   ridge_ops_per_byte: tensor operations per second / HBM bytes per second
 * Returns the weight group for an M x N x K W4A4 GEMM with 128-wide activation groups: 128
 * when the GEMM is below the ridge (memory-bound: the dequantisation hides behind the weight
 * stream) or when rho is low enough that the 128-wide groups' dequantisation (one scale
 * product and one fma per partial) costs at most half of the tensor time (4*rho/256 <= 0.5);
 * otherwise K, one weight scale per output channel (only the fma remains per partial).
 * Returns 0 for invalid arguments (non-positive sizes or rates, K % 128 != 0).  Accuracy is
 * not modelled (it needs trained weights); the choice is the speed side only.
 */
int32_t apex_select_weight_group(int64_t M, int64_t N, int64_t K, double rho,
                                 double ridge_ops_per_byte);

/*
 * Test hook: the next GEMM launch on this host thread skips the bulk copy of pipeline stage
 * `step` (two or four K-groups, counted within each CTA), so its consumers wait until the
 * time limit.  -1 turns it off.  Used only to test the timeout path; never needed by callers.
 */
void apex_debug_withhold_step(int32_t step);

/*
 * Test hook: the next apex_w4a4_group_partials call on this host thread (on != 0) divides
 * the work as apex_w4a4_gemm does when given its workspace -- tiles split over several
 * CTAs, in stream-K pieces -- instead of whole tiles.  Every (tile, K-group) is still
 * handled by one CTA, which stores its partials, so the export needs no scratch; the hook
 * checks the split plans' K ranges bit for bit.  It applies to one call, then resets.
 */
void apex_debug_partials_split(int32_t on);

/*
 * Tracing hook: the next apex_w4a4_gemm launch on this host thread writes timestamps for
 * its first `ctas` CTAs (persistent CTA index) into the device buffer trace[ctas][16][steps]
 * (uint64).  SM clock cycles (clock64): [c][0][s] producer issued stage s (a pair of
 * K-groups), [c][1][s] converters done with stage s, [c][2][i] MMAs of K-group i issued,
 * [c][3][i] epilogue done with K-group i, [c][4][s] converter inputs of stage s ready,
 * [c][6][i] MMA inputs of K-group i ready (after the tensor-core fence), [c][7][i]
 * epilogue inputs of K-group i ready, [c][8][i] MMA waits returned, [c][9][i] MMAs of
 * K-group i issued before their commits, [c][10][i] MMA wait for the operands of K-group i
 * returned, [c][11 + w][s] converter warp w (0..3 within its warpgroup) done with stage s,
 * [c][15][4k .. 4k+3] the epilogue's k-th segment: finished, partial published (global
 * hand-off; [c][15][1] is also a cluster partner's send), parts received by the owner, tile
 * written;
 * [c][5][0] / [c][5][1] %globaltimer (ns) at CTA start / end, [c][5][2] the SM it ran on,
 * [c][5][3] clock64 at CTA start, [c][5][4] / [c][5][5] clock64 when the producer enters its
 * loop / has its first work item, [c][5][6] %globaltimer at kernel entry (before the
 * prologue).  Steps beyond `steps` are not recorded.  clock64 counts cycles of the SM clock
 * the kernel ran at (below the nominal maximum under load), so convert those stamps with
 * that clock, or compare them only with each other, not with the %globaltimer ones.
 */
void apex_debug_trace_next_gemm(uint64_t *trace, int32_t ctas, int32_t steps);

/*
 * ---- The outlier dual path ("OSC: Hardware Efficient W4A4 Quantization via Outlier
 * Separation in Channel Dimension", abstract): a fixed set of input channels, the same for
 * every token and chosen offline, bypasses 4-bit quantization and is multiplied in 16 bits;
 * the rest goes through the W4A4 GEMM.  Here the 16-bit product runs inside the E4M3-carrier
 * GEMM, as extra K-steps of every tile on the tensor cores (fp16 x fp16, fp32 accumulation),
 * and is added to the fp32 result before the single fp16 rounding of Y.
 *
 * channels: device int32 [C], the outlier channel indices, sorted ascending, distinct, each
 *   in [0, K) (a list that breaks this gives wrong values, never an out-of-bounds access).
 *   1 <= C <= K.  Cp >= C, Cp % 64 == 0: the width of the compact fp16 operands, whose
 *   columns C..Cp-1 are written as zeros.  channels 4-byte aligned.
 */

/* Output forms of apex_quantize_act_int4_dual. */
#define APEX_FORM_PACKED 0   /* packed int4, as apex_quantize_act_int4 */
#define APEX_FORM_EXPANDED 1 /* 16*q bytes, as apex_quantize_act_int4_expanded */
#define APEX_FORM_FP8 2      /* E4M3 codes, as apex_quantize_act_int4_fp8 */

/*
 * Offline: the weights' outlier columns, w_out [N][Cp] fp16 (column c = w[:, channels[c]]),
 * from w_f16 [N][K].  The 4-bit weights are quantized as usual (their outlier columns meet
 * zero activations).  w_f16 2-byte, w_out_f16 16-byte aligned.
 */
apex_status_t apex_gather_weight_columns(const void *w_f16, int64_t N, int64_t K,
                                         const void *channels, int32_t C, void *w_out_f16,
                                         int32_t Cp, void *stream);

/*
 * Online: the activation quantizer (group_a must be 128) in the given form, with the
 * outlier channels copied to x_out [M][Cp] fp16 (channel order of the list) and treated as
 * zeros by the 4-bit path, so that they do not set its group scales.  x_f16 and x_out_f16
 * 16-byte aligned; x_q 4-byte (packed) or 8-byte aligned; x_scales_f16 [M][K/128].
 */
apex_status_t apex_quantize_act_int4_dual(const void *x_f16, int64_t M, int64_t K,
                                          int32_t group_a, const void *channels, int32_t C,
                                          int32_t form, void *x_q, void *x_scales_f16,
                                          void *x_out_f16, int32_t Cp, void *stream);

/*
 * The dual-path GEMM: Y = W4A4(a_codes, a_scales, w_codes, w_scales) + x_out . w_out^T, the
 * 16-bit product accumulated in fp32 and added before the single fp16 rounding.  The operand
 * rules of apex_w4a4_gemm_fp8; x_out_f16 [M][Cp] (from apex_quantize_act_int4_dual with
 * APEX_FORM_FP8) and w_out_f16 [N][Cp] (apex_gather_weight_columns), both 16-byte aligned;
 * 64 <= Cp <= K, Cp % 64 == 0.
 */
apex_status_t apex_w4a4_gemm_fp8_dual(int64_t M, int64_t N, int64_t K, int32_t group_a,
                                      int32_t group_w, const void *a_codes,
                                      const void *a_scales, const void *w_codes,
                                      const void *w_scales, const void *x_out_f16,
                                      const void *w_out_f16, int32_t Cp, void *y_f16,
                                      void *stream);

#ifdef __cplusplus
}
#endif

#endif /* APEX_W4A4_H */
