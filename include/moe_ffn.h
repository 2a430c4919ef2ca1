/*
 * moe_ffn.h -- C ABI of the B200 (sm_100a) fused MoE expert-FFN forward.
 *
 * The operations and their arguments follow two pages:
 *   [PFM] "Prime Flash MoE: Fused MoE Kernels for Blackwell" -- sections
 *         intro (fused gate/up GEMM, SwiGLU consumed from the accumulator,
 *         down GEMM, top-k weighted reduction; mxfp8 requant of the
 *         intermediate), API, Shapes, Scale layout (mxfp8), Constraints.
 *   [RFC] "[RFC] Fused W8A8 MoE megakernel on H20" -- sections Background
 *         (the five local steps) and Design (planner: expert histogram,
 *         prefix sums, row-to-token mapping; compute megakernel).
 *
 * Conventions shared by every entry point
 *   - All tensor pointers are DEVICE pointers owned by the caller, contiguous
 *     and row-major.  The library never allocates device memory per call and
 *     never takes ownership of anything passed in.
 *   - Every call is asynchronous on `stream` (0 = legacy default stream) and
 *     never synchronises with the host.
 *   - Return value: MOE_OK (0) or a negative MOE_ERR_* code.  Arguments are
 *     checked before anything is launched; on an argument error nothing is
 *     launched and moe_last_error() describes the problem.  MOE_ERR_CUDA
 *     reports a launch failure (the CUDA error string is in moe_last_error()).
 *   - Faults found on the device (a bounded wait that ran out) are recorded
 *     in a device status word read by moe_device_status().
 *
 * Readings of points the pages leave open (see the design notes):
 *   - gate = rows [0, N/2) of w1[e], up = rows [N/2, N); act = silu(gate)*up.
 *   - Inside an expert's segment of sorted_token_ids, route ids ascend.
 *   - Unused capacity of sorted_token_ids and expert_ids is filled with -1.
 *   - A topk_ids entry outside [0, E) routes nowhere: it gets no slot, and
 *     contributes nothing to out.
 */
#ifndef MOE_FFN_H
#define MOE_FFN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Every entry point below is exported from libmoe_ffn.so. */
#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

typedef struct CUstream_st* moe_stream_t; /* same type as cudaStream_t */

enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = -1, /* null pointer, negative or inconsistent size */
  MOE_ERR_UNSUPPORTED = -2, /* a shape outside the supported constraints   */
  MOE_ERR_ALIGNMENT = -3,   /* a pointer not aligned as the kernel needs   */
  MOE_ERR_WORKSPACE = -4,   /* workspace missing or smaller than required  */
  MOE_ERR_CUDA = -5,        /* a CUDA runtime / driver call failed         */
  MOE_ERR_TIMEOUT = -6      /* a device-side bounded wait ran out          */
};

enum { MOE_DTYPE_BF16 = 0, MOE_DTYPE_MXFP8 = 1, MOE_DTYPE_MXFP4 = 2 };

/* Message describing the last error returned on the calling host thread. */
MOE_API const char* moe_last_error(void);

/* Waits for `stream`, then returns MOE_OK, or MOE_ERR_TIMEOUT if a kernel of
 * this library running on the current device gave up a bounded wait since the
 * previous call; the status word is cleared. */
MOE_API int moe_device_status(moe_stream_t stream);

/* ------------------------------------------------------------------------
 * moe_align -- the routing planner.
 * [RFC] Design: count routed tokens per expert (histogram), prefix sums over
 * the counts, row-to-token mapping.  [PFM] API / Shapes: sorted_token_ids
 * holds flattened token*top_k+route ids grouped by expert, each group padded
 * to a multiple of block_m with -1; expert_ids gives the expert of every
 * block_m block; num_tokens_post_padded the padded total.
 *
 *   topk_ids            (T, top_k) int32, device, read only.
 *   sorted_token_ids    capacity int32, device, written in full: ids of the
 *                       routes to expert 0 (ascending), -1 up to a multiple
 *                       of block_m, then expert 1, ...; -1 from
 *                       num_tokens_post_padded to capacity.
 *   expert_ids          ceil(capacity / block_m) int32, device, written in
 *                       full: expert of block b for b < ntpp / block_m,
 *                       else -1.  Experts with no routes get no block.
 *   num_tokens_post_padded  one int32, device: sum over experts of
 *                       ceil(count / block_m) * block_m.
 *   capacity            must be >= moe_align_capacity(T, top_k, E, block_m).
 * Constraints: T >= 0, top_k >= 1, 1 <= E <= 1024, block_m in {16, 32, 64,
 * 128}; T * top_k + E * (block_m - 1) < 2^31.  T = 0 is allowed.
 * ---------------------------------------------------------------------- */
MOE_API int64_t moe_align_capacity(int T, int top_k, int E, int block_m);
MOE_API int moe_align(const int32_t* topk_ids, int T, int top_k, int E, int block_m,
              int32_t* sorted_token_ids, int32_t* expert_ids, int32_t* num_tokens_post_padded,
              int64_t capacity, moe_stream_t stream);

/* ------------------------------------------------------------------------
 * moe_route_align -- the router fused ahead of the planner: softmax over the
 * experts, top-k, renormalised weights, then exactly what moe_align does on
 * the resulting ids.  [PFM] Usage: topk_ids come from the caller's gate;
 * [RFC] Results so far: both paths use the same normalized routing weights.
 * Reading: score z[t][e] = logits[t][e] + bias[e] formed in fp32; experts
 * ranked by descending z, equal scores by ascending index; the first top_k
 * kept, weight j = exp(z_j - z_0) / sum over the kept of exp(z_i - z_0).
 *
 *   logits              (T, E) fp32, device, row major, read only; finite.
 *   bias                (E) fp32, device, or NULL for none.
 *   n_shared            shared experts (>= 0): every token also routes to
 *                       experts E .. E+n_shared-1 with weight 1 (reading: a
 *                       shared expert processes every token and its output
 *                       is added to the routed sum).  The FFN then runs with
 *                       E + n_shared experts (the shared ones stored after
 *                       the routed ones in w1/w2) and top_k + n_shared
 *                       routes per token, in the same fused kernels.
 *   topk_ids            (T, top_k + n_shared) int32, device, written: kept
 *                       experts in rank order, then the shared experts.
 *   topk_weights        (T, top_k + n_shared) fp32, device, written; the
 *                       routed part of each row sums to 1, shared entries 1.
 *   sorted_token_ids, expert_ids, num_tokens_post_padded, capacity: as for
 *                       moe_align on topk_ids with E + n_shared experts
 *                       (capacity >= moe_align_capacity(T, top_k + n_shared,
 *                       E + n_shared, block_m)).
 * Batches of at most 32 tokens are routed inside the planner's CTA; larger
 * ones by an all-SM router kernel chained to the planner.
 * Constraints: as moe_align, plus 1 <= top_k <= min(8, E), top_k + n_shared
 * <= 32 and E + n_shared <= 1024.  Returns
 * MOE_ERR_UNSUPPORTED / MOE_ERR_INVALID_ARG before any launch otherwise.
 * ---------------------------------------------------------------------- */
MOE_API int moe_route_align(const float* logits, const float* bias, int T, int E, int top_k, int n_shared,
                    int block_m, int32_t* topk_ids, float* topk_weights, int32_t* sorted_token_ids,
                    int32_t* expert_ids, int32_t* num_tokens_post_padded, int64_t capacity,
                    moe_stream_t stream);

/* ------------------------------------------------------------------------
 * pack_scales_blocked -- [PFM] Scale layout (mxfp8): weight scales (one e8m0
 * byte per 32 along K) reordered into a sequence of 512-byte tiles, each
 * covering 128 rows (MN) x 128 K (4 scale bytes).  Tile (e, mt, kt) starts at
 * byte ((e * MT + mt) * KT + kt) * 512 with MT = ceil(MN/128),
 * KT = ceil(KS/4); inside a tile, row r and scale column c sit at byte
 * (r % 32) * 16 + (r / 32) * 4 + c (the 128 x 4 scale-factor arrangement the
 * Blackwell block-scaled MMA reads).  Bytes outside (MN, KS) are written 0.
 *
 *   in   (E, MN, KS) uint8, row major, device.
 *   out  pack_scales_blocked_bytes(E, MN, KS) bytes, device, written in full.
 * Run once at weight-load time, not per step.
 * ---------------------------------------------------------------------- */
MOE_API int64_t pack_scales_blocked_bytes(int E, int MN, int KS);
MOE_API int pack_scales_blocked(const uint8_t* in, uint8_t* out, int E, int MN, int KS,
                        moe_stream_t stream);

/* ------------------------------------------------------------------------
 * Workspace -- [PFM] intro, the split=True form: the activation is written
 * to a workspace once and read back by the down projection.
 * fused_moe_* need caller-owned device scratch of at least
 * moe_workspace_bytes(...) bytes, 256-byte aligned.  It holds the SwiGLU
 * intermediate of every routed row (written once, read once by the down
 * projection), the weighted down-projection rows of every route, and one
 * flag per route.  Its contents need no initialisation and are garbage
 * afterwards; two calls that overlap in time must not share it.
 * ---------------------------------------------------------------------- */
MOE_API int64_t moe_workspace_bytes(int dtype, int T, int K, int N, int E, int top_k, int block_m);

/* Optional tuning knobs; pass NULL for the defaults (0 / NULL in a field
 * also means "default"). */
typedef struct moe_tuning {
  int stages;   /* shared-memory pipeline depth of the GEMM phases        */
  int num_ctas; /* persistent CTAs per phase (default: one per SM)        */
  /* Timing hook: if non-NULL, four caller-created cudaEvent_t handles that
   * are recorded on `stream` before the gate/up phase, between it (with the
   * split-K reduction after it) and the down phase, between the down phase
   * and the top-k reduction, and after the reduction. */
  void* const* phase_events;
  /* Limit, in ns of the GPU's global timer, of every bounded wait inside the
   * fused kernels (0: the default of 2 s).  A wait that runs out makes its
   * kernel stop, and moe_device_status() then reports MOE_ERR_TIMEOUT; the
   * call's out is undefined.  A tiny limit is a way to exercise that path;
   * it has no other use. */
  long long wait_timeout_ns;
  /* fused_moe_bf16 only: 0 lets the library choose between the tensor-core
   * phases and the small-batch form (two kernels that stream each touched
   * weight row once through warp-level MMAs, then the same top-k combine;
   * taken by default when T * top_k <= 128); 1 takes the small-batch form
   * whenever the shapes allow it (K and N/2 multiples of 256, T <= 8192);
   * -1 never.  Both give the same result within the bf16 tolerance; the
   * phase events then mark its gate/up kernel, down kernel and combine. */
  int small_batch;
} moe_tuning;

/* ------------------------------------------------------------------------
 * fused_moe_bf16 -- [PFM] intro / API / Shapes, bf16 path; [RFC] Background
 * steps 2-5.  For every routed row (token t, route j, expert e):
 *   H   = w1[e] . x[t]                  (N values, fp32 accumulation)
 *   a_i = bf16( silu(H_i) * H_{N/2+i} )  i < N/2
 *   Y   = w2[e] . a                      (K values, fp32 accumulation)
 * and out[t] = bf16( sum_j topk_weights[t, j] * Y_(t, j) ).
 *
 *   x             (T, K) bf16            w1 (E, N, K) bf16
 *   w2            (E, K, N/2) bf16       out (T, K) bf16, overwritten
 *   topk_weights  (T, top_k) fp32
 *   sorted_token_ids / expert_ids / num_tokens_post_padded: moe_align's
 *                 outputs for the same (T, top_k, E, block_m, capacity).
 * Constraints: K % 128 == 0, N % 16 == 0, N >= 16, block_m in {16, 32, 64,
 * 128}; every pointer 16-byte aligned, workspace 256-byte aligned.
 * Small batches ([RFC] Background: decode-sized calls stream their experts'
 * weights with little arithmetic per byte) -- T * top_k <= 128 with K and
 * N/2 multiples of 256, or as moe_tuning.small_batch says -- run as two
 * weight-streaming kernels (warp-level MMAs) after the planner, then the
 * same combine: the same result up to fp32 summation order, deterministic.
 * ---------------------------------------------------------------------- */
MOE_API int fused_moe_bf16(const void* x, const void* w1, const void* w2,
                   const int32_t* sorted_token_ids, const int32_t* expert_ids,
                   const int32_t* num_tokens_post_padded, const float* topk_weights, void* out,
                   int T, int K, int N, int E, int top_k, int block_m, int64_t capacity,
                   void* workspace, int64_t workspace_bytes, const moe_tuning* tune,
                   moe_stream_t stream);

/* ------------------------------------------------------------------------
 * fused_moe_mxfp8 -- [PFM] intro / API / Scale layout (mxfp8), mxfp8 path:
 * e4m3 values with one e8m0 scale per 32 along the contraction dimension on
 * both operands of both GEMMs, fp32 accumulation; the SwiGLU intermediate is
 * requantised on chip (per routed row, per 32 along N/2: amax, e8m0 scale
 * 2^(floor(log2 amax) - 8), e4m3 round-to-nearest-even with saturation)
 * before the down GEMM; bf16 out.
 *
 *   x_e4m3 (T, K) u8            x_scales (T, K/32) u8 e8m0, ROW MAJOR
 *   w1_e4m3 (E, N, K) u8        w1_scales_blocked = pack_scales_blocked of
 *                               the (E, N, K/32) scales
 *   w2_e4m3 (E, K, N/2) u8      w2_scales_blocked = pack_scales_blocked of
 *                               the (E, K, N/64) scales
 *   other arguments as fused_moe_bf16.
 * Constraints: K % 256 == 0, N % 256 == 0, block_m in {16, 32, 64, 128}.
 * ---------------------------------------------------------------------- */
MOE_API int fused_moe_mxfp8(const uint8_t* x_e4m3, const uint8_t* x_scales, const uint8_t* w1_e4m3,
                    const uint8_t* w1_scales_blocked, const uint8_t* w2_e4m3,
                    const uint8_t* w2_scales_blocked, const int32_t* sorted_token_ids,
                    const int32_t* expert_ids, const int32_t* num_tokens_post_padded,
                    const float* topk_weights, void* out, int T, int K, int N, int E, int top_k,
                    int block_m, int64_t capacity, void* workspace, int64_t workspace_bytes,
                    const moe_tuning* tune, moe_stream_t stream);

/* ------------------------------------------------------------------------
 * fused_moe_mxfp4 -- mxfp8 activations with MXFP4 weights (DeepGEMM #411
 * "SM90 FP8 x MXFP4 MegaMoE" pairs these operand formats; the element format
 * is OCP MX v1.0 FP4, E2M1).  The forward is fused_moe_mxfp8's; only the
 * weight encoding differs: e2m1 values (sign, 2 exponent bits with bias 1,
 * 1 mantissa bit: magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6) with one e8m0
 * scale per 32 along the contraction dimension, two values per byte, the
 * even-indexed value in the low nibble.  Half the weight bytes of mxfp8.
 *
 *   w1_e2m1 (E, N, K/2) u8      w1_scales_blocked as for fused_moe_mxfp8
 *   w2_e2m1 (E, K, N/4) u8      w2_scales_blocked as for fused_moe_mxfp8
 *   other arguments as fused_moe_mxfp8; workspace from
 *   moe_workspace_bytes(MOE_DTYPE_MXFP4, ...).
 * Constraints: as fused_moe_mxfp8, plus w1 and w2 32-byte aligned.
 * ---------------------------------------------------------------------- */
MOE_API int fused_moe_mxfp4(const uint8_t* x_e4m3, const uint8_t* x_scales, const uint8_t* w1_e2m1,
                    const uint8_t* w1_scales_blocked, const uint8_t* w2_e2m1,
                    const uint8_t* w2_scales_blocked, const int32_t* sorted_token_ids,
                    const int32_t* expert_ids, const int32_t* num_tokens_post_padded,
                    const float* topk_weights, void* out, int T, int K, int N, int E, int top_k,
                    int block_m, int64_t capacity, void* workspace, int64_t workspace_bytes,
                    const moe_tuning* tune, moe_stream_t stream);

/* ------------------------------------------------------------------------
 * Expert-parallel dispatch and combine -- DeepGEMM #411 "SM90 FP8 x MXFP4
 * MegaMoE", Summary, and "[SM90] Ring-buffered FP8 MegaMoE with a lag-ordered
 * L1/L2 schedule" (sgl DeepGEMM PR #88): the experts are sharded over the
 * `world` ranks of a group (rank r owns experts [r*E/world, (r+1)*E/world)),
 * each routed row goes to the owner of its expert (dispatch), the owners run
 * their experts, and the results come back to be summed per token (combine).
 * The exchanges are the caller's collectives; these calls do the device work
 * on either side.  All pointers device, caller-owned; asynchronous on
 * `stream`.  Constraints: 1 <= world <= 64, E % world == 0.
 *
 * moe_ep_dispatch_plan -- order (T*top_k int32, written in full): the route
 *   ids t*top_k+j whose expert is in [0, E), grouped by owner rank (rank 0
 *   first), ascending inside a group, then -1; send_counts (world int32): the
 *   size of each group.
 * moe_ep_dispatch_pack -- for i < n (n = sum of send_counts): rows_out[i] =
 *   the row (row_bytes bytes) of x of token order[i] / top_k; scales_out[i] =
 *   its scale row (scale_bytes bytes) when x_scales is not NULL;
 *   local_expert_out[i] = its expert minus the owner's first expert;
 *   weight_out[i] = its routing weight.  x and rows_out 16-byte aligned when
 *   row_bytes % 16 == 0.
 * moe_ep_combine -- y (n, K) bf16: the returned rows, row i for route
 *   order[i]; slot: T*top_k int32 scratch; out (T, K) bf16, overwritten:
 *   out[t] = bf16( sum over j of y[row of route t*top_k+j] ), routes in order,
 *   fp32 sums; a token none of whose routes is in `order` gets zeros.  K % 8
 *   == 0; y and out 16-byte aligned.
 * ---------------------------------------------------------------------- */
MOE_API int moe_ep_dispatch_plan(const int32_t* topk_ids, int T, int top_k, int E, int world, int32_t* order,
                                 int32_t* send_counts, moe_stream_t stream);
MOE_API int moe_ep_dispatch_pack(const void* x, int64_t row_bytes, const uint8_t* x_scales, int64_t scale_bytes,
                                 const int32_t* topk_ids, const float* topk_weights, const int32_t* order, int n,
                                 int T, int top_k, int E, int world, void* rows_out, uint8_t* scales_out,
                                 int32_t* local_expert_out, float* weight_out, moe_stream_t stream);
MOE_API int moe_ep_combine(const void* y, const int32_t* order, int n, int T, int top_k, int K, int32_t* slot,
                           void* out, moe_stream_t stream);

/* ------------------------------------------------------------------------
 * fused_moe_bf16_noalloc -- the pages have no counterpart to this call; it
 * is a convenience of this library.  It computes exactly what
 * fused_moe_bf16 computes, for callers that cannot allocate device memory
 * for the workspace: a plain C host program that links only this library
 * and has no device allocator of its own, or an application whose memory
 * pool owns all device memory and forbids further cudaMalloc calls.
 *
 * The workspace is a file-scope device array of MOE_NOALLOC_SCRATCH_BYTES
 * inside the library; every GPU that loads the library holds it until the
 * process exits.  Problems whose moe_workspace_bytes(MOE_DTYPE_BF16, ...)
 * exceeds that size are rejected with MOE_ERR_WORKSPACE before anything is
 * launched (small batches fit; e.g. T=64, K=N=1024, E=8, top_k=2 needs
 * about 1.2 MB, while E=256 experts with N=4096 need far more and must use
 * fused_moe_bf16).  The call allocates nothing.
 *
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture begins.
 *   - All calls share the one array, which keeps the last call's contents;
 *     nothing in it has to start at zero.  Calls whose kernels overlap on
 *     the GPU (different streams, or different host threads) race on it and
 *     must be serialised by the caller.
 *   Arguments, constraints and errors otherwise as fused_moe_bf16.
 * ---------------------------------------------------------------------- */
#define MOE_NOALLOC_SCRATCH_BYTES (16 * 1024 * 1024)
MOE_API int64_t fused_moe_bf16_noalloc_max_workspace(void);
MOE_API int fused_moe_bf16_noalloc(const void* x, const void* w1, const void* w2,
                                   const int32_t* sorted_token_ids, const int32_t* expert_ids,
                                   const int32_t* num_tokens_post_padded, const float* topk_weights,
                                   void* out, int T, int K, int N, int E, int top_k, int block_m,
                                   int64_t capacity, const moe_tuning* tune, moe_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* MOE_FFN_H */
