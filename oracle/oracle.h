/*
 * CPU oracle for the fused MoE expert-FFN forward (test infrastructure only).
 *
 * This header belongs to the oracle alone.  Nothing in the CUDA library
 * includes it, and the oracle includes nothing from the CUDA library.  Only
 * the test suite, the smoke check and the CPU-baseline leg of the benchmark
 * load the shared object built from oracle.c.
 *
 * Every routine is a plain, slow restatement of a definition from the pages:
 *   [RFC]   "[RFC] Fused W8A8 MoE megakernel on H20" (Background, Design)
 *   [PFM]   "Prime Flash MoE: Fused MoE Kernels for Blackwell"
 *           (intro, API, Shapes, Scale layout (mxfp8), Constraints)
 * Floating point is accumulated in double.
 */
#ifndef MOE_ORACLE_H
#define MOE_ORACLE_H

#include <stdint.h>
#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- scalar formats ---------------------------------------------------- */
double orc_bf16_to_double(uint16_t bits);
uint16_t orc_double_to_bf16(double x);          /* round to nearest even */
double orc_e4m3_to_double(uint8_t code);        /* OCP E4M3 (fn): NaN for 0x7F/0xFF */
uint8_t orc_double_to_e4m3(double x);           /* RNE, saturate to +-448 */
double orc_e2m1_to_double(uint8_t code);        /* OCP E2M1 (FP4), 4-bit code */
double orc_e8m0_to_double(uint8_t code);        /* 2^(code-127); NaN for 0xFF */
/* OCP MX block scale for a block whose largest magnitude is amax (fp32). */
uint8_t orc_mx_scale_byte(float amax);
/* Quantise n fp32 values (n a multiple of 32) to e4m3 codes + e8m0 scales. */
void orc_mx_quantize(const float* v, int64_t n, uint8_t* codes, uint8_t* scales);

/* ---- planner (moe_align) ---------------------------------------------- */
int64_t orc_align_capacity(int T, int top_k, int E, int block_m);
int orc_moe_align(const int32_t* topk_ids, int T, int top_k, int E, int block_m,
                  int32_t* sorted_token_ids, int32_t* expert_ids,
                  int32_t* num_tokens_post_padded, int64_t capacity);

/* ---- router (softmax, top-k, renormalisation) -------------------------- */
/* bias may be NULL.  ids ranked by descending fp32 score logits+bias (ties:
 * lower index); weights in double; then n_shared routes per token to the
 * shared experts E.. with weight 1 (rows of top_k + n_shared).  Returns 0,
 * or -1 on bad sizes. */
int orc_route_topk(const float* logits, const float* bias, int T, int E, int top_k, int n_shared,
                   int32_t* topk_ids, double* topk_weights);

/* ---- blocked weight-scale layout --------------------------------------- */
int64_t orc_pack_scales_bytes(int E, int MN, int KS);
void orc_pack_scales_blocked(const uint8_t* in, uint8_t* out, int E, int MN, int KS);
void orc_unpack_scales_blocked(const uint8_t* in, uint8_t* out, int E, int MN, int KS);

/* ---- expert FFN -------------------------------------------------------- */
/* out rows are written only for the tokens listed in `tokens` (n_tokens of
 * them, or all T when tokens == NULL).  out_f64 (nullable, (T, K)) receives
 * the same rows before the final rounding to bf16.  nthreads <= 0 uses the
 * OpenMP default. */
void orc_fused_moe_bf16(const uint16_t* x, const uint16_t* w1, const uint16_t* w2,
                        const int32_t* topk_ids, const float* topk_weights,
                        int T, int K, int N, int E, int top_k,
                        const int32_t* tokens, int n_tokens, uint16_t* out, double* out_f64,
                        int nthreads);

/* w1_scales / w2_scales are ROW-MAJOR here: (E, N, K/32) and (E, K, (N/2)/32). */
void orc_fused_moe_mxfp8(const uint8_t* x, const uint8_t* x_scales,
                         const uint8_t* w1, const uint8_t* w1_scales,
                         const uint8_t* w2, const uint8_t* w2_scales,
                         const int32_t* topk_ids, const float* topk_weights,
                         int T, int K, int N, int E, int top_k,
                         const int32_t* tokens, int n_tokens, uint16_t* out, double* out_f64,
                         int nthreads);

/* As orc_fused_moe_mxfp8 with MXFP4 weights: w1 (E, N, K/2) and w2
 * (E, K, N/4) bytes of packed e2m1 codes (even index in the low nibble),
 * scales as for mxfp8. */
void orc_fused_moe_mxfp4(const uint8_t* x, const uint8_t* x_scales,
                         const uint8_t* w1, const uint8_t* w1_scales,
                         const uint8_t* w2, const uint8_t* w2_scales,
                         const int32_t* topk_ids, const float* topk_weights,
                         int T, int K, int N, int E, int top_k,
                         const int32_t* tokens, int n_tokens, uint16_t* out, double* out_f64,
                         int nthreads);

/* The fp32 SwiGLU intermediate of the mxfp8 (fp4 = 0) or MXFP4 (fp4 = 1)
 * forward before its requant, one row of N/2 floats per (listed token, route):
 * act is (n_tokens or T) x top_k x N/2; rows of routes outside [0, E) are 0. */
void orc_mx_intermediate(const uint8_t* x, const uint8_t* x_scales, const uint8_t* w1, const uint8_t* w1_scales,
                         const int32_t* topk_ids, int T, int K, int N, int E, int top_k,
                         const int32_t* tokens, int n_tokens, float* act, int nthreads, int fp4);

/* Number of OpenMP threads a parallel region gets (for reporting). */
int orc_max_threads(void);

#ifdef __cplusplus
}
#endif
#endif
