/*
 * CPU oracle for the fused MoE expert-FFN forward.
 *
 * TEST INFRASTRUCTURE.  Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference legs of bench.py load this library.  The product
 * path (the CUDA library and its Python binding) never does.
 *
 * Plain C, double accumulation, loops written in the order of the definitions
 * on the pages; no blocking, no fusion, no reordering.  Sources:
 *   [RFC] "[RFC] Fused W8A8 MoE megakernel on H20": Background (the five local
 *         steps: count/gather, gate/up GroupGEMM, SiLU x gate + requant, down
 *         GroupGEMM, top-k weighted reduction) and Design (histogram, prefix
 *         sums, row-to-token mapping).
 *   [PFM] "Prime Flash MoE: Fused MoE Kernels for Blackwell": intro (SwiGLU
 *         consumed from the accumulator, mxfp8 requant of the intermediate),
 *         API (moe_align outputs), Shapes (x, w1, w2, out, topk_weights, the
 *         flattened token*top_k+route ids padded with -1), Scale layout
 *         (mxfp8) (row-major activation scales, 512-byte blocked weight-scale
 *         tiles of 128 MN x 128 K, OCP MX quantiser).
 * Readings where the pages are silent (gate = rows [0, N/2) of w1, stable
 * order inside an expert segment, -1 in unused capacity, e8m0 byte 0 for an
 * all-zero block, saturation to +-448, round-to-nearest-even everywhere) are
 * listed in the design notes and repeated beside the code that takes them.
 *
 * Parity status: every function here is pinned by tests/test_oracle_*.py
 * (closed forms, invariants, brute force, torch float64 / float8 library
 * routines on special cases).  Nothing is "parity unpinned".
 */
#include "oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ====================================================================== */
/* scalar formats                                                          */
/* ====================================================================== */

double orc_bf16_to_double(uint16_t bits) {
  uint32_t u = (uint32_t)bits << 16;
  float f;
  memcpy(&f, &u, 4);
  return (double)f;
}

/* Round a double to the nearest bfloat16 (8 significant bits, fp32 exponent
 * range), ties to even, overflow to infinity (IEEE default rounding). */
uint16_t orc_double_to_bf16(double x) {
  if (isnan(x)) return 0x7FC0;
  if (x == 0.0) return signbit(x) ? 0x8000 : 0x0000;
  int e;
  (void)frexp(x, &e);               /* |x| = m * 2^e, 0.5 <= m < 1 */
  int qe = e < -125 ? -125 : e;     /* smallest normal binade is 2^-126 */
  double quantum = ldexp(1.0, qe - 8);
  double q = nearbyint(x / quantum) * quantum;   /* default mode: ties-to-even */
  const double maxv = ldexp(255.0, 127 - 7);     /* (2 - 2^-7) * 2^127 */
  float f;
  if (fabs(q) > maxv) f = (float)(q > 0 ? INFINITY : -INFINITY);
  else f = (float)q;                              /* exact: q has <= 8 bits */
  uint32_t u;
  memcpy(&u, &f, 4);
  return (uint16_t)(u >> 16);
}

/* OCP E4M3 ("fn" flavour): bias 7, 3 mantissa bits, no infinities,
 * S.1111.111 is NaN, largest finite 448, subnormals m * 2^-9. */
double orc_e4m3_to_double(uint8_t code) {
  int s = code >> 7, ex = (code >> 3) & 0xF, m = code & 7;
  if (ex == 0xF && m == 7) return NAN;
  double v = ex == 0 ? ldexp((double)m, -9) : ldexp(1.0 + m / 8.0, ex - 7);
  return s ? -v : v;
}

/* Round to nearest e4m3, ties to even, magnitudes beyond 448 saturate. */
uint8_t orc_double_to_e4m3(double x) {
  if (isnan(x)) return 0x7F;
  uint8_t sign = signbit(x) ? 0x80 : 0x00;
  double a = fabs(x);
  if (a == 0.0) return sign;
  int e;
  (void)frexp(a, &e);               /* 2^(e-1) <= a < 2^e */
  int qe = e < -5 ? -5 : e;         /* smallest normal binade 2^-6 */
  double quantum = ldexp(1.0, qe - 4);            /* 4 significant bits */
  double q = nearbyint(a / quantum) * quantum;
  if (q > 448.0) q = 448.0;
  /* encode the (exactly representable) magnitude q */
  if (q < ldexp(1.0, -6)) {                       /* subnormal or zero */
    int m = (int)nearbyint(q / ldexp(1.0, -9));
    return sign | (uint8_t)m;
  }
  int qe2;
  double mq = frexp(q, &qe2);                     /* q = mq * 2^qe2 */
  int ex = qe2 - 1 + 7;                            /* biased exponent */
  int m = (int)nearbyint((mq * 2.0 - 1.0) * 8.0);
  return sign | (uint8_t)(ex << 3) | (uint8_t)m;
}

/* OCP E2M1 (FP4): bias 1, one mantissa bit, no infinities or NaN; the
 * magnitudes are 0, 0.5 (subnormal), 1, 1.5, 2, 3, 4, 6.  code is 4 bits. */
double orc_e2m1_to_double(uint8_t code) {
  int s = (code >> 3) & 1, ex = (code >> 1) & 3, m = code & 1;
  double v = ex == 0 ? 0.5 * m : ldexp(1.0 + 0.5 * m, ex - 1);
  return s ? -v : v;
}

double orc_e8m0_to_double(uint8_t code) {
  if (code == 0xFF) return NAN;
  return ldexp(1.0, (int)code - 127);
}

/* OCP MX v1.0 shared scale: X = 2^(floor(log2(amax)) - emax_elem), with
 * emax_elem = 8 for E4M3, stored as the biased e8m0 byte.  An all-zero block
 * takes byte 0 (reading: the spec leaves log2(0) open).  Clamped to the
 * finite e8m0 range [2^-127, 2^127]. */
uint8_t orc_mx_scale_byte(float amax) {
  if (!(amax > 0.0f)) return 0;
  int e;
  (void)frexp((double)amax, &e);    /* floor(log2(amax)) = e - 1, exact */
  int shared = (e - 1) - 8;
  if (shared < -127) shared = -127;
  if (shared > 127) shared = 127;
  return (uint8_t)(shared + 127);
}

void orc_mx_quantize(const float* v, int64_t n, uint8_t* codes, uint8_t* scales) {
  for (int64_t b = 0; b < n / 32; ++b) {
    float amax = 0.0f;
    for (int i = 0; i < 32; ++i) {
      float a = fabsf(v[b * 32 + i]);
      if (a > amax) amax = a;
    }
    uint8_t sb = orc_mx_scale_byte(amax);
    scales[b] = sb;
    double X = orc_e8m0_to_double(sb);
    for (int i = 0; i < 32; ++i) codes[b * 32 + i] = orc_double_to_e4m3((double)v[b * 32 + i] / X);
  }
}

/* ====================================================================== */
/* planner: moe_align                                                     */
/* [RFC] Design: expert histogram, prefix sums, row-to-token mapping.     */
/* [PFM] API / Shapes: sorted_token_ids holds flattened token*top_k+route */
/* ids grouped by expert and padded to block_m with -1; expert_ids gives  */
/* the expert of each block_m block; num_tokens_post_padded the total.    */
/* ====================================================================== */

int64_t orc_align_capacity(int T, int top_k, int E, int block_m) {
  return (int64_t)T * top_k + (int64_t)E * (block_m - 1);
}

int orc_moe_align(const int32_t* topk_ids, int T, int top_k, int E, int block_m,
                  int32_t* sorted_token_ids, int32_t* expert_ids,
                  int32_t* num_tokens_post_padded, int64_t capacity) {
  const int64_t R = (int64_t)T * top_k;
  int64_t* count = (int64_t*)calloc((size_t)E, sizeof(int64_t));
  int64_t* off = (int64_t*)calloc((size_t)E + 1, sizeof(int64_t));
  int64_t* cursor = (int64_t*)calloc((size_t)E, sizeof(int64_t));
  if (!count || !off || !cursor) { free(count); free(off); free(cursor); return -1; }

  /* step 1: histogram (ids outside [0, E) are not routed anywhere) */
  for (int64_t i = 0; i < R; ++i) {
    int e = topk_ids[i];
    if (e >= 0 && e < E) count[e] += 1;
  }
  /* step 2: exclusive prefix sum of counts padded up to block_m */
  off[0] = 0;
  for (int e = 0; e < E; ++e) {
    int64_t padded = (count[e] + block_m - 1) / block_m * block_m;
    off[e + 1] = off[e] + padded;
  }
  const int64_t ntpp = off[E];
  if (ntpp > capacity) { free(count); free(off); free(cursor); return -2; }
  *num_tokens_post_padded = (int32_t)ntpp;

  /* step 3: row-to-token map.  Every slot starts as -1 (padding and unused
   * capacity); ids are placed in ascending flattened order, so each expert
   * segment is stable (reading: the pages fix no order inside a segment). */
  for (int64_t p = 0; p < capacity; ++p) sorted_token_ids[p] = -1;
  for (int64_t i = 0; i < R; ++i) {
    int e = topk_ids[i];
    if (e < 0 || e >= E) continue;
    sorted_token_ids[off[e] + cursor[e]] = (int32_t)i;
    cursor[e] += 1;
  }
  /* expert of every block; -1 for blocks past the last padded segment */
  const int64_t nblk_cap = (capacity + block_m - 1) / block_m;
  for (int64_t b = 0; b < nblk_cap; ++b) expert_ids[b] = -1;
  for (int e = 0; e < E; ++e)
    for (int64_t p = off[e]; p < off[e + 1]; p += block_m) expert_ids[p / block_m] = e;

  free(count); free(off); free(cursor);
  return 0;
}

/* ====================================================================== */
/* Router ahead of the planner.  "Prime Flash MoE", Usage: topk_ids come  */
/* from the caller's gate; "[RFC] Fused W8A8 MoE megakernel on H20",      */
/* Results so far: both paths run with the same normalized routing        */
/* weights.  Reading taken (the plainest one those two support): a        */
/* softmax over the experts of a per-expert score, the top_k largest kept */
/* and their probabilities renormalised to sum to one.                    */
/*  - score z[t][e] = logits[t][e] + bias[e], formed in fp32: the scores  */
/*    decide integer ids, so the decision is taken in the precision the   */
/*    device forms them in;                                               */
/*  - experts ranked by descending z, equal scores by ascending index;    */
/*  - weight of kept expert j = exp(z_j) / sum over kept i of exp(z_i),   */
/*    in double (the full softmax denominator cancels in the              */
/*    renormalisation), evaluated as exp(z_j - z_max) for range.          */
/* Scores must be finite.                                                 */
/* Shared experts (n_shared >= 0) follow the routed ones: every token     */
/* gets n_shared more routes, to experts E .. E+n_shared-1, weight 1 --   */
/* reading: a shared expert processes every token and its output is added */
/* to the routed sum (the pages name shared experts beside routed ones in */
/* the fused megakernels of the sgl DeepGEMM PR and DeepGEMM #411 without */
/* further definition).  Row t of the outputs holds top_k + n_shared      */
/* entries.                                                               */
/* ====================================================================== */

int orc_route_topk(const float* logits, const float* bias, int T, int E, int top_k, int n_shared,
                   int32_t* topk_ids, double* topk_weights) {
  if (T < 0 || E < 1 || top_k < 1 || top_k > E || n_shared < 0) return -1;
  const int kk = top_k + n_shared;
  float* z = (float*)malloc((size_t)E * sizeof(float));
  unsigned char* taken = (unsigned char*)malloc((size_t)E);
  if (!z || !taken) { free(z); free(taken); return -1; }
  for (int t = 0; t < T; ++t) {
    for (int e = 0; e < E; ++e) {
      const float b = bias ? bias[e] : 0.0f;
      z[e] = logits[(int64_t)t * E + e] + b; /* one fp32 addition */
      taken[e] = 0;
    }
    int32_t* ids = topk_ids + (int64_t)t * kk;
    double* w = topk_weights + (int64_t)t * kk;
    /* selection: repeatedly the largest remaining score, lowest index first */
    for (int j = 0; j < top_k; ++j) {
      int best = -1;
      for (int e = 0; e < E; ++e) {
        if (taken[e]) continue;
        if (best < 0 || z[e] > z[best]) best = e;
      }
      taken[best] = 1;
      ids[j] = best;
    }
    /* renormalised softmax over the kept experts */
    const double zmax = (double)z[ids[0]];
    double sum = 0.0;
    for (int j = 0; j < top_k; ++j) {
      w[j] = exp((double)z[ids[j]] - zmax);
      sum += w[j];
    }
    for (int j = 0; j < top_k; ++j) w[j] /= sum;
    for (int j = 0; j < n_shared; ++j) {
      ids[top_k + j] = E + j;
      w[top_k + j] = 1.0;
    }
  }
  free(z);
  free(taken);
  return 0;
}

/* ====================================================================== */
/* [PFM] Scale layout (mxfp8): weight scales reordered into a sequence of */
/* 512-byte tiles, each covering 128 MN x 128 K (= 4 scale bytes along K). */
/* Tile order: expert, then MN tile, then K tile.  Inside a tile row r and */
/* scale column c sit at byte (r % 32) * 16 + (r / 32) * 4 + c (reading:  */
/* the layout the Blackwell block-scaled MMA consumes).  Pad bytes are 0. */
/* ====================================================================== */

int64_t orc_pack_scales_bytes(int E, int MN, int KS) {
  int64_t MT = (MN + 127) / 128, KT = (KS + 3) / 4;
  return (int64_t)E * MT * KT * 512;
}

static int64_t blocked_offset(int e, int row, int col, int MN, int KS) {
  int64_t MT = (MN + 127) / 128, KT = (KS + 3) / 4;
  int mt = row / 128, r = row % 128, kt = col / 4, c = col % 4;
  return (((int64_t)e * MT + mt) * KT + kt) * 512 + (r % 32) * 16 + (r / 32) * 4 + c;
}

void orc_pack_scales_blocked(const uint8_t* in, uint8_t* out, int E, int MN, int KS) {
  memset(out, 0, (size_t)orc_pack_scales_bytes(E, MN, KS));
  for (int e = 0; e < E; ++e)
    for (int row = 0; row < MN; ++row)
      for (int col = 0; col < KS; ++col)
        out[blocked_offset(e, row, col, MN, KS)] = in[((int64_t)e * MN + row) * KS + col];
}

void orc_unpack_scales_blocked(const uint8_t* in, uint8_t* out, int E, int MN, int KS) {
  for (int e = 0; e < E; ++e)
    for (int row = 0; row < MN; ++row)
      for (int col = 0; col < KS; ++col)
        out[((int64_t)e * MN + row) * KS + col] = in[blocked_offset(e, row, col, MN, KS)];
}

/* ====================================================================== */
/* expert FFN                                                             */
/* ====================================================================== */

static double silu(double g) { return g / (1.0 + exp(-g)); }

static void set_threads(int nthreads) {
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#else
  (void)nthreads;
#endif
}

int orc_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* Both FFN routines can also hand back out before its final rounding
 * (out_f64).  Reading: out is bf16 ([PFM] Shapes), and the last rounding is a
 * decision that the GPU takes from an fp32 sum and the oracle from a double
 * sum; the two can land one bf16 ulp apart, which for |out| >= 2.56 rms
 * already exceeds a tolerance of 2e-2 rms.  Parity is therefore measured
 * against the unrounded value.                                             */

/* bf16 path ([PFM] intro and Shapes; [RFC] Background steps 2-5), one token
 * at a time, straight from the definition:
 *   for each route j of token t, e = topk_ids[t, j]:
 *     H = w1[e] x[t]                      (N values; gate = H[0:I], up = H[I:N])
 *     a_i = bf16( silu(H_i) * H_{I+i} )   (activations are bf16 on this path)
 *     Y = w2[e] a                         (K values)
 *     acc += topk_weights[t, j] * Y
 *   out[t] = bf16(acc)                                                      */
void orc_fused_moe_bf16(const uint16_t* x, const uint16_t* w1, const uint16_t* w2,
                        const int32_t* topk_ids, const float* topk_weights,
                        int T, int K, int N, int E, int top_k,
                        const int32_t* tokens, int n_tokens, uint16_t* out, double* out_f64,
                        int nthreads) {
  const int I = N / 2;
  const int count = tokens ? n_tokens : T;
  set_threads(nthreads);
#pragma omp parallel
  {
    double* H = (double*)malloc(sizeof(double) * (size_t)N);
    double* a = (double*)malloc(sizeof(double) * (size_t)I);
    double* acc = (double*)malloc(sizeof(double) * (size_t)K);
#pragma omp for schedule(dynamic, 1)
    for (int idx = 0; idx < count; ++idx) {
      const int t = tokens ? tokens[idx] : idx;
      for (int h = 0; h < K; ++h) acc[h] = 0.0;
      for (int j = 0; j < top_k; ++j) {
        const int e = topk_ids[(int64_t)t * top_k + j];
        if (e < 0 || e >= E) continue;
        const uint16_t* W1 = w1 + (int64_t)e * N * K;
        const uint16_t* W2 = w2 + (int64_t)e * K * I;
        for (int n = 0; n < N; ++n) {
          double s = 0.0;
          for (int k = 0; k < K; ++k)
            s += orc_bf16_to_double(W1[(int64_t)n * K + k]) * orc_bf16_to_double(x[(int64_t)t * K + k]);
          H[n] = s;
        }
        for (int i = 0; i < I; ++i)
          a[i] = orc_bf16_to_double(orc_double_to_bf16(silu(H[i]) * H[I + i]));
        const double wgt = (double)topk_weights[(int64_t)t * top_k + j];
        for (int h = 0; h < K; ++h) {
          double s = 0.0;
          for (int i = 0; i < I; ++i) s += orc_bf16_to_double(W2[(int64_t)h * I + i]) * a[i];
          acc[h] += wgt * s;
        }
      }
      for (int h = 0; h < K; ++h) out[(int64_t)t * K + h] = orc_double_to_bf16(acc[h]);
      if (out_f64)
        for (int h = 0; h < K; ++h) out_f64[(int64_t)t * K + h] = acc[h];
    }
    free(H); free(a); free(acc);
  }
}

/* mxfp8 path ([PFM] intro: e4m3 values with e8m0 block scales on both
 * operands, intermediate requantised to mxfp8 before the down projection;
 * Scale layout (mxfp8): block size 32 along K).  Operands are dequantised
 * exactly (code value * 2^(scale-127)).  The SwiGLU value is rounded to
 * fp32 (the precision the kernel holds it in), then requantised per row in
 * blocks of 32 along the intermediate dimension with the OCP MX rule, and the
 * down projection uses the dequantised requantised values.                 */
/* Weight element idx (row-major inside one expert's matrix) decoded to its
 * code value: e4m3 (one byte per value) or e2m1 (two values per byte, the
 * even-indexed value in the low nibble -- reading: the usual packing order,
 * which the pages do not state). */
/* Decoded values of every code, filled from the decoders above (a lookup
 * of the same exact values, so that the sums below do not call ldexp per
 * element; results are bit for bit those of calling the decoders). */
typedef struct {
  double e4m3[256], e8m0[256], e2m1[16];
} decode_tables;

static void fill_decode_tables(decode_tables* d) {
  for (int c = 0; c < 256; ++c) {
    d->e4m3[c] = orc_e4m3_to_double((uint8_t)c);
    d->e8m0[c] = orc_e8m0_to_double((uint8_t)c);
  }
  for (int c = 0; c < 16; ++c) d->e2m1[c] = orc_e2m1_to_double((uint8_t)c);
}

static double weight_code(const decode_tables* d, const uint8_t* W, int64_t idx, int fp4) {
  if (!fp4) return d->e4m3[W[idx]];
  const uint8_t b = W[idx >> 1];
  return d->e2m1[(idx & 1) ? (b >> 4) : (b & 0xF)];
}

/* One routed row's SwiGLU intermediate before the requant: H = w1[e] x
 * (dequantised operands, double sums), af_i = fp32( silu(H_i) * H_{I+i} ).
 * xd holds x[t] dequantised; H is scratch of N doubles. */
static void mx_route_intermediate(const decode_tables* d, const double* xd, const uint8_t* W1, const uint8_t* S1,
                                  int K, int N, int fp4, double* H, float* af) {
  const int I = N / 2, KS = K / 32;
  for (int n = 0; n < N; ++n) {
    double s = 0.0;
    for (int k = 0; k < K; ++k)
      s += weight_code(d, W1, (int64_t)n * K + k, fp4) * d->e8m0[S1[(int64_t)n * KS + k / 32]] * xd[k];
    H[n] = s;
  }
  for (int i = 0; i < I; ++i) af[i] = (float)(silu(H[i]) * H[I + i]);
}

/* x[t] dequantised exactly: e4m3 value times its e8m0 block scale (per 32 along K). */
static void dequant_x(const decode_tables* d, const uint8_t* x, const uint8_t* x_scales, int t, int K, double* xd) {
  const int KS = K / 32;
  for (int k = 0; k < K; ++k) xd[k] = d->e4m3[x[(int64_t)t * K + k]] * d->e8m0[x_scales[(int64_t)t * KS + k / 32]];
}

static void fused_moe_mx(const uint8_t* x, const uint8_t* x_scales,
                         const uint8_t* w1, const uint8_t* w1_scales,
                         const uint8_t* w2, const uint8_t* w2_scales,
                         const int32_t* topk_ids, const float* topk_weights,
                         int T, int K, int N, int E, int top_k,
                         const int32_t* tokens, int n_tokens, uint16_t* out, double* out_f64,
                         int nthreads, int fp4) {
  const int I = N / 2;
  const int KS = K / 32, IS = I / 32;
  const int count = tokens ? n_tokens : T;
  decode_tables dt;
  fill_decode_tables(&dt);
  const decode_tables* d = &dt;
  set_threads(nthreads);
#pragma omp parallel
  {
    double* xd = (double*)malloc(sizeof(double) * (size_t)K);
    double* H = (double*)malloc(sizeof(double) * (size_t)N);
    float* af = (float*)malloc(sizeof(float) * (size_t)I);
    uint8_t* aq = (uint8_t*)malloc((size_t)I);
    uint8_t* as = (uint8_t*)malloc((size_t)IS);
    double* a = (double*)malloc(sizeof(double) * (size_t)I);
    double* acc = (double*)malloc(sizeof(double) * (size_t)K);
#pragma omp for schedule(dynamic, 1)
    for (int idx = 0; idx < count; ++idx) {
      const int t = tokens ? tokens[idx] : idx;
      dequant_x(d, x, x_scales, t, K, xd);
      for (int h = 0; h < K; ++h) acc[h] = 0.0;
      for (int j = 0; j < top_k; ++j) {
        const int e = topk_ids[(int64_t)t * top_k + j];
        if (e < 0 || e >= E) continue;
        const uint8_t* W1 = w1 + (int64_t)e * N * K / (fp4 ? 2 : 1);
        const uint8_t* S1 = w1_scales + (int64_t)e * N * KS;
        const uint8_t* W2 = w2 + (int64_t)e * K * I / (fp4 ? 2 : 1);
        const uint8_t* S2 = w2_scales + (int64_t)e * K * IS;
        mx_route_intermediate(d, xd, W1, S1, K, N, fp4, H, af);
        orc_mx_quantize(af, I, aq, as);
        for (int i = 0; i < I; ++i) a[i] = d->e4m3[aq[i]] * d->e8m0[as[i / 32]];
        const double wgt = (double)topk_weights[(int64_t)t * top_k + j];
        for (int h = 0; h < K; ++h) {
          double s = 0.0;
          for (int i = 0; i < I; ++i)
            s += weight_code(d, W2, (int64_t)h * I + i, fp4) * d->e8m0[S2[(int64_t)h * IS + i / 32]] * a[i];
          acc[h] += wgt * s;
        }
      }
      for (int h = 0; h < K; ++h) out[(int64_t)t * K + h] = orc_double_to_bf16(acc[h]);
      if (out_f64)
        for (int h = 0; h < K; ++h) out_f64[(int64_t)t * K + h] = acc[h];
    }
    free(xd); free(H); free(af); free(aq); free(as); free(a); free(acc);
  }
}

/* The fp32 SwiGLU intermediate of the mxfp8 / MXFP4 forward, per routed row,
 * before its requant ([PFM] intro: the intermediate is requantised to mxfp8
 * on chip; the requant itself is orc_mx_quantize).  act receives n_tokens x
 * top_k rows of N/2 floats (token order of `tokens`, or all T tokens when it
 * is NULL; routes in top-k order); the row of a route to an expert outside
 * [0, E) is zero.  The same routine the forward above runs. */
void orc_mx_intermediate(const uint8_t* x, const uint8_t* x_scales, const uint8_t* w1, const uint8_t* w1_scales,
                         const int32_t* topk_ids, int T, int K, int N, int E, int top_k,
                         const int32_t* tokens, int n_tokens, float* act, int nthreads, int fp4) {
  const int I = N / 2, KS = K / 32;
  const int count = tokens ? n_tokens : T;
  decode_tables dt;
  fill_decode_tables(&dt);
  const decode_tables* d = &dt;
  set_threads(nthreads);
#pragma omp parallel
  {
    double* xd = (double*)malloc(sizeof(double) * (size_t)K);
    double* H = (double*)malloc(sizeof(double) * (size_t)N);
#pragma omp for schedule(dynamic, 1)
    for (int idx = 0; idx < count; ++idx) {
      const int t = tokens ? tokens[idx] : idx;
      dequant_x(d, x, x_scales, t, K, xd);
      for (int j = 0; j < top_k; ++j) {
        float* row = act + ((int64_t)idx * top_k + j) * I;
        const int e = topk_ids[(int64_t)t * top_k + j];
        if (e < 0 || e >= E) {
          for (int i = 0; i < I; ++i) row[i] = 0.0f;
          continue;
        }
        mx_route_intermediate(d, xd, w1 + (int64_t)e * N * K / (fp4 ? 2 : 1), w1_scales + (int64_t)e * N * KS, K,
                              N, fp4, H, row);
      }
    }
    free(xd); free(H);
  }
}

void orc_fused_moe_mxfp8(const uint8_t* x, const uint8_t* x_scales,
                         const uint8_t* w1, const uint8_t* w1_scales,
                         const uint8_t* w2, const uint8_t* w2_scales,
                         const int32_t* topk_ids, const float* topk_weights,
                         int T, int K, int N, int E, int top_k,
                         const int32_t* tokens, int n_tokens, uint16_t* out, double* out_f64,
                         int nthreads) {
  fused_moe_mx(x, x_scales, w1, w1_scales, w2, w2_scales, topk_ids, topk_weights, T, K, N, E, top_k, tokens,
               n_tokens, out, out_f64, nthreads, 0);
}

/* MXFP4 weights (e2m1 values, e8m0 scale per 32 along the contraction
 * dimension) with mxfp8 activations: the same forward as the mxfp8 path,
 * the weights decoded from packed e2m1 codes.  DeepGEMM #411 "SM90 FP8 x
 * MXFP4 MegaMoE" runs this activation/weight pairing; the OCP MX v1.0 FP4
 * element format defines the codes. */
void orc_fused_moe_mxfp4(const uint8_t* x, const uint8_t* x_scales,
                         const uint8_t* w1, const uint8_t* w1_scales,
                         const uint8_t* w2, const uint8_t* w2_scales,
                         const int32_t* topk_ids, const float* topk_weights,
                         int T, int K, int N, int E, int top_k,
                         const int32_t* tokens, int n_tokens, uint16_t* out, double* out_f64,
                         int nthreads) {
  fused_moe_mx(x, x_scales, w1, w1_scales, w2, w2_scales, topk_ids, topk_weights, T, K, N, E, top_k, tokens,
               n_tokens, out, out_f64, nthreads, 1);
}
