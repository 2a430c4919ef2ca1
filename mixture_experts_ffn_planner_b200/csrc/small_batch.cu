// Small-batch form of the bf16 fused MoE forward.
//
// "[RFC] Fused W8A8 MoE megakernel on H20", Background: at decode sizes a
// MoE layer streams the weights of its few touched experts and does almost
// no arithmetic per weight byte, so the time is the weight stream plus the
// latency of every dependent step.  With a handful of routed rows per
// expert the tcgen05 phases spend most of a call in that latency chain
// (planner -> gate/up -> split-K reduction -> down -> combine), and their
// 128-row MMA tile is mostly padding, so small batches take this form
// instead: two streaming kernels after the planner, then the route-order
// combine of the tensor path.
//
//   moe_sb_up_kernel:   one CTA per (planner block, 8 intermediate columns):
//     the 8 gate rows and 8 up rows of w1[e] are the 16 rows of an
//     m16n8k16 MMA, up to 16 of the block's token rows its columns; each of
//     the 8 warps streams 1/8 of K straight from memory into MMA fragments
//     (16-byte loads, each weight byte read once), the partial tiles are
//     added in warp order, and bf16(silu(gate) * up) goes to the
//     intermediate -- the same values, in the same layout, as the gate/up
//     phase of the tensor path.  It also clears the route flags.
//   moe_sb_down_kernel: one item per (planner block, 16 output features):
//     those 16 rows of w2[e] against the block's intermediate rows -- a CTA
//     per item with the N/2 reduction split over its 8 warps the same way
//     when N/2 >= 512, else a warp per item; each routed row's 16 weighted
//     fp32 sums go to its partial row and its route flag is set.
//   The combine kernel then sums each token's partial rows in route order
//   (fp32, one bf16 rounding), exactly as after the tensor-core phases.
//
// The MMA is the warp-level mma.sync (bf16 in, fp32 accumulate): at these
// sizes the work is a weight stream with an 8..16-column GEMM attached, for
// which a warp-wide 16 x 8 tile wastes nothing and needs no tensor memory.
// Both operands are loaded with the same permutation of K inside every 32
// values (thread (g, q) holds elements 8q .. 8q+7), which leaves every dot
// product unchanged.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "internal.h"
#include "ptx.cuh"
#include "small_batch.h"

namespace moe {
namespace {

constexpr int kSbThreads = 256;
constexpr int kSbWarps = kSbThreads / 32;
constexpr int kSbMaxBm = 128;

struct SbParams {
  const __nv_bfloat16* x;
  const __nv_bfloat16* w1;
  const __nv_bfloat16* w2;
  const int32_t* sorted_ids;
  const int32_t* expert_ids;
  const int32_t* ntpp;
  const float* topk_w;
  __nv_bfloat16* act;
  float* yw;
  int32_t* flags;
  int T, K, N, I, E, top_k, bm, max_blocks, R;
  int pf_all;
};

__device__ __forceinline__ int sb_num_blocks(const SbParams& p) {
  const int n = __ldg(p.ntpp) / p.bm;
  return n < 0 ? 0 : (n > p.max_blocks ? p.max_blocks : n);
}

// Weight rows are read once: keep them out of L1.
__device__ __forceinline__ uint4 ld_stream(const void* ptr) {
  uint4 v;
  asm("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
      : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
      : "l"(ptr));
  return v;
}

// d += a(16x16, row) . b(16x8, col), bf16 inputs, fp32 accumulate.
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// The block's routed rows, compacted into this warp's tables in row order:
// token, planner row and route id of the i-th routed row.  Returns their
// number (0 for a block whose expert id is out of range).  Warp-collective.
__device__ __forceinline__ int sb_block_rows(const SbParams& p, int b, int e, int* tok, int* row, int* route,
                                             int lane) {
  int ids[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int r = 32 * q + lane;
    ids[q] = r < p.bm ? __ldg(p.sorted_ids + static_cast<int64_t>(b) * p.bm + r) : -1;
  }
  __syncwarp();  // the previous block's tables are no longer read
  if (e < 0 || e >= p.E) return 0;
  int n = 0;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const bool v = ids[q] >= 0 && ids[q] < p.R;
    const uint32_t m = __ballot_sync(0xffffffffu, v);
    if (v) {
      const int k = n + __popc(m & ((1u << lane) - 1u));
      tok[k] = ids[q] / p.top_k;
      row[k] = b * p.bm + 32 * q + lane;
      route[k] = ids[q];
    }
    n += __popc(m);
  }
  __syncwarp();
  return n;
}

// D(16 x 8 NT) = A . B^T over L values: A rows ra (rows g) and rb (rows g + 8)
// of 16 weight rows, B rows bn[0..NT) (row g of each 8-column tile).  Thread
// (g, q) loads 16 bytes of each of its rows per 32-value block (elements
// 8q .. 8q+7) and feeds them to two MMAs; the loads of U blocks are issued
// before their MMAs (fewer with two tiles, whose rows take the registers).
template <int NT, bool kStream, int U = NT == 1 ? 4 : 2>
__device__ __forceinline__ void sb_mma_rows(const __nv_bfloat16* ra, const __nv_bfloat16* rb,
                                            const __nv_bfloat16* const (&bn)[NT], int L, int q, float (&d)[NT][4]) {
#pragma unroll
  for (int t = 0; t < NT; ++t)
#pragma unroll
    for (int i = 0; i < 4; ++i) d[t][i] = 0.f;
  const int nblk = L / 32;
  for (int k0 = 0; k0 < nblk; k0 += U) {
    uint4 av[U], bv[U], xv[U][NT];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      if (k0 + u < nblk) {
        const int off = 32 * (k0 + u) + 8 * q;
        av[u] = kStream ? ld_stream(ra + off) : __ldg(reinterpret_cast<const uint4*>(ra + off));
        bv[u] = kStream ? ld_stream(rb + off) : __ldg(reinterpret_cast<const uint4*>(rb + off));
#pragma unroll
        for (int t = 0; t < NT; ++t) xv[u][t] = __ldg(reinterpret_cast<const uint4*>(bn[t] + off));
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      if (k0 + u < nblk) {
#pragma unroll
        for (int t = 0; t < NT; ++t) {
          mma_bf16_16816(d[t], av[u].x, bv[u].x, av[u].y, bv[u].y, xv[u][t].x, xv[u][t].y);
          mma_bf16_16816(d[t], av[u].z, bv[u].z, av[u].w, bv[u].w, xv[u][t].z, xv[u][t].w);
        }
      }
    }
  }
}

// Gate/up for 8 intermediate columns c0 .. c0+7 and up to 8 * NT routed rows
// (the block's rows tok/row, ng of them): every warp of the CTA takes K/8 of
// the reduction, the partial tiles meet in shared memory and warp 0 adds them
// in warp order, so thread (g, q) of warp 0 holds gate and up of column c0 + g
// for rows 2q, 2q + 1 of every tile.
template <int NT>
__device__ __forceinline__ void sb_up_tile(const SbParams& p, int e, int c0, const int* tok, const int* row, int ng,
                                           int warp, int lane, float (*red)[2][32][4]) {
  const int g = lane >> 2, q = lane & 3;
  const int kw = p.K / kSbWarps;  // a multiple of 32
  const __nv_bfloat16* ra = p.w1 + (static_cast<int64_t>(e) * p.N + c0 + g) * p.K + warp * kw;  // gate row
  const __nv_bfloat16* rb = ra + static_cast<int64_t>(p.I) * p.K;                               // up row
  const __nv_bfloat16* bn[NT];
#pragma unroll
  for (int t = 0; t < NT; ++t) {
    const int i = 8 * t + g;
    bn[t] = p.x + static_cast<int64_t>(tok[i < ng ? i : ng - 1]) * p.K + warp * kw;
  }
  float d[NT][4];
  sb_mma_rows<NT, true>(ra, rb, bn, kw, q, d);
#pragma unroll
  for (int t = 0; t < NT; ++t)
    *reinterpret_cast<float4*>(red[warp][t][lane]) = make_float4(d[t][0], d[t][1], d[t][2], d[t][3]);
  __syncthreads();
  if (warp == 0) {
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      float s4[4] = {0.f, 0.f, 0.f, 0.f};
      for (int w = 0; w < kSbWarps; ++w) {
        const float4 v = *reinterpret_cast<const float4*>(red[w][t][lane]);
        s4[0] += v.x;
        s4[1] += v.y;
        s4[2] += v.z;
        s4[3] += v.w;
      }
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int i = 8 * t + 2 * q + h;
        if (i < ng) p.act[static_cast<int64_t>(row[i]) * p.I + c0 + g] = __float2bfloat16_rn(silu_f32(s4[h]) * s4[2 + h]);
      }
    }
  }
  __syncthreads();  // red is reused by the next tile
}

__global__ void __launch_bounds__(kSbThreads, 2) moe_sb_up_kernel(const __grid_constant__ SbParams p) {
  __shared__ int s_tok[kSbMaxBm], s_row[kSbMaxBm], s_route[kSbMaxBm];
  __shared__ __align__(16) float s_red[kSbWarps][2][32][4];
  __shared__ int s_nr, s_e;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (p.pf_all && threadIdx.x == 0) {
    // every expert's weights fit the prefetch budget: this CTA's share goes
    // to L2 now, while the planner runs
    const uint8_t* src[2] = {reinterpret_cast<const uint8_t*>(p.w1), reinterpret_cast<const uint8_t*>(p.w2)};
    const int64_t bytes[2] = {static_cast<int64_t>(p.E) * p.N * p.K * 2, static_cast<int64_t>(p.E) * p.K * p.I * 2};
    for (int a = 0; a < 2; ++a) {
      const int64_t n16 = bytes[a] / 16;
      const int64_t lo = n16 * blockIdx.x / gridDim.x * 16, hi = n16 * (blockIdx.x + 1) / gridDim.x * 16;
      for (int64_t o = lo; o < hi; o += 32768)
        prefetch_l2(src[a] + o, static_cast<uint32_t>(hi - o < 32768 ? hi - o : 32768));
    }
  }
  pdl_wait();  // the planner's outputs are read below
  pdl_launch_dependents();
  {
    // the route flags the down kernel sets and the combine reads
    const int64_t gtid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    for (int64_t i = gtid; i < p.R; i += static_cast<int64_t>(gridDim.x) * blockDim.x) p.flags[i] = 0;
  }
  // contiguous ranges of (block, 8-column group) items per CTA: the block's
  // rows are read once per range, neighbouring CTAs stream neighbouring rows
  const int n_cg = p.I / 8;
  const int64_t n_items = static_cast<int64_t>(sb_num_blocks(p)) * n_cg;
  const int64_t per = (n_items + gridDim.x - 1) / gridDim.x;
  const int64_t it0 = per * blockIdx.x, it1 = it0 + per < n_items ? it0 + per : n_items;
  int cur_b = -1;
  for (int64_t it = it0; it < it1; ++it) {
    const int b = static_cast<int>(it / n_cg);
    const int c0 = 8 * static_cast<int>(it - static_cast<int64_t>(b) * n_cg);
    if (b != cur_b) {  // the same in every warp
      cur_b = b;
      __syncthreads();  // every warp has read the previous block's row count and rows
      if (warp == 0) {
        const int e = __ldg(p.expert_ids + b);
        const int n = sb_block_rows(p, b, e, s_tok, s_row, s_route, lane);
        if (lane == 0) {
          s_nr = n;
          s_e = e;
        }
      }
      __syncthreads();
    }
    const int nr = s_nr, e = s_e;
    for (int r0 = 0; r0 < nr; r0 += 16) {
      const int ng = nr - r0 < 16 ? nr - r0 : 16;
      if (ng <= 8)
        sb_up_tile<1>(p, e, c0, s_tok + r0, s_row + r0, ng, warp, lane, s_red);
      else
        sb_up_tile<2>(p, e, c0, s_tok + r0, s_row + r0, ng, warp, lane, s_red);
    }
  }
}

// Down projection of 16 output features k0 .. k0+15 for up to 8 * NT routed
// rows of the block: every warp of the CTA takes N/16 of the N/2-long
// reduction, the partial tiles are added in warp order by warp 0, whose
// thread (g, q) ends with features k0 + g and k0 + g + 8 of rows 2q, 2q + 1
// of every tile, weighted into the rows' partial rows.
template <int NT>
__device__ __forceinline__ void sb_down_tile(const SbParams& p, int e, int k0, const int* row, const int* route,
                                             int ng, int warp, int lane, float (*red)[2][32][4]) {
  const int g = lane >> 2, q = lane & 3;
  const int iw = p.I / kSbWarps;  // a multiple of 32
  const __nv_bfloat16* ra = p.w2 + (static_cast<int64_t>(e) * p.K + k0 + g) * p.I + warp * iw;
  const __nv_bfloat16* rb = ra + static_cast<int64_t>(8) * p.I;
  const __nv_bfloat16* bn[NT];
#pragma unroll
  for (int t = 0; t < NT; ++t) {
    const int i = 8 * t + g;
    bn[t] = p.act + static_cast<int64_t>(row[i < ng ? i : ng - 1]) * p.I + warp * iw;
  }
  float d[NT][4];
  sb_mma_rows<NT, true>(ra, rb, bn, iw, q, d);
#pragma unroll
  for (int t = 0; t < NT; ++t)
    *reinterpret_cast<float4*>(red[warp][t][lane]) = make_float4(d[t][0], d[t][1], d[t][2], d[t][3]);
  __syncthreads();
  if (warp == 0) {
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      float s4[4] = {0.f, 0.f, 0.f, 0.f};
      for (int w = 0; w < kSbWarps; ++w) {
        const float4 v = *reinterpret_cast<const float4*>(red[w][t][lane]);
        s4[0] += v.x;
        s4[1] += v.y;
        s4[2] += v.z;
        s4[3] += v.w;
      }
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int i = 8 * t + 2 * q + h;
        if (i < ng) {
          const int rt = route[i];
          const float w = __ldg(p.topk_w + rt);
          float* y = p.yw + static_cast<int64_t>(rt) * p.K + k0 + g;
          y[0] = w * s4[h];
          y[8] = w * s4[2 + h];
        }
      }
    }
  }
  __syncthreads();  // red is reused by the next tile
}

__device__ __forceinline__ void sb_down_per_cta(const SbParams& p) {
  __shared__ int s_tok[kSbMaxBm], s_row[kSbMaxBm], s_route[kSbMaxBm];
  __shared__ __align__(16) float s_red[kSbWarps][2][32][4];
  __shared__ int s_nr, s_e;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // contiguous ranges of (block, 16-feature group) items per CTA
  const int n_fg = p.K / 16;
  const int64_t n_items = static_cast<int64_t>(sb_num_blocks(p)) * n_fg;
  const int64_t per = (n_items + gridDim.x - 1) / gridDim.x;
  const int64_t it0 = per * blockIdx.x, it1 = it0 + per < n_items ? it0 + per : n_items;
  int cur_b = -1;
  for (int64_t it = it0; it < it1; ++it) {
    const int b = static_cast<int>(it / n_fg);
    const int k0 = 16 * static_cast<int>(it - static_cast<int64_t>(b) * n_fg);
    if (b != cur_b) {  // the same in every warp
      cur_b = b;
      __syncthreads();  // every warp has read the previous block's row count and rows
      if (warp == 0) {
        const int e = __ldg(p.expert_ids + b);
        const int n = sb_block_rows(p, b, e, s_tok, s_row, s_route, lane);
        if (lane == 0) {
          s_nr = n;
          s_e = e;
        }
      }
      __syncthreads();
    }
    const int nr = s_nr, e = s_e;
    for (int r0 = 0; r0 < nr; r0 += 16) {
      const int ng = nr - r0 < 16 ? nr - r0 : 16;
      if (ng <= 8)
        sb_down_tile<1>(p, e, k0, s_row + r0, s_route + r0, ng, warp, lane, s_red);
      else
        sb_down_tile<2>(p, e, k0, s_row + r0, s_route + r0, ng, warp, lane, s_red);
    }
    if (k0 == 0 && warp == 0)
      for (int i = lane; i < nr; i += 32) p.flags[s_route[i]] = 1;
  }
}

// Warp-per-item schedule of the down projection (below).
// Down projection of 16 output features k0 .. k0+15 for up to 8 * NT routed
// rows of the block: thread (g, q) ends with features k0 + g and k0 + g + 8
// of rows 2q, 2q + 1 of every tile, weighted into the rows' partial rows.
template <int NT>
__device__ __forceinline__ void sb_down_tile_warp(const SbParams& p, int e, int k0, const int* row, const int* route,
                                             int ng, int lane) {
  const int g = lane >> 2, q = lane & 3;
  const __nv_bfloat16* ra = p.w2 + (static_cast<int64_t>(e) * p.K + k0 + g) * p.I;
  const __nv_bfloat16* rb = ra + static_cast<int64_t>(8) * p.I;
  const __nv_bfloat16* bn[NT];
#pragma unroll
  for (int t = 0; t < NT; ++t) {
    const int i = 8 * t + g;
    bn[t] = p.act + static_cast<int64_t>(row[i < ng ? i : ng - 1]) * p.I;
  }
  float d[NT][4];
  sb_mma_rows<NT, true>(ra, rb, bn, p.I, q, d);
#pragma unroll
  for (int t = 0; t < NT; ++t)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int i = 8 * t + 2 * q + h;
      if (i < ng) {
        const int rt = route[i];
        const float w = __ldg(p.topk_w + rt);
        float* y = p.yw + static_cast<int64_t>(rt) * p.K + k0 + g;
        y[0] = w * d[t][h];
        y[8] = w * d[t][2 + h];
      }
    }
}

__device__ __forceinline__ void sb_down_per_warp(const SbParams& p) {
  __shared__ int s_tok[kSbWarps][kSbMaxBm], s_row[kSbWarps][kSbMaxBm], s_route[kSbWarps][kSbMaxBm];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t gtid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t nw = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5, gw = gtid >> 5;
  const int n_fg = p.K / 16;  // groups of 16 output features
  const int64_t n_items = static_cast<int64_t>(sb_num_blocks(p)) * n_fg;
  const int64_t per = (n_items + nw - 1) / nw;
  const int64_t it0 = gw * per, it1 = it0 + per < n_items ? it0 + per : n_items;
  int cur_b = -1, nr = 0, e = 0;
  for (int64_t it = it0; it < it1; ++it) {
    const int b = static_cast<int>(it / n_fg);
    const int k0 = 16 * static_cast<int>(it - static_cast<int64_t>(b) * n_fg);
    if (b != cur_b) {
      cur_b = b;
      e = __ldg(p.expert_ids + b);
      nr = sb_block_rows(p, b, e, s_tok[warp], s_row[warp], s_route[warp], lane);
    }
    for (int r0 = 0; r0 < nr; r0 += 16) {
      const int ng = nr - r0 < 16 ? nr - r0 : 16;
      if (ng <= 8)
        sb_down_tile_warp<1>(p, e, k0, s_row[warp] + r0, s_route[warp] + r0, ng, lane);
      else
        sb_down_tile_warp<2>(p, e, k0, s_row[warp] + r0, s_route[warp] + r0, ng, lane);
    }
    if (k0 == 0)
      for (int i = lane; i < nr; i += 32) p.flags[s_route[warp][i]] = 1;
  }
}

// One kernel, two schedules: a CTA per item (the reduction split over its
// warps) when N/2 is long enough to give every warp several 32-value blocks,
// else a warp per item (N/2 = 256: one block per warp would leave each item
// a chain of barriers around a single load).
template <bool kPerCta>
__global__ void __launch_bounds__(kSbThreads, 2) moe_sb_down_kernel(const __grid_constant__ SbParams p) {
  pdl_wait();  // the intermediate and the cleared flags are read below
  pdl_launch_dependents();
  if (kPerCta)
    sb_down_per_cta(p);
  else
    sb_down_per_warp(p);
}

}  // namespace

bool small_batch_shapes_ok(int T, int K, int N, int top_k) {
  (void)top_k;
  // K and N/2 split into 8 warp shares of whole 32-value blocks
  return T > 0 && T <= kSbMaxT && K % 256 == 0 && N % 2 == 0 && (N / 2) % 256 == 0;
}

int run_small_batch(const SbArgs& a, cudaStream_t stream, void* const* ev) {
  SbParams p{};
  p.x = static_cast<const __nv_bfloat16*>(a.x);
  p.w1 = static_cast<const __nv_bfloat16*>(a.w1);
  p.w2 = static_cast<const __nv_bfloat16*>(a.w2);
  p.sorted_ids = a.sorted_ids;
  p.expert_ids = a.expert_ids;
  p.ntpp = a.ntpp;
  p.topk_w = a.topk_w;
  p.act = static_cast<__nv_bfloat16*>(a.act);
  p.yw = a.yw;
  p.flags = a.flags;
  p.T = a.T; p.K = a.K; p.N = a.N; p.I = a.N / 2; p.E = a.E; p.top_k = a.top_k; p.bm = a.bm;
  p.max_blocks = a.max_blocks;
  p.R = a.T * a.top_k;
  p.pf_all = a.pf_all ? 1 : 0;

  const int nsm = sm_count();
  if (nsm <= 0) return cuda_fail("cudaDeviceGetAttribute(SM count)");
  auto mark = [&](int i) -> int {
    if (ev && cudaEventRecord(static_cast<cudaEvent_t>(ev[i]), stream) != cudaSuccess)
      return cuda_fail("fused_moe_bf16: cudaEventRecord");
    return MOE_OK;
  };
  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t c = {};
  c.gridDim = dim3(2 * nsm, 1, 1);
  c.blockDim = dim3(kSbThreads, 1, 1);
  c.stream = stream;
  c.attrs = pdl;
  c.numAttrs = 1;
  int rc;
  if ((rc = mark(0)) != MOE_OK) return rc;
  cudaError_t err = cudaLaunchKernelEx(&c, moe_sb_up_kernel, p);
  if (err != cudaSuccess) return cuda_fail("fused_moe_bf16: small-batch gate/up launch", err);
  if ((rc = mark(1)) != MOE_OK) return rc;
  err = p.I >= 512 ? cudaLaunchKernelEx(&c, moe_sb_down_kernel<true>, p)
                   : cudaLaunchKernelEx(&c, moe_sb_down_kernel<false>, p);
  if (err != cudaSuccess) return cuda_fail("fused_moe_bf16: small-batch down launch", err);
  return mark(2);
}

}  // namespace moe
