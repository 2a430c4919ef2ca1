// moe_align: the routing planner.
//
// "[RFC] Fused W8A8 MoE megakernel on H20", Design: count the routed tokens
// of every expert (histogram), take prefix sums of the counts, and build the
// row-to-token mapping; the histogram and the prefix sum are dependencies
// across the whole input, which is why the planner is its own kernel.
// "Prime Flash MoE: Fused MoE Kernels for Blackwell", API / Shapes:
// sorted_token_ids holds flattened token*top_k+route ids grouped by expert and
// padded to block_m with -1; expert_ids names the expert of each block;
// num_tokens_post_padded is the padded total.
//
// The planner runs as one thread-block cluster of C CTAs (C = 1 for small
// inputs, 8 otherwise) of 32 warps; the CTAs exchange their per-expert counts
// through distributed shared memory, so neither global scratch nor a
// grid-wide synchronisation is needed.  CTA c owns the contiguous id range
// [c*chunk, (c+1)*chunk) and, inside it, warp w a contiguous sub-range:
//   0. the CTA's ids are staged in shared memory as uint16 with independent
//      loads (when they fit; otherwise they are re-read from global memory);
//   1. every warp counts its sub-range into a private histogram row
//      hist[w][:] (lanes with the same expert are grouped with
//      __match_any_sync; the group leader adds the group size -- no atomics);
//      per expert the rows are then scanned over w, giving each warp its start
//      inside the CTA's share, and the CTA total cnt[e] is published;
//   2. after a cluster barrier every CTA reads all CTAs' cnt[e] through
//      distributed shared memory: before[e] (the counts of lower CTAs) and
//      the expert totals, whose padded exclusive scan gives the segment
//      offsets off[e] (computed identically in every CTA);
//   3. every warp walks its range again and writes each id to
//      off[e] + before[e] + start[w][e] + (rank among earlier lanes with the
//      same expert), so ids ascend inside a segment -- the result is unique
//      and bit-exact.
// Slots that receive no id (segment padding and the capacity tail) get -1,
// and expert_ids is filled block by block; these writes are spread over the
// cluster's CTAs.
#include <algorithm>
#include <atomic>

#include "internal.h"
#include "ptx.cuh"

namespace moe {

constexpr int kAlignThreads = 1024;
constexpr int kAlignWarps = kAlignThreads / 32;
constexpr int kAlignSmemLimit = 232448;
constexpr int kAlignClusterMax = 8;
constexpr int kAlignClusterMinIds = 4096;  // inputs smaller than this use one CTA
constexpr uint16_t kNoExpert = 0xFFFFu;

// Shared memory (int32): hist[kAlignWarps][E], cnt[E], before[E], off[E + 1],
// warp_tot[kAlignWarps]; then -- when they fit -- the CTA's ids as uint16.
__host__ __device__ inline size_t align_smem_base(int E) {
  return sizeof(int32_t) * (static_cast<size_t>(kAlignWarps) * E + 3 * static_cast<size_t>(E) + 1 + kAlignWarps);
}

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_nctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Reads a 32-bit word of CTA `rank`'s shared memory at the address that
// `local` has in this CTA.
__device__ __forceinline__ int32_t ld_dsmem(const int32_t* local, uint32_t rank) {
  uint32_t remote;
  int32_t v;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(static_cast<uint32_t>(__cvta_generic_to_shared(local))), "r"(rank));
  asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(remote) : "memory");
  return v;
}

// ------------------------------------------------------------------ router
// Softmax -> top-k -> renormalisation ahead of the planner.  "Prime Flash
// MoE", Usage: topk_ids come from the caller's gate; "[RFC] Fused W8A8 MoE
// megakernel on H20", Results so far: the paths share normalized routing
// weights.  Reading: score z = logit + bias (fp32), experts ranked by
// descending z with equal scores by ascending index, the first top_k kept,
// weights = exp(z_j - z_0) / sum over the kept of exp(z_i - z_0) (the full
// softmax denominator cancels in the renormalisation).  Scores must be finite.
constexpr int kRouteMaxK = 8;
// Batches of at most this many tokens (one per warp of the planner CTA) are
// routed inside the planner; larger ones in their own all-SM kernel, which
// measured faster from two tokens per warp on.
constexpr int kRouteFusedMaxTokens = 32;

// Shared experts follow the routed ones: with n_shared > 0 every token also
// routes, with weight 1, to experts E .. E+n_shared-1 (reading: a shared
// expert processes every token and its output is added to the routed sum;
// the fused megakernels of the sgl DeepGEMM PR and DeepGEMM #411 run shared
// experts beside the routed ones).  Their GEMMs then run as ordinary,
// densely filled units of the same fused kernels.
//
// One warp routes token t.  Lane l scans experts l, l+32, ... keeping its
// best kRouteMaxK in a sorted register list (compare-and-swap down a fixed
// list, so equal scores keep the earlier, lower index ahead); k rounds of a
// warp-wide arg-max (ties to the lower index) then merge the 32 lists.  Lane
// j < k ends with the j-th expert and its weight, lane k + s with shared
// expert E + s; row t of the outputs holds k + n_shared entries, also written
// to the staged id array (when ids16 is given) at t*(k + n_shared) + j - id0.
__device__ __forceinline__ void route_token(const float* __restrict__ logits, const float* __restrict__ bias,
                                            int t, int E, int k, int n_shared, int lane,
                                            int32_t* __restrict__ topk_ids, float* __restrict__ topk_w,
                                            uint16_t* ids16, int id0) {
  float lv[kRouteMaxK];
  int le[kRouteMaxK];
#pragma unroll
  for (int p = 0; p < kRouteMaxK; ++p) {
    lv[p] = -INFINITY;
    le[p] = 0x7fffffff;
  }
  const float* row = logits + static_cast<int64_t>(t) * E;
  for (int e = lane; e < E; e += 32) {
    float cv = __ldg(row + e) + (bias ? __ldg(bias + e) : 0.0f);
    int ce = e;
#pragma unroll
    for (int p = 0; p < kRouteMaxK; ++p) {
      if (cv > lv[p]) {
        const float tv = lv[p];
        const int te = le[p];
        lv[p] = cv;
        le[p] = ce;
        cv = tv;
        ce = te;
      }
    }
  }
  float my_v = 0.f;
  int my_e = -1;
  for (int j = 0; j < k; ++j) {
    float bv = lv[0];
    int be = le[0];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
      const int oe = __shfl_xor_sync(0xffffffffu, be, off);
      if (ov > bv || (ov == bv && oe < be)) {
        bv = ov;
        be = oe;
      }
    }
    if (lane == j) {
      my_v = bv;
      my_e = be;
    }
    if (le[0] == be) {  // the owning lane drops its head
#pragma unroll
      for (int p = 0; p + 1 < kRouteMaxK; ++p) {
        lv[p] = lv[p + 1];
        le[p] = le[p + 1];
      }
      lv[kRouteMaxK - 1] = -INFINITY;
      le[kRouteMaxK - 1] = 0x7fffffff;
    }
  }
  const float z0 = __shfl_sync(0xffffffffu, my_v, 0);
  float w = lane < k ? expf(my_v - z0) : 0.f;
  float sum = w;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
  const int kk = k + n_shared;
  if (lane < kk) {
    const int64_t r = static_cast<int64_t>(t) * kk + lane;
    const int e = lane < k ? my_e : E + (lane - k);
    topk_ids[r] = e;
    topk_w[r] = lane < k ? w / sum : 1.0f;
    if (ids16) ids16[r - id0] = static_cast<uint16_t>(e);
  }
}

// Router for larger batches: one warp per token over the whole GPU; the
// planner that follows is chained by programmatic dependent launch.
__global__ void __launch_bounds__(256) moe_route_kernel(const float* __restrict__ logits,
                                                        const float* __restrict__ bias, int T, int E, int k,
                                                        int n_shared, int32_t* __restrict__ topk_ids,
                                                        float* __restrict__ topk_w) {
  pdl_launch_dependents();
  const int lane = threadIdx.x & 31;
  const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, nw = (gridDim.x * blockDim.x) >> 5;
  for (int t = gw; t < T; t += nw)
    route_token(logits, bias, t, E, k, n_shared, lane, topk_ids, topk_w, nullptr, 0);
}

// Planner.  With route_T > 0 (one CTA, at most one token per warp) the CTA first
// routes route_T tokens itself from logits/bias, writing topk_ids/topk_w and
// staging the ids directly; otherwise it reads topk_ids.
__global__ void __launch_bounds__(kAlignThreads, 1)
    moe_align_kernel(const int32_t* __restrict__ topk_ids, int R, int E, int block_m,
                     int32_t* __restrict__ sorted_ids, int32_t* __restrict__ expert_ids,
                     int32_t* __restrict__ ntpp_out, int64_t capacity, int staged,
                     const float* __restrict__ logits, const float* __restrict__ bias, int route_T, int route_k,
                     int route_shared, int32_t* route_ids, float* __restrict__ route_w) {
  extern __shared__ int32_t sm[];
  int32_t* hist = sm;                         // [kAlignWarps][E], later start offsets
  int32_t* cnt = hist + kAlignWarps * E;      // [E] this CTA's count per expert
  int32_t* before = cnt + E;                  // [E] counts of lower-ranked CTAs
  int32_t* off = before + E;                  // [E + 1] segment offsets
  int32_t* warp_tot = off + E + 1;            // [kAlignWarps]
  uint16_t* ids16 = reinterpret_cast<uint16_t*>(warp_tot + kAlignWarps);  // [chunk] when staged

  pdl_launch_dependents();  // the fused phases may start their prologue now
  pdl_wait();               // a preceding router kernel's ids (no-op after an ordinary launch)
  const uint32_t crank = cluster_ctarank(), csize = cluster_nctarank();
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int cchunk = (R + static_cast<int>(csize) - 1) / static_cast<int>(csize);
  const int clo = min(R, static_cast<int>(crank) * cchunk), chi = min(R, clo + cchunk);

  for (int i = tid; i < kAlignWarps * E; i += kAlignThreads) hist[i] = 0;
  // 0. stage this CTA's ids (independent loads, so their latencies overlap);
  //    ids outside [0, E) route nowhere.  A routing CTA (one CTA, clo = 0)
  //    produces them instead.
  if (route_T > 0) {
    for (int t = warp; t < route_T; t += kAlignWarps)
      route_token(logits, bias, t, E - route_shared, route_k, route_shared, lane, route_ids, route_w, ids16, 0);
  } else if (staged) {
#pragma unroll 4
    for (int i = clo + tid; i < chi; i += kAlignThreads) {
      const int e = __ldg(topk_ids + i);
      ids16[i - clo] = (e >= 0 && e < E) ? static_cast<uint16_t>(e) : kNoExpert;
    }
  }
  __syncthreads();
  auto expert_of = [&](int i) -> int {
    if (staged) {
      const uint16_t v = ids16[i - clo];
      return v == kNoExpert ? -1 : static_cast<int>(v);
    }
    const int e = __ldg(topk_ids + i);
    return (e >= 0 && e < E) ? e : -1;
  };

  const int wchunk = (chi - clo + kAlignWarps - 1) / kAlignWarps;
  const int lo = min(chi, clo + warp * wchunk), hi = min(chi, lo + wchunk);
  const unsigned lt_mask = (1u << lane) - 1u;

  // 1. warp-private histograms, then the scan over warps and the CTA count
  for (int base = lo; base < hi; base += 32) {
    const int i = base + lane;
    const int e = (i < hi) ? expert_of(i) : -1;
    const unsigned same = __match_any_sync(0xffffffffu, e);
    if (e >= 0 && (same & lt_mask) == 0) hist[warp * E + e] += __popc(same);
    __syncwarp();
  }
  __syncthreads();
  for (int e = tid; e < E; e += kAlignThreads) {
    int run = 0;
    for (int w = 0; w < kAlignWarps; ++w) {
      const int c = hist[w * E + e];
      hist[w * E + e] = run;
      run += c;
    }
    cnt[e] = run;
  }
  cluster_sync();  // every CTA's cnt[] is published

  // 2a. counts of lower CTAs and expert totals, read from every CTA; the
  //     totals are parked in off[] until the scan replaces them
  for (int e = tid; e < E; e += kAlignThreads) {
    int lower = 0, total = 0;
    for (uint32_t c = 0; c < csize; ++c) {
      const int v = (c == crank) ? cnt[e] : ld_dsmem(cnt + e, c);
      if (c < crank) lower += v;
      total += v;
    }
    before[e] = lower;
    off[e] = total;  // total for now; replaced by the offset below
  }
  cluster_sync();  // no CTA reads another's shared memory after this point

  // 2b. exclusive scan of the padded totals over experts (block-wide, in
  // rounds of kAlignThreads experts); identical in every CTA
  int carry = 0;
  for (int e0 = 0; e0 < E; e0 += kAlignThreads) {
    const int e = e0 + tid;
    const int padded = (e < E) ? (off[e] + block_m - 1) / block_m * block_m : 0;
    int v = padded;
    for (int d = 1; d < 32; d <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, v, d);
      if (lane >= d) v += y;
    }
    if (lane == 31) warp_tot[warp] = v;
    __syncthreads();
    if (warp == 0) {
      int t = warp_tot[lane];
      for (int d = 1; d < 32; d <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, t, d);
        if (lane >= d) t += y;
      }
      warp_tot[lane] = t;  // inclusive over warps
    }
    __syncthreads();
    const int incl = v + (warp > 0 ? warp_tot[warp - 1] : 0) + carry;
    const int total = (e < E) ? off[e] : 0;
    __syncthreads();
    if (e < E) {
      off[e] = incl - padded;
      cnt[e] = total;  // cnt now holds the expert total
    }
    const int round_total = warp_tot[kAlignWarps - 1];
    __syncthreads();
    carry += round_total;
  }
  if (tid == 0) {
    off[E] = carry;
    if (crank == 0) *ntpp_out = carry;
  }
  __syncthreads();
  const int ntpp = off[E];

  // 3. stable scatter
  for (int base = lo; base < hi; base += 32) {
    const int i = base + lane;
    const int e = (i < hi) ? expert_of(i) : -1;
    const unsigned same = __match_any_sync(0xffffffffu, e);
    if (e >= 0) {
      const int rank = __popc(same & lt_mask);
      sorted_ids[off[e] + before[e] + hist[warp * E + e] + rank] = i;
    }
    __syncwarp();
    if (e >= 0 && (same & lt_mask) == 0) hist[warp * E + e] += __popc(same);
    __syncwarp();
  }

  // padding inside each segment (expert e by CTA e % csize), then the
  // capacity tail (strided over the cluster)
  for (int e = static_cast<int>(crank) * kAlignWarps + warp; e < E; e += static_cast<int>(csize) * kAlignWarps) {
    const int s = off[e] + cnt[e], t = off[e + 1];
    for (int p = s + lane; p < t; p += 32) sorted_ids[p] = -1;
    for (int b = off[e] / block_m + lane; b < t / block_m; b += 32) expert_ids[b] = e;
  }
  const int64_t stride = static_cast<int64_t>(csize) * kAlignThreads;
  const int64_t first = static_cast<int64_t>(crank) * kAlignThreads + tid;
  for (int64_t p = ntpp + first; p < capacity; p += stride) sorted_ids[p] = -1;
  const int64_t nblk_cap = (capacity + block_m - 1) / block_m;
  for (int64_t b = ntpp / block_m + first; b < nblk_cap; b += stride) expert_ids[b] = -1;
}

}  // namespace moe

using namespace moe;

extern "C" int64_t moe_align_capacity(int T, int top_k, int E, int block_m) {
  if (T < 0 || top_k < 1 || E < 1 || block_m < 1) return -1;
  return static_cast<int64_t>(T) * top_k + static_cast<int64_t>(E) * (block_m - 1);
}

// Launches the planner: one CTA, or one cluster of kAlignClusterMax CTAs for
// large inputs.  route_T > 0 makes the (single) CTA route the tokens itself;
// after_router chains the launch to a preceding router kernel.
static int launch_align(const int32_t* topk_ids, int T, int top_k, int E, int block_m, int32_t* sorted_token_ids,
                        int32_t* expert_ids, int32_t* num_tokens_post_padded, int64_t capacity, moe_stream_t stream,
                        const float* logits, const float* bias, int route_T, int route_k, int route_shared,
                        int32_t* route_ids, float* route_w, bool after_router) {
  const int R = T * top_k;
  const int csize = R >= kAlignClusterMinIds ? kAlignClusterMax : 1;
  const int cchunk = (R + csize - 1) / csize;
  const size_t base = align_smem_base(E);
  const size_t staged_bytes = base + sizeof(uint16_t) * static_cast<size_t>(cchunk);
  const int staged = staged_bytes <= static_cast<size_t>(kAlignSmemLimit) ? 1 : 0;
  const size_t smem = staged ? staged_bytes : base;
  if (route_T > 0 && (csize != 1 || !staged))
    return fail(MOE_ERR_UNSUPPORTED, "moe_route_align: the in-planner router needs one CTA with staged ids");
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cuda_fail("moe_align: cudaGetDevice");
  static std::atomic<bool> attr_set[kMaxDevices];  // per device; setting it twice is harmless
  if (dev < kMaxDevices && !attr_set[dev].load(std::memory_order_relaxed)) {
    if (cudaFuncSetAttribute(moe_align_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kAlignSmemLimit) !=
        cudaSuccess)
      return cuda_fail("moe_align: cudaFuncSetAttribute");
    attr_set[dev].store(true, std::memory_order_relaxed);
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(csize, 1, 1);
  cfg.blockDim = dim3(kAlignThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = reinterpret_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = csize;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = after_router ? 2 : 1;
  const cudaError_t lerr = cudaLaunchKernelEx(&cfg, moe_align_kernel, topk_ids, R, E, block_m, sorted_token_ids,
                                              expert_ids, num_tokens_post_padded, capacity, staged, logits, bias,
                                              route_T, route_k, route_shared, route_ids, route_w);
  if (lerr != cudaSuccess) return cuda_fail("moe_align: launch", lerr);
  const cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return cuda_fail("moe_align: launch", err);
  return MOE_OK;
}

extern "C" int moe_align(const int32_t* topk_ids, int T, int top_k, int E, int block_m,
                         int32_t* sorted_token_ids, int32_t* expert_ids, int32_t* num_tokens_post_padded,
                         int64_t capacity, moe_stream_t stream) {
  if (T < 0 || top_k < 1) return fail(MOE_ERR_INVALID_ARG, "moe_align: need T >= 0 and top_k >= 1");
  if (E < 1 || E > kMaxExperts)
    return fail(MOE_ERR_UNSUPPORTED, "moe_align: E must be in [1, %d], got %d", kMaxExperts, E);
  if (!valid_block_m(block_m))
    return fail(MOE_ERR_UNSUPPORTED, "moe_align: block_m must be 16, 32, 64 or 128, got %d", block_m);
  const int64_t need = moe_align_capacity(T, top_k, E, block_m);
  if (need >= (int64_t(1) << 31))
    return fail(MOE_ERR_UNSUPPORTED, "moe_align: T*top_k + E*(block_m-1) must be < 2^31");
  if (capacity < need)
    return fail(MOE_ERR_INVALID_ARG, "moe_align: capacity %lld < required %lld", (long long)capacity,
                (long long)need);
  if (capacity >= (int64_t(1) << 31)) return fail(MOE_ERR_UNSUPPORTED, "moe_align: capacity must be < 2^31");
  if ((T > 0 && !topk_ids) || !sorted_token_ids || !expert_ids || !num_tokens_post_padded)
    return fail(MOE_ERR_INVALID_ARG, "moe_align: null pointer");

  return launch_align(topk_ids, T, top_k, E, block_m, sorted_token_ids, expert_ids, num_tokens_post_padded, capacity,
                      stream, nullptr, nullptr, 0, 0, 0, nullptr, nullptr, false);
}

extern "C" int moe_route_align(const float* logits, const float* bias, int T, int E, int top_k, int n_shared,
                               int block_m, int32_t* topk_ids, float* topk_weights, int32_t* sorted_token_ids,
                               int32_t* expert_ids, int32_t* num_tokens_post_padded, int64_t capacity,
                               moe_stream_t stream) {
  if (T < 0) return fail(MOE_ERR_INVALID_ARG, "moe_route_align: need T >= 0");
  if (E < 1 || E > kMaxExperts)
    return fail(MOE_ERR_UNSUPPORTED, "moe_route_align: E must be in [1, %d], got %d", kMaxExperts, E);
  if (top_k < 1 || top_k > kRouteMaxK || top_k > E)
    return fail(MOE_ERR_UNSUPPORTED, "moe_route_align: top_k must be in [1, min(%d, E)], got %d", kRouteMaxK, top_k);
  if (n_shared < 0 || top_k + n_shared > 32 || E + n_shared > kMaxExperts)
    return fail(MOE_ERR_UNSUPPORTED,
                "moe_route_align: need n_shared >= 0, top_k + n_shared <= 32 and E + n_shared <= %d", kMaxExperts);
  const int kk = top_k + n_shared, Et = E + n_shared;  // the planner sees the shared routes as ordinary ones
  if (!valid_block_m(block_m))
    return fail(MOE_ERR_UNSUPPORTED, "moe_route_align: block_m must be 16, 32, 64 or 128, got %d", block_m);
  const int64_t need = moe_align_capacity(T, kk, Et, block_m);
  if (need >= (int64_t(1) << 31))
    return fail(MOE_ERR_UNSUPPORTED, "moe_route_align: T*(top_k+n_shared) + (E+n_shared)*(block_m-1) must be < 2^31");
  if (capacity < need)
    return fail(MOE_ERR_INVALID_ARG, "moe_route_align: capacity %lld < required %lld", (long long)capacity,
                (long long)need);
  if (capacity >= (int64_t(1) << 31))
    return fail(MOE_ERR_UNSUPPORTED, "moe_route_align: capacity must be < 2^31");
  if ((T > 0 && (!logits || !topk_ids || !topk_weights)) || !sorted_token_ids || !expert_ids ||
      !num_tokens_post_padded)
    return fail(MOE_ERR_INVALID_ARG, "moe_route_align: null pointer");
  const bool fused = T <= kRouteFusedMaxTokens;
  if (!fused && T > 0) {
    const int blocks = std::min<int64_t>((static_cast<int64_t>(T) + 7) / 8, static_cast<int64_t>(sm_count()) * 8);
    moe_route_kernel<<<blocks, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(logits, bias, T, E, top_k, n_shared,
                                                                               topk_ids, topk_weights);
    const cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return cuda_fail("moe_route_align: router launch", err);
  }
  return launch_align(topk_ids, T, kk, Et, block_m, sorted_token_ids, expert_ids, num_tokens_post_padded, capacity,
                      stream, logits, bias, fused ? T : 0, top_k, n_shared, topk_ids, topk_weights, !fused && T > 0);
}
