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
// One CTA of 32 warps does the three phases in shared memory, so no grid-wide
// synchronisation is needed.  When they fit (uint16 each, next to the
// histograms), the R expert ids are first staged in shared memory with
// independent loads, so the two passes below read shared memory instead of
// waiting on one global load per 32 ids:
//   1. warp w owns the contiguous id range [w*chunk, (w+1)*chunk) and counts
//      it into its private histogram row hist[w][:] (lanes with the same
//      expert are grouped with __match_any_sync; the group leader adds the
//      group size -- no atomics);
//   2. per expert, the rows are scanned over w (giving each warp its start
//      inside the expert's segment) and the padded counts are scanned over e
//      (the segment offsets);
//   3. every warp walks its range again and writes each id to
//      off[e] + start[w][e] + (rank among earlier lanes with the same expert),
//      so ids ascend inside a segment -- the result is unique and bit-exact.
// Slots that receive no id (segment padding and the capacity tail) get -1,
// and expert_ids is filled block by block.
#include "internal.h"

namespace moe {

constexpr int kAlignThreads = 1024;
constexpr int kAlignWarps = kAlignThreads / 32;
constexpr int kAlignSmemLimit = 232448;
constexpr uint16_t kNoExpert = 0xFFFFu;

// Shared memory: hist[kAlignWarps][E], count[E], off[E + 1], warp_tot[kAlignWarps]
// (int32), then -- when they fit -- the R expert ids as uint16.
__host__ __device__ inline size_t align_smem_base(int E) {
  return sizeof(int32_t) * (static_cast<size_t>(kAlignWarps) * E + E + E + 1 + kAlignWarps);
}

__global__ void __launch_bounds__(kAlignThreads, 1)
    moe_align_kernel(const int32_t* __restrict__ topk_ids, int R, int E, int block_m,
                     int32_t* __restrict__ sorted_ids, int32_t* __restrict__ expert_ids,
                     int32_t* __restrict__ ntpp_out, int64_t capacity, int staged) {
  extern __shared__ int32_t sm[];
  int32_t* hist = sm;                         // [kAlignWarps][E], later start offsets
  int32_t* count = hist + kAlignWarps * E;    // [E]
  int32_t* off = count + E;                   // [E + 1]
  int32_t* warp_tot = off + E + 1;            // [kAlignWarps]
  uint16_t* ids16 = reinterpret_cast<uint16_t*>(warp_tot + kAlignWarps);  // [R] when staged

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int i = tid; i < kAlignWarps * E; i += kAlignThreads) hist[i] = 0;
  // 0. stage the ids (independent loads, so their latencies overlap); ids
  //    outside [0, E) route nowhere
  if (staged) {
#pragma unroll 4
    for (int i = tid; i < R; i += kAlignThreads) {
      const int e = __ldg(topk_ids + i);
      ids16[i] = (e >= 0 && e < E) ? static_cast<uint16_t>(e) : kNoExpert;
    }
  }
  __syncthreads();
  auto expert_of = [&](int i) -> int {
    if (staged) {
      const uint16_t v = ids16[i];
      return v == kNoExpert ? -1 : static_cast<int>(v);
    }
    const int e = __ldg(topk_ids + i);
    return (e >= 0 && e < E) ? e : -1;
  };

  const int chunk = (R + kAlignWarps - 1) / kAlignWarps;
  const int lo = min(R, warp * chunk), hi = min(R, lo + chunk);
  const unsigned lt_mask = (1u << lane) - 1u;

  // 1. warp-private histograms
  for (int base = lo; base < hi; base += 32) {
    const int i = base + lane;
    const int e = (i < hi) ? expert_of(i) : -1;
    const unsigned same = __match_any_sync(0xffffffffu, e);
    if (e >= 0 && (same & lt_mask) == 0) hist[warp * E + e] += __popc(same);
    __syncwarp();
  }
  __syncthreads();

  // 2a. per expert: exclusive scan over warps, total count
  for (int e = tid; e < E; e += kAlignThreads) {
    int run = 0;
    for (int w = 0; w < kAlignWarps; ++w) {
      const int c = hist[w * E + e];
      hist[w * E + e] = run;
      run += c;
    }
    count[e] = run;
  }
  __syncthreads();

  // 2b. exclusive scan of the padded counts over experts (block-wide, in
  // rounds of kAlignThreads experts)
  int carry = 0;
  for (int e0 = 0; e0 < E; e0 += kAlignThreads) {
    const int e = e0 + tid;
    const int padded = (e < E) ? (count[e] + block_m - 1) / block_m * block_m : 0;
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
    if (e < E) off[e] = incl - padded;
    const int round_total = warp_tot[kAlignWarps - 1];
    __syncthreads();
    carry += round_total;
  }
  if (tid == 0) {
    off[E] = carry;
    *ntpp_out = carry;
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
      sorted_ids[off[e] + hist[warp * E + e] + rank] = i;
    }
    __syncwarp();
    if (e >= 0 && (same & lt_mask) == 0) hist[warp * E + e] += __popc(same);
    __syncwarp();
  }

  // padding inside each segment, then the capacity tail
  for (int e = warp; e < E; e += kAlignWarps) {
    const int s = off[e] + count[e], t = off[e + 1];
    for (int p = s + lane; p < t; p += 32) sorted_ids[p] = -1;
    for (int b = off[e] / block_m + lane; b < t / block_m; b += 32) expert_ids[b] = e;
  }
  for (int64_t p = ntpp + tid; p < capacity; p += kAlignThreads) sorted_ids[p] = -1;
  const int64_t nblk_cap = (capacity + block_m - 1) / block_m;
  for (int64_t b = ntpp / block_m + tid; b < nblk_cap; b += kAlignThreads) expert_ids[b] = -1;
}

}  // namespace moe

using namespace moe;

extern "C" int64_t moe_align_capacity(int T, int top_k, int E, int block_m) {
  if (T < 0 || top_k < 1 || E < 1 || block_m < 1) return -1;
  return static_cast<int64_t>(T) * top_k + static_cast<int64_t>(E) * (block_m - 1);
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

  const int R = T * top_k;
  const size_t base = align_smem_base(E);
  const size_t staged_bytes = base + sizeof(uint16_t) * static_cast<size_t>(R);
  const int staged = staged_bytes <= static_cast<size_t>(kAlignSmemLimit) ? 1 : 0;
  const size_t smem = staged ? staged_bytes : base;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cuda_fail("moe_align: cudaGetDevice");
  static bool attr_set[kMaxDevices] = {};
  if (dev < kMaxDevices && !attr_set[dev]) {
    if (cudaFuncSetAttribute(moe_align_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kAlignSmemLimit) !=
        cudaSuccess)
      return cuda_fail("moe_align: cudaFuncSetAttribute");
    attr_set[dev] = true;
  }
  moe_align_kernel<<<1, kAlignThreads, smem, reinterpret_cast<cudaStream_t>(stream)>>>(
      topk_ids, R, E, block_m, sorted_token_ids, expert_ids, num_tokens_post_padded, capacity, staged);
  const cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return cuda_fail("moe_align: launch", err);
  return MOE_OK;
}
