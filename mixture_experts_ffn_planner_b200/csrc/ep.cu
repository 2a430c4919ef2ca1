// Expert-parallel dispatch and combine around the local fused forward.
//
// DeepGEMM #411 "SM90 FP8 x MXFP4 MegaMoE", Summary, and "[SM90]
// Ring-buffered FP8 MegaMoE with a lag-ordered L1/L2 schedule" (sgl DeepGEMM
// PR #88): with the experts sharded over the ranks of a group (EP), every
// rank sends each routed row to the rank that owns the route's expert
// (dispatch), the owners run their local experts, and the results travel back
// to be reduced per token over its top-k routes (combine).  The exchanges
// themselves are collectives of the caller's process group; these kernels do
// the device-side work on either side of them:
//   plan     a stable counting sort of the routes by owner rank: `order` lists
//            the route ids t*top_k + j that reach an expert, grouped by owner
//            rank, ascending inside a group; send_counts[r] the group sizes;
//   pack     the send buffers in that order: the token row (and its e8m0
//            scales on the mxfp8 path), the expert index local to the owner
//            and the routing weight;
//   combine  out[t] = bf16( sum over j in route order of y[slot of (t, j)] ),
//            with y the returned rows (one per entry of `order`), summed in
//            fp32 in the same order whatever the rank count.
#include <algorithm>
#include <cuda_bf16.h>

#include "internal.h"

namespace moe {

constexpr int kPlanThreads = 1024;
constexpr int kPlanWarps = kPlanThreads / 32;
constexpr int kEpMaxWorld = 64;

// One CTA.  Warp w walks a contiguous share of the routes twice: first it
// counts its routes per owner rank into hist[w][rank] (lanes with the same
// owner grouped by __match_any_sync, the leader adding the group size), then,
// after the per-rank scan over warps and the scan over ranks, it writes every
// route at offset[rank] + start[w][rank] + (its rank among earlier lanes with
// that owner) -- a stable order, unique and deterministic.
__global__ void __launch_bounds__(kPlanThreads, 1)
    ep_plan_kernel(const int32_t* __restrict__ topk_ids, int R, int E, int world, int32_t* __restrict__ order,
                   int32_t* __restrict__ send_counts) {
  __shared__ int32_t hist[kPlanWarps][kEpMaxWorld];
  __shared__ int32_t base[kEpMaxWorld + 1];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int per = E / world;
  const unsigned lt = (1u << lane) - 1u;
  for (int i = threadIdx.x; i < kPlanWarps * kEpMaxWorld; i += kPlanThreads) (&hist[0][0])[i] = 0;
  __syncthreads();
  const int chunk = (R + kPlanWarps - 1) / kPlanWarps;
  const int lo = min(R, warp * chunk), hi = min(R, lo + chunk);
  auto owner = [&](int i) -> int {
    if (i >= hi) return -1;
    const int e = __ldg(topk_ids + i);
    return (e >= 0 && e < E) ? e / per : -1;
  };
  for (int b = lo; b < hi; b += 32) {
    const int d = owner(b + lane);
    const unsigned same = __match_any_sync(0xffffffffu, d);
    if (d >= 0 && (same & lt) == 0) hist[warp][d] += __popc(same);
    __syncwarp();
  }
  __syncthreads();
  if (threadIdx.x < world) {  // per rank: exclusive scan over the warps, the rank's total
    const int d = threadIdx.x;
    int run = 0;
    for (int w = 0; w < kPlanWarps; ++w) {
      const int c = hist[w][d];
      hist[w][d] = run;
      run += c;
    }
    send_counts[d] = run;
    base[d] = run;
  }
  __syncthreads();
  if (threadIdx.x == 0) {  // exclusive scan over the ranks (world <= 64)
    int run = 0;
    for (int d = 0; d < world; ++d) {
      const int c = base[d];
      base[d] = run;
      run += c;
    }
    base[world] = run;
  }
  __syncthreads();
  for (int b = lo; b < hi; b += 32) {
    const int d = owner(b + lane);
    const unsigned same = __match_any_sync(0xffffffffu, d);
    if (d >= 0) order[base[d] + hist[warp][d] + __popc(same & lt)] = b + lane;
    __syncwarp();
    if (d >= 0 && (same & lt) == 0) hist[warp][d] += __popc(same);
    __syncwarp();
  }
  // the entries past the routes that reach an expert
  for (int i = base[world] + threadIdx.x; i < R; i += kPlanThreads) order[i] = -1;
}

// One warp per packed row: the token's row (16-byte vectors when the row
// allows, else bytes), its scales, the owner-local expert and the weight.
__global__ void __launch_bounds__(256)
    ep_pack_kernel(const uint8_t* __restrict__ x, int64_t row_bytes, const uint8_t* __restrict__ x_scales,
                   int64_t scale_bytes, const int32_t* __restrict__ topk_ids, const float* __restrict__ topk_w,
                   const int32_t* __restrict__ order, int n, int top_k, int per, uint8_t* __restrict__ rows_out,
                   uint8_t* __restrict__ scales_out, int32_t* __restrict__ local_e, float* __restrict__ w_out) {
  const int lane = threadIdx.x & 31;
  const int64_t nw = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  for (int64_t i = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; i < n; i += nw) {
    const int r = __ldg(order + i);
    if (r < 0) continue;  // past the routes that reach an expert (n too large): nothing to pack
    const int64_t t = r / top_k;
    const uint8_t* src = x + t * row_bytes;
    uint8_t* dst = rows_out + i * row_bytes;
    if ((row_bytes & 15) == 0) {
      for (int64_t c = lane; c < row_bytes / 16; c += 32)
        reinterpret_cast<uint4*>(dst)[c] = __ldg(reinterpret_cast<const uint4*>(src) + c);
    } else {
      for (int64_t c = lane; c < row_bytes; c += 32) dst[c] = __ldg(src + c);
    }
    if (x_scales)
      for (int64_t c = lane; c < scale_bytes; c += 32) scales_out[i * scale_bytes + c] = __ldg(x_scales + t * scale_bytes + c);
    if (lane == 0) {
      const int e = __ldg(topk_ids + r);
      local_e[i] = e - (e / per) * per;
      w_out[i] = __ldg(topk_w + r);
    }
  }
}

__global__ void ep_slot_fill_kernel(int32_t* __restrict__ slot, int64_t R) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < R;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    slot[i] = -1;
}

__global__ void ep_slot_scatter_kernel(const int32_t* __restrict__ order, int n, int32_t* __restrict__ slot) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    if (__ldg(order + i) >= 0) slot[__ldg(order + i)] = static_cast<int32_t>(i);
}

// One thread per 8 consecutive features of a token: its routes' returned rows
// (bf16) are added in route order in fp32, then rounded once to bf16.
__global__ void __launch_bounds__(256)
    ep_combine_kernel(const __nv_bfloat16* __restrict__ y, const int32_t* __restrict__ slot, int T, int top_k, int K,
                      __nv_bfloat16* __restrict__ out) {
  const int kv = K / 8;
  const int64_t total = static_cast<int64_t>(T) * kv;
  for (int64_t v = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; v < total;
       v += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t t = v / kv;
    const int c = static_cast<int>(v - t * kv) * 8;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int j = 0; j < top_k; ++j) {
      const int s = __ldg(slot + t * top_k + j);
      if (s < 0) continue;
      const uint4 u = __ldg(reinterpret_cast<const uint4*>(y + static_cast<int64_t>(s) * K + c));
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        acc[2 * i] += __uint_as_float(w[i] << 16);
        acc[2 * i + 1] += __uint_as_float(w[i] & 0xFFFF0000u);
      }
    }
    __nv_bfloat162 o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) o[i] = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
    *reinterpret_cast<uint4*>(out + t * K + c) = *reinterpret_cast<const uint4*>(o);
  }
}

static int grid_for(int64_t items, int per_block) {
  const int64_t b = (items + per_block - 1) / per_block;
  const int64_t cap = static_cast<int64_t>(std::max(1, sm_count())) * 8;
  return static_cast<int>(std::max<int64_t>(1, std::min(b, cap)));
}

}  // namespace moe

using namespace moe;

extern "C" int moe_ep_dispatch_plan(const int32_t* topk_ids, int T, int top_k, int E, int world, int32_t* order,
                                    int32_t* send_counts, moe_stream_t stream) {
  if (T < 0 || top_k < 1 || E < 1) return fail(MOE_ERR_INVALID_ARG, "moe_ep_dispatch_plan: need T >= 0, top_k >= 1, E >= 1");
  if (world < 1 || world > kEpMaxWorld || E % world)
    return fail(MOE_ERR_UNSUPPORTED, "moe_ep_dispatch_plan: world must be in [1, %d] and divide E (E=%d, world=%d)",
                kEpMaxWorld, E, world);
  if (static_cast<int64_t>(T) * top_k >= (int64_t(1) << 31))
    return fail(MOE_ERR_UNSUPPORTED, "moe_ep_dispatch_plan: T * top_k must be < 2^31");
  if ((T > 0 && (!topk_ids || !order)) || !send_counts) return fail(MOE_ERR_INVALID_ARG, "moe_ep_dispatch_plan: null pointer");
  ep_plan_kernel<<<1, kPlanThreads, 0, reinterpret_cast<cudaStream_t>(stream)>>>(topk_ids, T * top_k, E, world, order,
                                                                                 send_counts);
  const cudaError_t err = cudaGetLastError();
  return err == cudaSuccess ? MOE_OK : cuda_fail("moe_ep_dispatch_plan: launch", err);
}

extern "C" int moe_ep_dispatch_pack(const void* x, int64_t row_bytes, const uint8_t* x_scales, int64_t scale_bytes,
                                    const int32_t* topk_ids, const float* topk_weights, const int32_t* order, int n,
                                    int T, int top_k, int E, int world, void* rows_out, uint8_t* scales_out,
                                    int32_t* local_expert_out, float* weight_out, moe_stream_t stream) {
  if (n < 0 || T < 0 || top_k < 1 || E < 1 || row_bytes < 1 || scale_bytes < 0 ||
      n > static_cast<int64_t>(T) * top_k)
    return fail(MOE_ERR_INVALID_ARG, "moe_ep_dispatch_pack: need 0 <= n <= T*top_k, row_bytes >= 1, E >= 1");
  if (world < 1 || world > kEpMaxWorld || E % world)
    return fail(MOE_ERR_UNSUPPORTED, "moe_ep_dispatch_pack: world must be in [1, %d] and divide E", kEpMaxWorld);
  if (n == 0) return MOE_OK;
  if (!x || !topk_ids || !topk_weights || !order || !rows_out || !local_expert_out || !weight_out ||
      (x_scales && !scales_out))
    return fail(MOE_ERR_INVALID_ARG, "moe_ep_dispatch_pack: null pointer");
  if ((row_bytes % 16 == 0) &&
      ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(rows_out)) & 15))
    return fail(MOE_ERR_ALIGNMENT, "moe_ep_dispatch_pack: x and rows_out must be 16-byte aligned");
  ep_pack_kernel<<<grid_for(static_cast<int64_t>(n) * 32, 256), 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint8_t*>(x), row_bytes, x_scales, scale_bytes, topk_ids, topk_weights, order, n, top_k,
      E / world, static_cast<uint8_t*>(rows_out), scales_out, local_expert_out, weight_out);
  const cudaError_t err = cudaGetLastError();
  return err == cudaSuccess ? MOE_OK : cuda_fail("moe_ep_dispatch_pack: launch", err);
}

extern "C" int moe_ep_combine(const void* y, const int32_t* order, int n, int T, int top_k, int K, int32_t* slot,
                              void* out, moe_stream_t stream) {
  if (n < 0 || T < 0 || top_k < 1 || K < 8 || K % 8 || n > static_cast<int64_t>(T) * top_k)
    return fail(MOE_ERR_INVALID_ARG, "moe_ep_combine: need 0 <= n <= T*top_k and K a positive multiple of 8");
  if (T == 0) return MOE_OK;
  if (!out || !slot || (n > 0 && (!y || !order))) return fail(MOE_ERR_INVALID_ARG, "moe_ep_combine: null pointer");
  if ((reinterpret_cast<uintptr_t>(y) | reinterpret_cast<uintptr_t>(out)) & 15)
    return fail(MOE_ERR_ALIGNMENT, "moe_ep_combine: y and out must be 16-byte aligned");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int64_t R = static_cast<int64_t>(T) * top_k;
  ep_slot_fill_kernel<<<grid_for(R, 256), 256, 0, s>>>(slot, R);
  if (n > 0) ep_slot_scatter_kernel<<<grid_for(n, 256), 256, 0, s>>>(order, n, slot);
  ep_combine_kernel<<<grid_for(static_cast<int64_t>(T) * (K / 8), 256), 256, 0, s>>>(
      static_cast<const __nv_bfloat16*>(y), slot, T, top_k, K, static_cast<__nv_bfloat16*>(out));
  const cudaError_t err = cudaGetLastError();
  return err == cudaSuccess ? MOE_OK : cuda_fail("moe_ep_combine: launch", err);
}
