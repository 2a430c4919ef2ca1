// The small-batch form of the bf16 forward (host side).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace moe {

// Largest routed-row count (T * top_k) for which fused_moe_bf16 takes the
// small-batch form by itself; moe_tuning.small_batch forces it on or off.
constexpr int kSbAutoRoutes = 128;
// Largest T the small-batch form is offered for (it is meant for decode sizes).
constexpr int kSbMaxT = 8192;

struct SbArgs {
  const void* x;   // (T, K) bf16
  const void* w1;  // (E, N, K) bf16
  const void* w2;  // (E, K, N/2) bf16
  const int32_t* sorted_ids;
  const int32_t* expert_ids;
  const int32_t* ntpp;
  const float* topk_w;
  int T, K, N, E, top_k, bm, max_blocks;
  void* act;        // planner rows x N/2 bf16 (workspace)
  float* yw;        // T*top_k rows x K fp32: each route's weighted down-projection row (workspace)
  int32_t* flags;   // T*top_k route flags (workspace): set for the routes that reach an expert
  bool pf_all;      // all expert weights fit the L2 prefetch budget
};

// Whether the shapes allow the small-batch form at all (K and N/2 multiples
// of 256, T <= kSbMaxT).
bool small_batch_shapes_ok(int T, int K, int N, int top_k);

// Launches the two kernels on `stream`, after which the caller launches the
// route-order combine over `yw` and `flags` (one partial row per route).
// `phase_events` (4 cudaEvent_t or NULL): [0] and [1] are recorded before and
// after the gate/up kernel, [2] after the down kernel; the caller records [3]
// after the combine.
int run_small_batch(const SbArgs& a, cudaStream_t stream, void* const* phase_events);

}  // namespace moe
