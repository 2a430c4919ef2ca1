// Host-side helpers shared by the library's translation units.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "moe_ffn.h"

namespace moe {

constexpr int kMaxExperts = 1024;  // planner keeps 32 x E histogram words in shared memory
constexpr int kMaxDevices = 64;

inline bool valid_block_m(int bm) { return bm == 16 || bm == 32 || bm == 64 || bm == 128; }

// Records a formatted message for moe_last_error() and returns `code`.
int fail(int code, const char* fmt, ...);
// Records "<what>: <cuda error string>" and returns MOE_ERR_CUDA.
int cuda_fail(const char* what, cudaError_t err = cudaGetLastError());

// Number of SMs of the current device (cached per device).
int sm_count();

}  // namespace moe
