// pack_scales_blocked: weight scales into the blocked tile layout.
//
// "Prime Flash MoE: Fused MoE Kernels for Blackwell", Scale layout (mxfp8):
// weight scales (one e8m0 byte per 32 along K) are reordered into a sequence
// of 512-byte tiles, each covering 128 MN x 128 K, and the packing is done
// once at load time.  Tile (e, mt, kt) starts at ((e*MT + mt)*KT + kt)*512;
// row r / scale column c of the tile sits at (r%32)*16 + (r/32)*4 + c, the
// 128 x 4 arrangement the block-scaled tensor-core MMA reads, so that one
// 512-byte tile can be copied into tensor memory as-is.
//
// One thread writes one 32-bit word of the output (the four scale columns of
// one row): output writes are fully coalesced, input reads are 4 contiguous
// bytes per row (gathered rows).
#include "internal.h"

namespace moe {

__global__ void pack_scales_kernel(const uint8_t* __restrict__ in, uint32_t* __restrict__ out, int MN,
                                   int KS, int MT, int KT, int64_t n_words) {
  for (int64_t w = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; w < n_words;
       w += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t tile = w >> 7;             // 128 words per 512-byte tile
    const int within = static_cast<int>(w & 127);
    const int r = (within >> 2) + 32 * (within & 3);   // word (r%32)*4 + r/32
    const int kt = static_cast<int>(tile % KT);
    const int64_t em = tile / KT;
    const int mt = static_cast<int>(em % MT);
    const int64_t e = em / MT;
    const int row = mt * 128 + r;
    uint32_t v = 0;
    if (row < MN) {
      const uint8_t* src = in + (e * MN + row) * KS;
      for (int c = 0; c < 4; ++c) {
        const int col = kt * 4 + c;
        if (col < KS) v |= static_cast<uint32_t>(src[col]) << (8 * c);
      }
    }
    out[w] = v;
  }
}

}  // namespace moe

using namespace moe;

extern "C" int64_t pack_scales_blocked_bytes(int E, int MN, int KS) {
  if (E < 0 || MN < 0 || KS < 0) return -1;
  const int64_t MT = (MN + 127) / 128, KT = (KS + 3) / 4;
  return static_cast<int64_t>(E) * MT * KT * 512;
}

extern "C" int pack_scales_blocked(const uint8_t* in, uint8_t* out, int E, int MN, int KS,
                                   moe_stream_t stream) {
  if (E < 0 || MN < 0 || KS < 0) return fail(MOE_ERR_INVALID_ARG, "pack_scales_blocked: negative size");
  const int64_t bytes = pack_scales_blocked_bytes(E, MN, KS);
  if (bytes == 0) return MOE_OK;
  if (!in || !out) return fail(MOE_ERR_INVALID_ARG, "pack_scales_blocked: null pointer");
  if (reinterpret_cast<uintptr_t>(out) % 4 != 0)
    return fail(MOE_ERR_ALIGNMENT, "pack_scales_blocked: out must be 4-byte aligned");
  const int MT = (MN + 127) / 128, KT = (KS + 3) / 4;
  const int64_t n_words = bytes / 4;
  const int threads = 256;
  const int64_t want = (n_words + threads - 1) / threads;
  const int blocks = static_cast<int>(want < 148 * 32 ? want : 148 * 32);
  pack_scales_kernel<<<blocks, threads, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      in, reinterpret_cast<uint32_t*>(out), MN, KS, MT, KT, n_words);
  const cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return cuda_fail("pack_scales_blocked: launch", err);
  return MOE_OK;
}
