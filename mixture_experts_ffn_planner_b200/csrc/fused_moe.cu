// Fused MoE expert-FFN forward for sm_100a (bf16 and mxfp8 paths; the mxfp8
// path also takes MXFP4 weights).
//
// What is computed -- "Prime Flash MoE: Fused MoE Kernels for Blackwell",
// intro / API / Shapes, and "[RFC] Fused W8A8 MoE megakernel on H20",
// Background: for every routed row (token t, route j, expert e) the gate/up
// GEMM H = w1[e] x[t], SwiGLU a = silu(H[:N/2]) * H[N/2:] taken straight from
// the accumulator (never stored as the 2H-wide tensor), on the mxfp8 path a
// requantisation of a to e4m3 + e8m0 per 32 on chip, the down GEMM
// Y = w2[e] a, and the top-k weighted reduction out[t] = sum_j w[t,j] Y.
//
// How (sm_100a), token-major tiles:
//   phase 1  persistent kernel, one CTA per SM.  A work unit is (planner block
//            b, intermediate tile j of 128 columns).  The block's routed token
//            rows (gathered by cp.async into the 128-byte-swizzled layout) are
//            the M = 128 operand of tcgen05.mma; the expert's 128 gate rows and
//            128 up rows, streamed by TMA, form one N = 256 operand, so one MMA
//            per 32-byte K slice fills a TMEM accumulator laid out as [token
//            (lane)] x [gate 0..127 | up 0..127].  Each epilogue thread owns one
//            token row: SwiGLU, the 32-wide amax, the e8m0 scale and the e4m3
//            codes all stay in its registers, and the intermediate row segment
//            is written with 16-byte stores into an L2-resident workspace.
//            Warp roles: 0 TMA producer (weight tiles, weight scale tiles),
//            1 MMA issuer, 2-5 token gather (cp.async of the routed rows and,
//            on mxfp8, their scales; completion is tracked by the stage's
//            mbarrier, so the gather warps never wait on their own copies),
//            6-13 epilogue (two warps per TMEM lane quadrant, one per column
//            half).  When the units cannot fill the SMs (decode-sized
//            problems), a unit's K range is split over several CTAs and the
//            fp32 partial accumulators are summed, in split order, by
//   reduce   a small kernel that applies SwiGLU (and the requant) to the sum.
//   phase 2  persistent kernel, unit = (block b, 256 output features).  A =
//            the block's intermediate rows (TMA, one 128-row box for blocks of
//            at least 64 rows), B = 256 rows of w2[e] (TMA, one box),
//            D in TMEM; each epilogue thread scales its row by the routing
//            weight and writes one row segment per route (fp32 on the bf16
//            path; bf16 on the mxfp8 path, whose tolerance leaves room for
//            the extra rounding).
//   combine  out[t] = bf16(sum over the token's routes, in route order), a
//            deterministic HBM-bound pass.
// The weight tiles are streamed once per unit through a multi-stage shared
// memory ring by TMA; the weights are the dominant HBM traffic.  MXFP4
// weights (e2m1, two per byte) are expanded by the copy itself into the
// unpacked shared-memory form the block-scaled MMA reads, so the two GEMM
// kernels differ only in byte counts and the MMA's B format.
#include <algorithm>
#include <atomic>
#include <mutex>

#include "internal.h"
#include "ptx.cuh"
#include "small_batch.h"

namespace moe {

__device__ int g_moe_status = 0;

constexpr int kM = 128;           // MMA M: routed rows of one planner block (rows >= block_m unused)
constexpr int kTI = 128;          // intermediate columns per gate/up unit (gate 128 + up 128 = MMA N 256)
// Split-K of the gate/up phase for small problems: when there are fewer work
// units than half the CTAs, a unit whose block has at most kSplitRows routed
// rows is cut into up to kMaxSplit K-ranges, each on its own CTA; the fp32
// partial accumulators go to the workspace and moe_p1_reduce_kernel sums them
// (in split order) and applies SwiGLU.
constexpr int kSplitRows = 32;
constexpr int kMaxSplit = 8;
constexpr int kMaxSplitItems = 256;  // bounds the partial workspace
constexpr int kTH = 256;          // output features per down unit (MMA N)
constexpr int kRowBytes = 128;    // bytes of one operand row per pipeline stage
constexpr int kSfTileBytes = 512; // one blocked scale tile: 128 rows x 4 scales
constexpr int kSmemLimit = 232448;  // 227 KB of dynamic shared memory per CTA
// L2 prefetch budgets of small calls (the L2 holds 126 MB): all expert
// weights when they fit kPrefetchAllBytes; else the down phase's w2 tiles of
// the planner blocks when they fit kPrefetchW2Bytes.
constexpr int64_t kPrefetchAllBytes = int64_t(40) << 20;
constexpr int64_t kPrefetchW2Bytes = int64_t(48) << 20;

// TMEM column map: accumulators first; on the mxfp8 path (one accumulator)
// the scale factors follow it, one set of 12 columns per pipeline stage (4
// for the 128 rows of A, 8 for the 256 rows of B).  A stage's scales are
// copied into its own columns, so the copy never waits for the MMAs of the
// previous stage, which still read theirs; a set is rewritten only after the
// stage's MMAs completed (the stage was released through its empty barrier).
constexpr uint32_t kSfCol0 = 256;
constexpr uint32_t kSfColsPerStage = 12;
constexpr int kMaxStages = 8;  // 256 + 8 * 12 <= 512 TMEM columns
__device__ __forceinline__ uint32_t sfa_col(int s) { return kSfCol0 + kSfColsPerStage * static_cast<uint32_t>(s); }
__device__ __forceinline__ uint32_t sfb_col(int s) { return sfa_col(s) + 4; }

constexpr int kEpiWarps = 8;
constexpr int kGatherWarps = 4;
constexpr int kGatherSlots = 128 * 8 / (32 * kGatherWarps);  // 16-byte row chunks per gather lane and stage
constexpr int kP1FirstEpi = 2 + kGatherWarps;
constexpr int kP1Threads = 32 * (kP1FirstEpi + kEpiWarps);  // 14 warps
constexpr int kP2FirstEpi = 2;
constexpr int kP2Threads = 32 * (kP2FirstEpi + kEpiWarps);  // 10 warps

// Control area after the stages: mbarriers, TMEM base, abort flag; in
// phase 2 followed by each epilogue warp's 32 x 16 fp32 store staging.
constexpr int kP2Ctrl = 64 * 16 + 16;
constexpr int kStageFloatsPerWarp = 32 * 16;
constexpr int kP2Staging = kEpiWarps * kStageFloatsPerWarp * 4;

// Stage layout (both phases): [A a_rows x 128 B][B 256 rows x 128 B][SFA 512][SFB 2 x 512].
// a_rows (a multiple of 16, at most 128) bounds the routed rows of any
// planner block -- min(block_m, T * top_k) -- so small batches get a small A
// region and more pipeline stages (more weight bytes in flight per SM).  The
// MMA still reads 128 A rows; the rows past a_rows belong to the B region and
// only produce accumulator rows that are never read.

struct P1Params {
  const uint8_t* x;         // (T, K) bf16 or e4m3
  const uint8_t* x_sf;      // (T, K/32) e8m0, row major (mxfp8)
  const uint8_t* w1_sf;     // blocked scales of w1 (mxfp8)
  const int32_t* sorted_ids;
  const int32_t* expert_ids;
  const int32_t* ntpp;
  uint8_t* act;             // (cap_rows, I) bf16 or e4m3
  uint8_t* act_sf;          // blocked scales of act, one tile per (block, 128 intermediate columns) (mxfp8)
  int32_t* flags;           // one per route, cleared here
  int* status;
  int K, N, I, E, top_k, bm, R;
  int max_blocks;           // blocks a kernel may visit
  int w_reuse;              // 1: experts average more than one planner block (weights re-read)
  float* part;              // split-K partials: [kMaxSplitItems][kSplitRows][256] fp32
  int w_fp4;                // weights are MXFP4: e2m1 codes, half the bytes per copy
  int n_jt;                 // ceil(I / 128): work units per planner block
  int stages, stage_bytes;
  int off_b, off_sf;        // stage offsets of the B tile and of the scale tiles
  unsigned long long wait_ns;  // limit of every bounded wait
  // L2 prefetch for small calls (0 / null: none).  pf_all: the byte ranges of
  // all expert weights (and scales), fetched while the planner still runs;
  // otherwise, when the blocks' down-projection tiles fit pf_w2_budget bytes,
  // the w2 tiles the down phase will read, fetched while this phase computes.
  const uint8_t* pf_src[4];
  int64_t pf_bytes[4];
  int pf_all;
  const uint8_t* w2;        // (E, K, N/2) codes: w2_row_bytes per row
  const uint8_t* w2_sf;     // blocked scales of w2 (mxfp8), or null
  int64_t w2_row_bytes;
  int64_t pf_w2_budget;
};

struct P2Params {
  const uint8_t* w2_sf;     // blocked scales of w2 (mxfp8)
  const uint8_t* act_sf;
  const int32_t* sorted_ids;
  const int32_t* expert_ids;
  const int32_t* ntpp;
  const float* topk_w;
  void* yw;                 // weighted down-projection rows, one per (route, split): fp32 (bf16 path) or bf16 (mxfp8 path)
  int32_t* flags;
  int* status;
  int K, I, E, top_k, bm, R;
  int max_blocks;
  int w_reuse;
  int n_ht;                 // ceil(K / 256): work units per planner block
  int n_kc;                 // K-chunks of the down GEMM
  int nsplit2;              // small calls: the down GEMM's N/2 range is split this many ways
  int a_full;               // the stage's A region holds 128 rows
  int w_fp4;                // weights are MXFP4 (as in the gate/up phase)
  int stages, stage_bytes;
  int off_b, off_sf;
  unsigned long long wait_ns;
};

// Per-unit facts every warp role derives the same way (warp-collective).
struct BlockInfo {
  int e;            // expert of the block
  int nend;         // 1 + index of the last routed row in the block (0: none)
  int n16;          // nend rounded up to 16
  uint32_t vm[4];   // routed-row mask, rows 32q .. 32q+31
};

__device__ __forceinline__ BlockInfo block_info(const int32_t* sorted_ids, const int32_t* expert_ids, int b,
                                                int bm, int R, int E) {
  BlockInfo bi;
  const int lane = static_cast<int>(lane_id());
  bi.e = __ldg(expert_ids + b);
  bi.nend = 0;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int r = 32 * q + lane;
    bool v = false;
    if (r < bm) {
      const int id = __ldg(sorted_ids + static_cast<int64_t>(b) * bm + r);
      v = id >= 0 && id < R;
    }
    bi.vm[q] = __ballot_sync(0xffffffffu, v);
    if (bi.vm[q]) bi.nend = 32 * q + 32 - __clz(static_cast<int>(bi.vm[q]));
  }
  if (bi.e < 0 || bi.e >= E) bi.nend = 0;
  bi.n16 = (bi.nend + 15) & ~15;
  return bi;
}

// The global reads block_info needs, issued one unit ahead: every role
// prefetches the next unit's expert id and row ids into registers while it
// works on the current unit, so the loads' latency never sits on the
// pipeline's critical path.  Lane l holds rows l, l+32, l+64, l+96.
struct BlockPf {
  int e;
  int id[4];
};

__device__ __forceinline__ BlockPf block_prefetch(const int32_t* sorted_ids, const int32_t* expert_ids, int u,
                                                  int n_units, int per_block, int bm) {
  BlockPf f;
  f.e = -1;
#pragma unroll
  for (int q = 0; q < 4; ++q) f.id[q] = -1;
  if (u < n_units) {
    const int b = u / per_block;
    const int lane = static_cast<int>(lane_id());
    f.e = __ldg(expert_ids + b);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int r = 32 * q + lane;
      if (r < bm) f.id[q] = __ldg(sorted_ids + static_cast<int64_t>(b) * bm + r);
    }
  }
  return f;
}

// block_info from prefetched data (warp-collective).
__device__ __forceinline__ BlockInfo block_finalize(const BlockPf& f, int R, int E) {
  BlockInfo bi;
  bi.e = f.e;
  bi.nend = 0;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const bool v = f.id[q] >= 0 && f.id[q] < R;
    bi.vm[q] = __ballot_sync(0xffffffffu, v);
    if (bi.vm[q]) bi.nend = 32 * q + 32 - __clz(static_cast<int>(bi.vm[q]));
  }
  if (bi.e < 0 || bi.e >= E) bi.nend = 0;
  bi.n16 = (bi.nend + 15) & ~15;
  return bi;
}

// f.id[q] for a warp-uniform or per-thread q in 0..3 without local memory.
__device__ __forceinline__ int pf_id(const BlockPf& f, int q) {
  return q == 0 ? f.id[0] : q == 1 ? f.id[1] : q == 2 ? f.id[2] : f.id[3];
}

// Number of K-splits per gate/up unit (1: no split), identical in every CTA
// and in the reduction kernel.  Splitting is used only while at least two
// CTAs per unit would otherwise sit idle; more concurrent streams of smaller
// K ranges measured slower on the weight stream than fewer longer ones.
__device__ __forceinline__ int split_count(int n_units, int grid, int n_kc) {
  if (n_units <= 0 || 2 * n_units > grid) return 1;
  int sk = min(min(grid, kMaxSplitItems) / n_units, kMaxSplit);
  sk = min(sk, n_kc / 2);
  return max(sk, 1);
}

__device__ __forceinline__ bool row_valid(const BlockInfo& bi, int c) {
  return (bi.vm[c >> 5] >> (c & 31)) & 1u;
}

__device__ __forceinline__ int num_blocks(const int32_t* ntpp, int bm, int max_blocks) {
  const int n = __ldg(ntpp) / bm;
  return n < 0 ? 0 : (n > max_blocks ? max_blocks : n);
}

// After a wait gave up, copies and MMAs issued before the abort may still be
// landing in shared memory / TMEM.  They finish within microseconds; wait a
// bounded 100 us before the CTA releases its TMEM and exits.
__device__ __forceinline__ void drain_after_abort() {
  const unsigned long long t0 = globaltimer();
  while (globaltimer() - t0 < 100000ull) __nanosleep(1000);
}

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  const uint32_t a = smem_u32(p);
  return p + ((1024u - (a & 1023u)) & 1023u);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// ========================================================================
// phase 1: gate/up GEMM + SwiGLU (+ mxfp8 requant) -> intermediate
// ========================================================================
template <bool kFp8>
__global__ void __launch_bounds__(kP1Threads, 1)
    moe_p1_kernel(const __grid_constant__ CUtensorMap tm_w1, const __grid_constant__ P1Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  const int S = p.stages;
  uint8_t* ctrl = smem + static_cast<size_t>(S) * p.stage_bytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(ctrl);
  uint64_t* empty = full + S;
  uint64_t* acc_full = empty + S;
  uint64_t* acc_empty = acc_full + 2;
  uint32_t* tmem_base_sm = reinterpret_cast<uint32_t*>(acc_empty + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_base_sm + 1);

  constexpr int kNumAcc = kFp8 ? 1 : 2;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  pdl_launch_dependents();
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      // producer lane 0 (with the TMA byte count) + the cp.async completion
      // arrivals of every gather lane
      mbar_init(&full[s], 1 + 32 * kGatherWarps);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], kEpiWarps);
    }
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tm_w1);
  }
  if (warp == 1) {
    tmem_alloc(tmem_base_sm, 512);
    tmem_relinquish();
  }
  if (warp == 2 && lane == 0 && p.pf_all) {
    // small expert set: this CTA's share of every weight byte range goes to
    // L2 now, while the planner runs (the touched experts are not known yet)
    for (int a = 0; a < 4; ++a) {
      const int64_t n16 = p.pf_bytes[a] / 16;
      const int64_t lo = n16 * blockIdx.x / gridDim.x * 16, hi = n16 * (blockIdx.x + 1) / gridDim.x * 16;
      for (int64_t o = lo; o < hi; o += 32768)
        prefetch_l2(p.pf_src[a] + o, static_cast<uint32_t>(hi - o < 32768 ? hi - o : 32768));
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_base_sm;
  // everything above overlaps the planner; its outputs are read below
  pdl_wait();
  // clear the route flags (phase 2 sets them); nothing reads them in this phase
  for (int i = blockIdx.x * kP1Threads + threadIdx.x; i < p.R; i += gridDim.x * kP1Threads) p.flags[i] = 0;

  const int n_blocks = num_blocks(p.ntpp, p.bm, p.max_blocks);
  const int n_jt = p.n_jt;
  const int n_units = n_blocks * n_jt;
  constexpr int kKC = kFp8 ? 128 : 64;  // K elements per stage (128 bytes per row)
  const int n_kc = p.K / kKC;
  const int esize = kFp8 ? 1 : 2;
  // Work items: (unit, K-split).  Without splitting an item is a unit.
  const int nsplit = split_count(n_units, gridDim.x, n_kc);
  const int n_items = n_units * nsplit;
  const int per_block = n_jt * nsplit;  // items per planner block
  // k-range of item w (whose block has bi.nend rows); empty when the item is
  // a non-first split of a unit that is not split.
  auto krange = [&](int w, const BlockInfo& bi, int& k0, int& k1) {
    const int sidx = w % nsplit;
    if (nsplit > 1 && bi.nend <= kSplitRows) {
      k0 = sidx * n_kc / nsplit;
      k1 = (sidx + 1) * n_kc / nsplit;
    } else {
      k0 = 0;
      k1 = sidx == 0 ? n_kc : 0;
    }
  };

  auto stage_ptr = [&](int s) { return smem + static_cast<size_t>(s) * p.stage_bytes; };

  if (warp == 0) {
    // ------------------------------------------------ TMA producer (weights)
    // A weight tile is read by every planner block of its expert: when
    // experts average more than one block (large T) those reads come close
    // together, so the tiles keep normal L2 priority; otherwise each is read
    // once and is evicted first.
    const uint64_t pol = p.w_reuse ? policy_evict_normal() : policy_evict_first();
    // an MXFP4 weight row of a stage is 64 packed bytes, expanded by the copy
    // into the 128-byte row of the unpacked form the MMA reads
    const uint32_t w_row_bytes = p.w_fp4 ? kRowBytes / 2 : kRowBytes;
    const uint32_t tx = 2 * kTI * w_row_bytes + (kFp8 ? 2 * kSfTileBytes : 0);
    const int MT1 = p.N / 128, KT1 = p.K / 128;
    int s = 0;
    uint32_t ph = 0;
    bool ok = true;
    BlockPf pf = block_prefetch(p.sorted_ids, p.expert_ids, blockIdx.x, n_items, per_block, p.bm);
    for (int w = blockIdx.x; w < n_items && ok; w += gridDim.x) {
      const int u = w / nsplit;
      const int j = u - (u / n_jt) * n_jt;
      const BlockPf cur = pf;
      pf = block_prefetch(p.sorted_ids, p.expert_ids, w + gridDim.x, n_items, per_block, p.bm);
      const BlockInfo bi = block_finalize(cur, p.R, p.E);
      if (bi.nend == 0) continue;
      int k0, k1;
      krange(w, bi, k0, k1);
      if (k0 == k1) continue;
      const int gate_row = bi.e * p.N + j * kTI;
      const int up_row = bi.e * p.N + p.I + j * kTI;
      for (int kc = k0; kc < k1; ++kc) {
        if (lane == 0) {
          ok = mbar_wait(&empty[s], ph ^ 1u, abort_flag, p.status, p.wait_ns);
          if (ok) {
            uint8_t* st = stage_ptr(s);
            mbar_arrive_expect_tx(&full[s], tx);
            tma_load_2d(st + p.off_b, &tm_w1, &full[s], kc * kKC, gate_row, pol);
            tma_load_2d(st + p.off_b + 128 * kRowBytes, &tm_w1, &full[s], kc * kKC, up_row, pol);
            if (kFp8) {
              const uint8_t* sfg = p.w1_sf + ((static_cast<int64_t>(bi.e) * MT1 + j) * KT1 + kc) * kSfTileBytes;
              const uint8_t* sfu =
                  p.w1_sf + ((static_cast<int64_t>(bi.e) * MT1 + p.I / 128 + j) * KT1 + kc) * kSfTileBytes;
              bulk_load(st + p.off_sf + kSfTileBytes, sfg, kSfTileBytes, &full[s]);
              bulk_load(st + p.off_sf + 2 * kSfTileBytes, sfu, kSfTileBytes, &full[s]);
            }
          }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        if (++s == S) { s = 0; ph ^= 1u; }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer
    constexpr uint32_t kIdesc = kFp8 ? 0u : idesc_bf16(kM, 256);
    int s = 0;
    uint32_t ph = 0;
    int acc_it = 0;
    bool ok = true;
    BlockPf pf = block_prefetch(p.sorted_ids, p.expert_ids, blockIdx.x, n_items, per_block, p.bm);
    for (int w = blockIdx.x; w < n_items && ok; w += gridDim.x) {
      const BlockPf cur = pf;
      pf = block_prefetch(p.sorted_ids, p.expert_ids, w + gridDim.x, n_items, per_block, p.bm);
      const BlockInfo bi = block_finalize(cur, p.R, p.E);
      if (bi.nend == 0) continue;
      int k0, k1;
      krange(w, bi, k0, k1);
      if (k0 == k1) continue;
      const int buf = acc_it % kNumAcc;
      const uint32_t acc_ph = static_cast<uint32_t>(acc_it / kNumAcc) & 1u;
      if (lane == 0) ok = mbar_wait(&acc_empty[buf], acc_ph ^ 1u, abort_flag, p.status, p.wait_ns);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      tc_fence_after();
      const uint32_t d = tbase + static_cast<uint32_t>(buf) * 256u;
      for (int kc = k0; kc < k1; ++kc) {
        if (lane == 0) {
          ok = mbar_wait(&full[s], ph, abort_flag, p.status, p.wait_ns);
          if (ok) {
            tc_fence_after();
            // the token rows (and scales) arrived through cp.async (generic
            // proxy); the MMA and tcgen05.cp read them through the async proxy
            fence_proxy_async_smem();
            uint8_t* st = stage_ptr(s);
            const uint64_t ad = sdesc_sw128(smem_u32(st));
            const uint64_t bd = sdesc_sw128(smem_u32(st + p.off_b));
            if (kFp8) {
              tc_cp_32x128b_x4(tbase + sfa_col(s), sdesc_sf(smem_u32(st + p.off_sf)));
              tc_cp_32x128b_x4(tbase + sfb_col(s), sdesc_sf(smem_u32(st + p.off_sf + kSfTileBytes)));
              tc_cp_32x128b_x4(tbase + sfb_col(s) + 4, sdesc_sf(smem_u32(st + p.off_sf + 2 * kSfTileBytes)));
            }
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint32_t acc = (kc != k0 || kk != 0) ? 1u : 0u;
              const uint64_t step = static_cast<uint64_t>(2 * kk);  // 32 bytes along K
              if (kFp8) {
                const uint32_t sfid = static_cast<uint32_t>(kk) << 30;
                mma_mxf8(d, ad + step, bd + step, idesc_mxf8(kM, 256, kk, kk, p.w_fp4 ? kFmtE2M1 : kFmtE4M3),
                         (tbase + sfa_col(s)) | sfid, (tbase + sfb_col(s)) | sfid, acc);
              } else {
                mma_f16(d, ad + step, bd + step, kIdesc, acc);
              }
            }
            tc_commit(&empty[s]);
          }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        if (++s == S) { s = 0; ph ^= 1u; }
      }
      if (ok && lane == 0) tc_commit(&acc_full[buf]);
      ++acc_it;
    }
  } else if (warp < kP1FirstEpi) {
    // ------------------------------------------------ token gather
    // The 128 rows x 8 chunks of 16 bytes of a stage's A tile are dealt out
    // once per unit: lane l of gather warp g owns chunk q = l % 8 of rows
    // 4 g + 16 i + l / 8 (i < kGatherSlots), and on mxfp8 the 4-byte token
    // scale of row 32 g + l.  Source addresses are computed once per unit,
    // so a stage costs each lane a handful of independent cp.async; the
    // stage's mbarrier tracks their completion (cp.async.mbarrier.arrive),
    // so the gather warps never wait on their own copies.  Rows past the
    // block's last routed row are not loaded: the accumulator rows they
    // produce are never read.
    const int g = warp - 2;
    const int KS = p.K / 32;
    const int q = lane & 7;
    int s = 0;
    uint32_t ph = 0;
    bool ok = true;
    BlockPf pf = block_prefetch(p.sorted_ids, p.expert_ids, blockIdx.x, n_items, per_block, p.bm);
    for (int w = blockIdx.x; w < n_items && ok; w += gridDim.x) {
      const BlockPf cur = pf;
      pf = block_prefetch(p.sorted_ids, p.expert_ids, w + gridDim.x, n_items, per_block, p.bm);
      const BlockInfo bi = block_finalize(cur, p.R, p.E);
      if (bi.nend == 0) continue;
      int k0, k1;
      krange(w, bi, k0, k1);
      if (k0 == k1) continue;
      const uint8_t* src[kGatherSlots];
      uint32_t dst[kGatherSlots];
      uint32_t live = 0;
#pragma unroll
      for (int i = 0; i < kGatherSlots; ++i) {
        const int r = 4 * g + 16 * i + (lane >> 3);  // row id held by lane r % 32 in cur.id[r / 32 = i / 2]
        const int id = __shfl_sync(0xffffffffu, cur.id[i >> 1], r & 31);
        dst[i] = static_cast<uint32_t>(r * kRowBytes + ((q ^ (r & 7)) << 4));
        src[i] = p.x;
        if (r < bi.nend && row_valid(bi, r)) {
          src[i] = p.x + static_cast<int64_t>(id / p.top_k) * p.K * esize + q * 16;
          live |= 1u << i;
        }
      }
      const uint8_t* sf_src = nullptr;
      const uint32_t sf_dst = static_cast<uint32_t>((lane & 31) * 16 + g * 4);  // row r = 32 g + lane
      if (kFp8) {
        const int r = 32 * g + lane;
        if (r < bi.nend && row_valid(bi, r)) sf_src = p.x_sf + static_cast<int64_t>(pf_id(cur, g) / p.top_k) * KS;
      }
      for (int kc = k0; kc < k1; ++kc) {
        if (lane == 0) ok = mbar_wait(&empty[s], ph ^ 1u, abort_flag, p.status, p.wait_ns);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        const uint32_t abase = smem_u32(stage_ptr(s));
#pragma unroll
        for (int i = 0; i < kGatherSlots; ++i)
          if (live & (1u << i)) cp_async_16(abase + dst[i], src[i] + kc * kRowBytes);
        if (kFp8 && sf_src) cp_async_4(abase + p.off_sf + sf_dst, sf_src + 4 * kc);
        cp_async_mbar_arrive(&full[s]);
        if (++s == S) { s = 0; ph ^= 1u; }
      }
    }
  } else {
    // ------------------------------------------------ epilogue (8 warps)
    if (warp == kP1FirstEpi && lane == 0 && !p.pf_all && p.pf_w2_budget > 0) {
      // Small calls: while this phase computes, pull into L2 the w2 tiles
      // (256 rows each) the down phase's units will read, this CTA's share
      // of the down phase's unit list, unless they exceed the budget.
      const int n_ht2 = (p.K + kTH - 1) / kTH;
      if (static_cast<int64_t>(n_blocks) * p.K * p.w2_row_bytes <= p.pf_w2_budget) {
        const int KT2 = p.I / 128, MT2 = p.K / 128;
        for (int u = blockIdx.x; u < n_blocks * n_ht2; u += gridDim.x) {
          const int e = __ldg(p.expert_ids + u / n_ht2), ht = u % n_ht2;
          if (e < 0 || e >= p.E) continue;
          const int rows = min(kTH, p.K - ht * kTH);
          prefetch_l2(p.w2 + (static_cast<int64_t>(e) * p.K + ht * kTH) * p.w2_row_bytes,
                      static_cast<uint32_t>(rows * p.w2_row_bytes));
          if (p.w2_sf)
            prefetch_l2(p.w2_sf + ((static_cast<int64_t>(e) * MT2 + ht * (kTH / 128)) * KT2) * kSfTileBytes,
                        static_cast<uint32_t>(rows / 128 * KT2 * kSfTileBytes));
        }
      }
    }
    // Warp w reads TMEM lane quadrant w % 4 (rows 32q..32q+31, one per
    // thread) and intermediate columns [64h, 64h + 64) of the unit's tile.
    const int q = warp & 3;
    const int h = (warp - kP1FirstEpi) >> 2;
    const int r = 32 * q + lane;
    int acc_it = 0;
    bool ok = true;
    BlockPf pf = block_prefetch(p.sorted_ids, p.expert_ids, blockIdx.x, n_items, per_block, p.bm);
    for (int w = blockIdx.x; w < n_items && ok; w += gridDim.x) {
      const int u = w / nsplit;
      const int b = u / n_jt, j = u - (u / n_jt) * n_jt;
      const BlockPf cur = pf;
      pf = block_prefetch(p.sorted_ids, p.expert_ids, w + gridDim.x, n_items, per_block, p.bm);
      const BlockInfo bi = block_finalize(cur, p.R, p.E);
      if (bi.nend == 0) continue;
      int k0, k1;
      krange(w, bi, k0, k1);
      if (k0 == k1) continue;
      const int buf = acc_it % kNumAcc;
      const uint32_t acc_ph = static_cast<uint32_t>(acc_it / kNumAcc) & 1u;
      ok = mbar_wait(&acc_full[buf], acc_ph, abort_flag, p.status, p.wait_ns);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const bool mine = row_valid(bi, r);
      const int64_t row = static_cast<int64_t>(b) * p.bm + r;
      const uint32_t tacc = tbase + (static_cast<uint32_t>(32 * q) << 16) + static_cast<uint32_t>(buf) * 256u;
      bool released = false;
      if (nsplit > 1 && bi.nend <= kSplitRows) {
        // split item: hand the raw gate/up partials (rows < 32, quadrant 0)
        // to the reduction kernel
        if (q == 0) {
          float* dst_row = p.part + (static_cast<int64_t>(w) * kSplitRows + r) * 256;
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            const int col = (c < 2 ? 0 : 128) + 64 * h + 32 * (c & 1);  // gate halves, then up halves
            uint32_t v[32];
            tmem_ld32(tacc + col, v);
            tmem_ld_wait();
            if (mine) {
              float4* d4 = reinterpret_cast<float4*>(dst_row + col);
#pragma unroll
              for (int i = 0; i < 8; ++i)
                d4[i] = make_float4(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]),
                                    __uint_as_float(v[4 * i + 2]), __uint_as_float(v[4 * i + 3]));
            }
          }
        }
      } else if (32 * q < bi.nend && kFp8) {
        // One TMEM accumulator on this path: the thread's whole slice (64
        // intermediate columns of row r) is converted in registers and the
        // accumulator handed back to the MMA warp before the global stores.
        uint32_t wq[2][8];
        int scq[2];
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const int col0 = 64 * h + 32 * c;  // within the unit's 128-column tile
          uint32_t gr[32], ur[32];
          tmem_ld32(tacc + col0, gr);
          tmem_ld32(tacc + 128 + col0, ur);
          tmem_ld_wait();
          float a[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) a[i] = silu_f32(__uint_as_float(gr[i])) * __uint_as_float(ur[i]);
          float amax = 0.f;
#pragma unroll
          for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(a[i]));
          int sc = static_cast<int>((__float_as_uint(amax) >> 23) & 0xFFu) - 127 - 8;
          sc = sc < -127 ? -127 : (sc > 127 ? 127 : sc);
          const float inv = __uint_as_float(static_cast<uint32_t>(127 - sc) << 23);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            wq[c][i] = static_cast<uint32_t>(cvt_e4m3x2(a[4 * i] * inv, a[4 * i + 1] * inv)) |
                       (static_cast<uint32_t>(cvt_e4m3x2(a[4 * i + 2] * inv, a[4 * i + 3] * inv)) << 16);
          scq[c] = sc;
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[buf]);
        released = true;
        if (mine) {
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            const int col0 = 64 * h + 32 * c;
            uint4* dst = reinterpret_cast<uint4*>(p.act + row * p.I + j * kTI + col0);
            dst[0] = make_uint4(wq[c][0], wq[c][1], wq[c][2], wq[c][3]);
            dst[1] = make_uint4(wq[c][4], wq[c][5], wq[c][6], wq[c][7]);
            p.act_sf[(static_cast<int64_t>(b) * n_jt + j) * kSfTileBytes + (r & 31) * 16 + (r >> 5) * 4 +
                     (col0 >> 5)] = static_cast<uint8_t>(scq[c] + 127);
          }
        }
      } else if (32 * q < bi.nend) {  // bf16 (two accumulators: the stores overlap the next unit's MMAs)
#pragma unroll 1
        for (int c = 0; c < 2; ++c) {
          const int col0 = 64 * h + 32 * c;  // within the unit's 128-column tile
          uint32_t gr[32], ur[32];
          tmem_ld32(tacc + col0, gr);
          tmem_ld32(tacc + 128 + col0, ur);
          tmem_ld_wait();
          float a[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) a[i] = silu_f32(__uint_as_float(gr[i])) * __uint_as_float(ur[i]);
          const int icol = j * kTI + col0;
          if (mine && icol < p.I) {
            __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(p.act) + row * p.I + icol;
            if (icol + 32 <= p.I) {
              uint32_t w[16];
#pragma unroll
              for (int i = 0; i < 16; ++i) w[i] = pack_bf16x2(a[2 * i], a[2 * i + 1]);
              uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
              for (int i = 0; i < 4; ++i) d4[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
            } else {
#pragma unroll
              for (int i = 0; i < 32; ++i)
                if (icol + i < p.I) dst[i] = __float2bfloat16_rn(a[i]);
            }
          }
        }
      }
      if (!released) {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[buf]);
      }
      ++acc_it;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (*abort_flag) drain_after_abort();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

// ========================================================================
// split-K reduction of the gate/up phase (small problems only)
// ========================================================================
// One warp per (split unit, row): lane l sums columns 4l..4l+3 of the
// gate and up partials over the splits in split order (deterministic),
// applies SwiGLU and writes the intermediate exactly as the gate/up epilogue
// does (bf16, or e4m3 codes with one e8m0 scale per 32 columns -- the amax of
// a 32-column block is reduced over its 8 lanes).
template <bool kFp8>
__global__ void __launch_bounds__(256) moe_p1_reduce_kernel(const __grid_constant__ P1Params p, int grid1) {
  pdl_launch_dependents();
  pdl_wait();  // the gate/up phase's partials are read below
  const int n_blocks = num_blocks(p.ntpp, p.bm, p.max_blocks);
  const int n_units = n_blocks * p.n_jt;
  constexpr int kKC = kFp8 ? 128 : 64;
  const int nsplit = split_count(n_units, grid1, p.K / kKC);
  if (nsplit <= 1) return;
  const int lane = threadIdx.x & 31;
  const int gw = static_cast<int>((blockIdx.x * blockDim.x + threadIdx.x) >> 5);
  const int nw = static_cast<int>((gridDim.x * blockDim.x) >> 5);
  for (int task = gw; task < n_units * kSplitRows; task += nw) {
    const int u = task / kSplitRows, r = task - (task / kSplitRows) * kSplitRows;
    const int b = u / p.n_jt, j = u - (u / p.n_jt) * p.n_jt;
    const BlockInfo bi = block_finalize(block_prefetch(p.sorted_ids, p.expert_ids, b, n_blocks, 1, p.bm), p.R, p.E);
    if (bi.nend == 0 || bi.nend > kSplitRows || r >= bi.nend || !row_valid(bi, r)) continue;  // warp-uniform
    float g[4] = {0.f, 0.f, 0.f, 0.f}, up[4] = {0.f, 0.f, 0.f, 0.f};
    for (int sidx = 0; sidx < nsplit; ++sidx) {
      const float* src = p.part + (static_cast<int64_t>(u * nsplit + sidx) * kSplitRows + r) * 256;
      const float4 a = *reinterpret_cast<const float4*>(src + 4 * lane);
      const float4 c = *reinterpret_cast<const float4*>(src + 128 + 4 * lane);
      g[0] += a.x; g[1] += a.y; g[2] += a.z; g[3] += a.w;
      up[0] += c.x; up[1] += c.y; up[2] += c.z; up[3] += c.w;
    }
    float a[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) a[i] = silu_f32(g[i]) * up[i];
    const int64_t row = static_cast<int64_t>(b) * p.bm + r;
    const int icol = j * kTI + 4 * lane;
    if (kFp8) {
      float amax = fmaxf(fmaxf(fabsf(a[0]), fabsf(a[1])), fmaxf(fabsf(a[2]), fabsf(a[3])));
#pragma unroll
      for (int d = 1; d < 8; d <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, d));
      int sc = static_cast<int>((__float_as_uint(amax) >> 23) & 0xFFu) - 127 - 8;
      sc = sc < -127 ? -127 : (sc > 127 ? 127 : sc);
      const float inv = __uint_as_float(static_cast<uint32_t>(127 - sc) << 23);
      const uint32_t wv = static_cast<uint32_t>(cvt_e4m3x2(a[0] * inv, a[1] * inv)) |
                          (static_cast<uint32_t>(cvt_e4m3x2(a[2] * inv, a[3] * inv)) << 16);
      *reinterpret_cast<uint32_t*>(p.act + row * p.I + icol) = wv;
      if ((lane & 7) == 0)
        p.act_sf[(static_cast<int64_t>(b) * p.n_jt + j) * kSfTileBytes + (r & 31) * 16 + (r >> 5) * 4 + (lane >> 3)] =
            static_cast<uint8_t>(sc + 127);
    } else if (icol < p.I) {
      __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(p.act) + row * p.I + icol;
      if (icol + 4 <= p.I) {
        *reinterpret_cast<uint2*>(dst) = make_uint2(pack_bf16x2(a[0], a[1]), pack_bf16x2(a[2], a[3]));
      } else {
#pragma unroll
        for (int i = 0; i < 4; ++i)
          if (icol + i < p.I) dst[i] = __float2bfloat16_rn(a[i]);
      }
    }
  }
}

// ========================================================================
// phase 2: down GEMM + routing weight -> one fp32 row per route
// ========================================================================
template <bool kFp8>
__global__ void __launch_bounds__(kP2Threads, 1)
    moe_p2_kernel(const __grid_constant__ CUtensorMap tm_w2, const __grid_constant__ CUtensorMap tm_w2x,
                  const __grid_constant__ CUtensorMap tm_act, const __grid_constant__ CUtensorMap tm_actx,
                  const __grid_constant__ P2Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  const int S = p.stages;
  uint8_t* ctrl = smem + static_cast<size_t>(S) * p.stage_bytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(ctrl);
  uint64_t* empty = full + S;
  uint64_t* acc_full = empty + S;
  uint64_t* acc_empty = acc_full + 2;
  uint32_t* tmem_base_sm = reinterpret_cast<uint32_t*>(acc_empty + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_base_sm + 1);

  constexpr int kNumAcc = kFp8 ? 1 : 2;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_launch_dependents();
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], kEpiWarps);
    }
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tm_w2);
    prefetch_tmap(&tm_w2x);
    prefetch_tmap(&tm_act);
    prefetch_tmap(&tm_actx);
  }
  if (warp == 1) {
    tmem_alloc(tmem_base_sm, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_base_sm;
  pdl_wait();  // the gate/up phase's intermediate is read below

  const int n_blocks = num_blocks(p.ntpp, p.bm, p.max_blocks);
  constexpr int TH = kTH;
  const int n_ht = p.n_ht;
  const int n_units = n_blocks * n_ht;
  // work items: (unit, split of the N/2 contraction); without splitting an item is a unit
  const int S2 = p.nsplit2;
  const int n_items = n_units * S2, per_block = n_ht * S2;
  constexpr int kKC = kFp8 ? 128 : 64;
  auto stage_ptr = [&](int s) { return smem + static_cast<size_t>(s) * p.stage_bytes; };

  if (warp == 0) {
    // ------------------------------------------------ TMA producer
    const uint64_t pol_w = p.w_reuse ? policy_evict_normal() : policy_evict_first();  // as in the gate/up phase
    const uint64_t pol_a = policy_evict_last();
    const int MT2 = p.K / 128, KT2 = p.I / 128;
    int s = 0;
    uint32_t ph = 0;
    bool ok = true;
    BlockPf pf = block_prefetch(p.sorted_ids, p.expert_ids, blockIdx.x, n_items, per_block, p.bm);
    for (int w = blockIdx.x; w < n_items && ok; w += gridDim.x) {
      const int u = w / S2, b = u / n_ht, ht = u - (u / n_ht) * n_ht;
      const int k0 = (w - u * S2) * p.n_kc / S2, k1 = (w - u * S2 + 1) * p.n_kc / S2;
      const BlockPf cur = pf;
      pf = block_prefetch(p.sorted_ids, p.expert_ids, w + gridDim.x, n_items, per_block, p.bm);
      const BlockInfo bi = block_finalize(cur, p.R, p.E);
      if (bi.nend == 0) continue;
      const int nb = min(TH, p.K - ht * TH) / 128;  // 128-row pieces of this feature tile
      const int w2_row = bi.e * p.K + ht * TH;
      // A block of at least 64 rows takes its intermediate rows as one
      // 128-row box (rows past the block are loaded and never stored) and a
      // full feature tile its w2 rows as one 256-row box: fewer, larger copies
      // per stage than 16-row and 128-row pieces.
      const bool big_a = p.a_full && bi.n16 >= 64;
      const int a_rows = big_a ? 128 : bi.n16;
      const uint32_t w_row_bytes = p.w_fp4 ? kRowBytes / 2 : kRowBytes;  // packed MXFP4 rows
      const uint32_t tx = nb * 128 * w_row_bytes + a_rows * kRowBytes + (kFp8 ? (1 + nb) * kSfTileBytes : 0);
      for (int kc = k0; kc < k1; ++kc) {
        if (lane == 0) {
          ok = mbar_wait(&empty[s], ph ^ 1u, abort_flag, p.status, p.wait_ns);
          if (ok) {
            uint8_t* st = stage_ptr(s);
            mbar_arrive_expect_tx(&full[s], tx);
            if (big_a) {
              tma_load_2d(st, &tm_actx, &full[s], kc * kKC, b * p.bm, pol_a);
            } else {
              for (int i = 0; i < bi.n16 / 16; ++i)
                tma_load_2d(st + i * 16 * kRowBytes, &tm_act, &full[s], kc * kKC, b * p.bm + 16 * i, pol_a);
            }
            if (nb == 2)
              tma_load_2d(st + p.off_b, &tm_w2x, &full[s], kc * kKC, w2_row, pol_w);
            else
              tma_load_2d(st + p.off_b, &tm_w2, &full[s], kc * kKC, w2_row, pol_w);
            if (kFp8) {
              bulk_load(st + p.off_sf, p.act_sf + (static_cast<int64_t>(b) * KT2 + kc) * kSfTileBytes, kSfTileBytes,
                        &full[s]);
              for (int i = 0; i < nb; ++i)
                bulk_load(st + p.off_sf + (1 + i) * kSfTileBytes,
                          p.w2_sf + ((static_cast<int64_t>(bi.e) * MT2 + (ht * TH) / 128 + i) * KT2 + kc) * kSfTileBytes,
                          kSfTileBytes, &full[s]);
            }
          }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        if (++s == S) { s = 0; ph ^= 1u; }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer
    int s = 0;
    uint32_t ph = 0;
    int acc_it = 0;
    bool ok = true;
    BlockPf pf = block_prefetch(p.sorted_ids, p.expert_ids, blockIdx.x, n_items, per_block, p.bm);
    for (int w = blockIdx.x; w < n_items && ok; w += gridDim.x) {
      const int u = w / S2, ht = u - (u / n_ht) * n_ht;
      const int k0 = (w - u * S2) * p.n_kc / S2, k1 = (w - u * S2 + 1) * p.n_kc / S2;
      const BlockPf cur = pf;
      pf = block_prefetch(p.sorted_ids, p.expert_ids, w + gridDim.x, n_items, per_block, p.bm);
      const BlockInfo bi = block_finalize(cur, p.R, p.E);
      if (bi.nend == 0) continue;
      const int nn = min(TH, p.K - ht * TH);
      const int buf = acc_it % kNumAcc;
      const uint32_t acc_ph = static_cast<uint32_t>(acc_it / kNumAcc) & 1u;
      if (lane == 0) ok = mbar_wait(&acc_empty[buf], acc_ph ^ 1u, abort_flag, p.status, p.wait_ns);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      tc_fence_after();
      const uint32_t d = tbase + static_cast<uint32_t>(buf) * 256u;
      for (int kc = k0; kc < k1; ++kc) {
        if (lane == 0) {
          ok = mbar_wait(&full[s], ph, abort_flag, p.status, p.wait_ns);
          if (ok) {
            tc_fence_after();
            uint8_t* st = stage_ptr(s);
            const uint64_t ad = sdesc_sw128(smem_u32(st));
            const uint64_t bd = sdesc_sw128(smem_u32(st + p.off_b));
            if (kFp8) {
              tc_cp_32x128b_x4(tbase + sfa_col(s), sdesc_sf(smem_u32(st + p.off_sf)));
              tc_cp_32x128b_x4(tbase + sfb_col(s), sdesc_sf(smem_u32(st + p.off_sf + kSfTileBytes)));
              tc_cp_32x128b_x4(tbase + sfb_col(s) + 4, sdesc_sf(smem_u32(st + p.off_sf + 2 * kSfTileBytes)));
            }
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint32_t acc = (kc != k0 || kk != 0) ? 1u : 0u;
              const uint64_t step = static_cast<uint64_t>(2 * kk);
              if (kFp8) {
                const uint32_t sfid = static_cast<uint32_t>(kk) << 30;
                mma_mxf8(d, ad + step, bd + step, idesc_mxf8(kM, nn, kk, kk, p.w_fp4 ? kFmtE2M1 : kFmtE4M3),
                         (tbase + sfa_col(s)) | sfid, (tbase + sfb_col(s)) | sfid, acc);
              } else {
                mma_f16(d, ad + step, bd + step, idesc_bf16(kM, nn), acc);
              }
            }
            tc_commit(&empty[s]);
          }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        if (++s == S) { s = 0; ph ^= 1u; }
      }
      if (ok && lane == 0) tc_commit(&acc_full[buf]);
      ++acc_it;
    }
  } else {
    // ------------------------------------------------ epilogue (8 warps)
    // Warp w reads TMEM lane quadrant w % 4 (rows 32q..32q+31, one per
    // thread) and half h of the unit's output features.
    const int q = warp & 3;
    const int h = (warp - kP2FirstEpi) >> 2;
    const int r = 32 * q + lane;
    uint4* stg4 = reinterpret_cast<uint4*>(ctrl + kP2Ctrl) + (warp - kP2FirstEpi) * (kStageFloatsPerWarp / 4);
    int acc_it = 0;
    bool ok = true;
    BlockPf pf = block_prefetch(p.sorted_ids, p.expert_ids, blockIdx.x, n_items, per_block, p.bm);
    for (int w = blockIdx.x; w < n_items && ok; w += gridDim.x) {
      const int u = w / S2, s2 = w - u * S2, ht = u - (u / n_ht) * n_ht;
      const BlockPf cur = pf;
      pf = block_prefetch(p.sorted_ids, p.expert_ids, w + gridDim.x, n_items, per_block, p.bm);
      const BlockInfo bi = block_finalize(cur, p.R, p.E);
      if (bi.nend == 0) continue;
      const int nn = min(TH, p.K - ht * TH);
      // the route, its partial row (one per route and split of N/2) and its
      // weight, fetched while the MMAs run
      const bool mine = row_valid(bi, r);
      int route = 0, prow = 0;
      float wgt = 0.f;
      if (mine) {
        route = pf_id(cur, q);
        prow = route * S2 + s2;
        wgt = __ldg(p.topk_w + route);
      }
      const int buf = acc_it % kNumAcc;
      const uint32_t acc_ph = static_cast<uint32_t>(acc_it / kNumAcc) & 1u;
      ok = mbar_wait(&acc_full[buf], acc_ph, abort_flag, p.status, p.wait_ns);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const uint32_t tacc = tbase + (static_cast<uint32_t>(32 * q) << 16) + static_cast<uint32_t>(buf) * 256u;
      bool released = false;
      if (32 * q < bi.nend && kFp8) {
        // One TMEM accumulator on this path: the thread's weighted half-row is
        // packed to bf16 in registers (up to 4 slices of 32 features) and the
        // accumulator handed back to the MMA warp before the slices go through
        // the staging buffer to global memory, as below.
        const int half = nn / 2;
        const int64_t col_base = static_cast<int64_t>(ht) * TH + h * half;
        uint32_t pk[4][16];
#pragma unroll
        for (int sl = 0; sl < 4; ++sl) {
          if (32 * sl < half) {  // uniform
            uint32_t yr[32];
            tmem_ld32(tacc + h * half + 32 * sl, yr);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 16; ++i)
              pk[sl][i] = pack_bf16x2(wgt * __uint_as_float(yr[2 * i]), wgt * __uint_as_float(yr[2 * i + 1]));
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[buf]);
        released = true;
#pragma unroll
        for (int sl = 0; sl < 4; ++sl) {
          if (32 * sl < half) {
            __syncwarp();
#pragma unroll
            for (int i = 0; i < 4; ++i)
              stg4[lane * 4 + (i ^ ((lane >> 1) & 3))] =
                  make_uint4(pk[sl][4 * i], pk[sl][4 * i + 1], pk[sl][4 * i + 2], pk[sl][4 * i + 3]);
            __syncwarp();
#pragma unroll
            for (int it = 0; it < 4; ++it) {
              const int rl = 8 * it + (lane >> 2), cq = lane & 3;
              const uint4 v = stg4[rl * 4 + (cq ^ ((rl >> 1) & 3))];
              const int route_l = __shfl_sync(0xffffffffu, prow, rl);
              const int mine_l = __shfl_sync(0xffffffffu, static_cast<int>(mine), rl);
              if (mine_l) {
                const int64_t e0 = static_cast<int64_t>(route_l) * p.K + col_base + 32 * sl;
                *reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(p.yw) + e0 + 8 * cq) = v;
              }
            }
          }
        }
        if (mine && ht == 0 && h == 0 && s2 == 0) p.flags[route] = 1;
      } else if (32 * q < bi.nend) {
        // Thread = row.  Each slice of the warp's 32 rows goes through shared
        // memory so that the stores leave as 64 contiguous bytes per row (8
        // rows per instruction) instead of 16 bytes to 32 different rows.
        // 16-byte slot i of row l sits at i ^ ((l >> 1) & 3), so both the
        // row-per-lane writes and the 8-rows-per-instruction reads touch all
        // 32 banks (4 wavefronts per 512 bytes).  The weighted rows stay fp32
        // (16 columns per staging pass).
        const int half = nn / 2;
        const int64_t col_base = static_cast<int64_t>(ht) * TH + h * half;
#pragma unroll 1
        for (int c = 0; c < half; c += 32) {
          uint32_t yr[32];
          tmem_ld32(tacc + h * half + c, yr);
          tmem_ld_wait();
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            __syncwarp();
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int k = 16 * hh + 4 * i;
              stg4[lane * 4 + (i ^ ((lane >> 1) & 3))] =
                  make_uint4(__float_as_uint(wgt * __uint_as_float(yr[k])),
                             __float_as_uint(wgt * __uint_as_float(yr[k + 1])),
                             __float_as_uint(wgt * __uint_as_float(yr[k + 2])),
                             __float_as_uint(wgt * __uint_as_float(yr[k + 3])));
            }
            __syncwarp();
#pragma unroll
            for (int it = 0; it < 4; ++it) {
              const int rl = 8 * it + (lane >> 2), cq = lane & 3;
              const uint4 v = stg4[rl * 4 + (cq ^ ((rl >> 1) & 3))];
              const int route_l = __shfl_sync(0xffffffffu, prow, rl);
              const int mine_l = __shfl_sync(0xffffffffu, static_cast<int>(mine), rl);
              if (mine_l) {
                const int64_t e0 = static_cast<int64_t>(route_l) * p.K + col_base + c;
                *reinterpret_cast<uint4*>(reinterpret_cast<float*>(p.yw) + e0 + 16 * hh + 4 * cq) = v;
              }
            }
          }
        }
        if (mine && ht == 0 && h == 0 && s2 == 0) p.flags[route] = 1;
      }
      if (!released) {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[buf]);
      }
      ++acc_it;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (*abort_flag) drain_after_abort();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

// ========================================================================
// combine: out[t] = bf16( sum over j, s of yw[(t*top_k + j)*nsplit2 + s] ),
// routes in order
// ========================================================================
// 8 consecutive partials of one row, kept packed in registers until they are
// summed (bf16: one 16-byte load, fp32: two).
template <typename TP>
struct Raw8;
template <>
struct Raw8<__nv_bfloat16> {
  uint4 a;
};
template <>
struct Raw8<float> {
  uint4 a, b;
};
__device__ __forceinline__ void load_raw8(const __nv_bfloat16* p, Raw8<__nv_bfloat16>& r) {
  r.a = __ldg(reinterpret_cast<const uint4*>(p));
}
__device__ __forceinline__ void load_raw8(const float* p, Raw8<float>& r) {
  r.a = __ldg(reinterpret_cast<const uint4*>(p));
  r.b = __ldg(reinterpret_cast<const uint4*>(p) + 1);
}
__device__ __forceinline__ void add_raw8(const Raw8<__nv_bfloat16>& r, float (&acc)[8]) {
  const uint32_t w[4] = {r.a.x, r.a.y, r.a.z, r.a.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    acc[2 * i] += __uint_as_float(w[i] << 16);
    acc[2 * i + 1] += __uint_as_float(w[i] & 0xFFFF0000u);
  }
}
__device__ __forceinline__ void add_raw8(const Raw8<float>& r, float (&acc)[8]) {
  const uint32_t w[8] = {r.a.x, r.a.y, r.a.z, r.a.w, r.b.x, r.b.y, r.b.z, r.b.w};
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] += __uint_as_float(w[i]);
}

// One thread sums 8 consecutive features of one token over its top_k routes
// (and their splits).  The route flags and every route's 8 partials are loaded
// before any of them is used (the loads of a route whose flag is 0 read
// workspace bytes that are then discarded), so a thread has all its loads in
// flight at once; the sum runs in route order, so the result does not depend
// on scheduling.
template <typename TP, int kMaxK>
__global__ void __launch_bounds__(256, sizeof(TP) == 2 ? 4 : 2)
    moe_combine_kernel(const TP* __restrict__ yw, const int32_t* __restrict__ flags, __nv_bfloat16* __restrict__ out,
                       int T, int K, int top_k, int nsplit2) {
  pdl_wait();  // the down phase's partial rows are read below
  const int kv = K / 8;
  const int64_t n = static_cast<int64_t>(T) * kv;
  for (int64_t v = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; v < n;
       v += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t t = v / kv;
    const int h = static_cast<int>(v - t * kv) * 8;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    // the token's partial rows: route j, split s at row (t * top_k + j) * nsplit2 + s, summed in
    // that (route-major) order
    const int nrows = top_k * nsplit2;
    for (int j0 = 0; j0 < nrows; j0 += kMaxK) {
      int f[kMaxK];
      Raw8<TP> y[kMaxK];
#pragma unroll
      for (int j = 0; j < kMaxK; ++j) {
        f[j] = 0;
        if (j0 + j < nrows) {
          f[j] = __ldg(flags + t * top_k + (j0 + j) / nsplit2);
          load_raw8(yw + (t * nrows + j0 + j) * K + h, y[j]);
        }
      }
#pragma unroll
      for (int j = 0; j < kMaxK; ++j)
        if (f[j]) add_raw8(y[j], acc);
    }
    __nv_bfloat162 o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) o[i] = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
    *reinterpret_cast<uint4*>(out + t * K + h) = *reinterpret_cast<const uint4*>(o);
  }
}

// ========================================================================
// host side
// ========================================================================
struct WsLayout {
  int64_t act, act_sf, yw, flags, part, total;
  int64_t cap_rows;
};

static int64_t round_up(int64_t a, int64_t b) { return (a + b - 1) / b * b; }

// Splits of the down GEMM's N/2 contraction: small calls (at most 64 down
// units even if every planner block were used) spread it over up to 4 CTAs
// per unit, each writing its own partial row, which the combine adds in
// order.  A function of the problem's sizes only (the workspace size follows
// from it).
static int down_splits(bool fp8, int T, int K, int N, int E, int top_k, int bm) {
  const int64_t R = static_cast<int64_t>(T) * top_k;
  const int64_t blocks = round_up(R + static_cast<int64_t>(E) * (bm - 1), bm) / bm;
  const int64_t units = blocks * ((K + kTH - 1) / kTH);
  const int I = N / 2;
  const int n_kc = fp8 ? I / 128 : (I + 63) / 64;
  if (units > 64) return 1;
  return std::max(1, std::min(4, n_kc / 2));
}

static WsLayout ws_layout(bool fp8, int T, int K, int N, int E, int top_k, int bm) {
  WsLayout w{};
  const int64_t R = static_cast<int64_t>(T) * top_k;
  const int64_t cap = R + static_cast<int64_t>(E) * (bm - 1);
  w.cap_rows = round_up(cap, bm);
  const int64_t I = N / 2;
  int64_t off = 0;
  w.act = off;
  off = round_up(off + w.cap_rows * I * (fp8 ? 1 : 2), 1024);
  w.act_sf = off;
  if (fp8) off = round_up(off + (w.cap_rows / bm) * (I / 128) * kSfTileBytes, 1024);
  w.yw = off;
  off = round_up(off + R * down_splits(fp8, T, K, N, E, top_k, bm) * K * (fp8 ? 2 : 4), 1024);
  w.flags = off;
  off = round_up(off + R * 4, 1024);
  w.part = off;
  {
    // split items never exceed kMaxSplitItems nor kMaxSplit per possible unit
    const int64_t max_units = (w.cap_rows / bm) * ((I + kTI - 1) / kTI);
    const int64_t items = std::min<int64_t>(kMaxSplitItems, max_units * kMaxSplit);
    off = round_up(off + items * kSplitRows * 256 * 4, 256);
  }
  w.total = off;
  return w;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encode() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// 2-D row-major [rows x cols] tensor, box [box_rows x 128 bytes], 128-byte swizzle.
// Element kinds of the 2-D tensor maps: bf16, one-byte codes (e4m3 / e8m0),
// and packed e2m1 pairs, which the copy expands into the unpacked form (each
// 16 values' 8 bytes followed by an 8-byte gap) that the block-scaled MMA
// reads as one byte per value; a box row is then 128 values in both cases.
enum TmapKind { kTmBf16, kTmU8, kTmFp4 };

static int make_tmap(CUtensorMap* m, const void* base, TmapKind kind, int64_t rows, int64_t cols, int box_rows) {
  EncodeTiledFn enc = get_encode();
  if (!enc) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled entry point not available");
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  const int64_t row_bytes = kind == kTmBf16 ? cols * 2 : (kind == kTmU8 ? cols : cols / 2);
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(row_bytes)};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(kind == kTmBf16 ? kRowBytes / 2 : kRowBytes),
                       static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  const CUtensorMapDataType dt = kind == kTmBf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                 : kind == kTmU8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                                 : CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B;
  const CUresult r = enc(m, dt, 2,
                         const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return MOE_OK;
}

static bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// done[dev]: the attribute is set on that device (host threads may race to
// set it; setting it twice is harmless)
template <typename K>
static int set_smem_attr(K kernel, int bytes, std::atomic<bool>* done) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cuda_fail("cudaGetDevice");
  if (dev < kMaxDevices && done[dev].load(std::memory_order_relaxed)) return MOE_OK;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit) != cudaSuccess)
    return cuda_fail("cudaFuncSetAttribute");
  (void)bytes;
  if (dev < kMaxDevices) done[dev].store(true, std::memory_order_relaxed);
  return MOE_OK;
}

struct FusedArgs {
  bool fp8;
  bool w_fp4;  // mxfp8 activations with MXFP4 weights
  const void* x;
  const uint8_t* x_sf;
  const void* w1;
  const uint8_t* w1_sf;
  const void* w2;
  const uint8_t* w2_sf;
  const int32_t* sorted_ids;
  const int32_t* expert_ids;
  const int32_t* ntpp;
  const float* topk_w;
  void* out;
  int T, K, N, E, top_k, bm;
  int64_t capacity;
  void* ws;
  int64_t ws_bytes;
  const moe_tuning* tune;
  cudaStream_t stream;
};

static int a_region_rows(int bm, int64_t R) {
  const int64_t r = std::min<int64_t>(bm, R);
  return static_cast<int>(std::min<int64_t>(kM, round_up(std::max<int64_t>(r, 1), 16)));
}
static int off_b_of(int a_rows) { return static_cast<int>(round_up(static_cast<int64_t>(a_rows) * kRowBytes, 1024)); }
static int off_sf_of(int a_rows) { return off_b_of(a_rows) + 2 * 128 * kRowBytes; }
static int stage_bytes(bool fp8, int a_rows) {
  return static_cast<int>(round_up(off_sf_of(a_rows) + (fp8 ? 3 * kSfTileBytes : 0), 1024));
}
constexpr int kP1Ctrl = 64 * 16 + 16;  // barriers, tmem base, abort flag

static int pick_stages(int stage_bytes, int ctrl, int requested, int max_stages) {
  int s = (kSmemLimit - 1024 - ctrl) / stage_bytes;
  if (s > max_stages) s = max_stages;
  if (requested > 0 && requested < s) s = requested;
  return s;
}

// Every argument check of the fused forward that does not depend on the
// workspace, in the order the status codes are documented.  Returns MOE_OK or
// the error status (message in moe_last_error()).  `has_ws`: the workspace
// pointer is checked for null and alignment as well.
static int check_fused(const FusedArgs& a, bool has_ws) {
  const char* nm = a.w_fp4 ? "fused_moe_mxfp4" : (a.fp8 ? "fused_moe_mxfp8" : "fused_moe_bf16");
  if (a.T < 0 || a.K <= 0 || a.N <= 0 || a.E < 1 || a.top_k < 1)
    return fail(MOE_ERR_INVALID_ARG, "%s: need T >= 0, K > 0, N > 0, E >= 1, top_k >= 1", nm);
  if (!valid_block_m(a.bm)) return fail(MOE_ERR_UNSUPPORTED, "%s: block_m must be 16, 32, 64 or 128", nm);
  if (a.fp8) {
    if (a.K % 256 != 0 || a.N % 256 != 0)
      return fail(MOE_ERR_UNSUPPORTED, "%s: K and N must be multiples of 256 (K=%d N=%d)", nm, a.K, a.N);
  } else {
    if (a.K % 128 != 0 || a.N % 16 != 0)
      return fail(MOE_ERR_UNSUPPORTED, "%s: K %% 128 == 0 and N %% 16 == 0 required (K=%d N=%d)", nm, a.K, a.N);
  }
  const int64_t need_cap = moe_align_capacity(a.T, a.top_k, a.E, a.bm);
  if (need_cap >= (int64_t(1) << 31)) return fail(MOE_ERR_UNSUPPORTED, "%s: T*top_k + E*(block_m-1) >= 2^31", nm);
  if (a.capacity < need_cap)
    return fail(MOE_ERR_INVALID_ARG, "%s: capacity %lld < required %lld", nm, (long long)a.capacity,
                (long long)need_cap);
  if (static_cast<int64_t>(a.E) * a.N >= (int64_t(1) << 31) || static_cast<int64_t>(a.E) * a.K >= (int64_t(1) << 31))
    return fail(MOE_ERR_UNSUPPORTED, "%s: E*N and E*K must be < 2^31", nm);
  if (a.T == 0) return MOE_OK;
  if (!a.x || !a.w1 || !a.w2 || !a.sorted_ids || !a.expert_ids || !a.ntpp || !a.topk_w || !a.out ||
      (has_ws && !a.ws))
    return fail(MOE_ERR_INVALID_ARG, "%s: null pointer", nm);
  if (a.fp8 && (!a.x_sf || !a.w1_sf || !a.w2_sf)) return fail(MOE_ERR_INVALID_ARG, "%s: null scale pointer", nm);
  if (!aligned(a.x, 16) || !aligned(a.w1, 16) || !aligned(a.w2, 16) || !aligned(a.out, 16) ||
      (has_ws && !aligned(a.ws, 256)) ||
      (a.fp8 && (!aligned(a.x_sf, 16) || !aligned(a.w1_sf, 16) || !aligned(a.w2_sf, 16))) ||
      !aligned(a.sorted_ids, 4) || !aligned(a.expert_ids, 4) || !aligned(a.ntpp, 4) || !aligned(a.topk_w, 4))
    return fail(MOE_ERR_ALIGNMENT, "%s: tensors must be 16-byte aligned and the workspace 256-byte aligned", nm);
  if (a.w_fp4 && (!aligned(a.w1, 32) || !aligned(a.w2, 32)))
    return fail(MOE_ERR_ALIGNMENT, "%s: packed e2m1 weights must be 32-byte aligned", nm);
  return MOE_OK;
}

// The top-k reduction: one wave of resident blocks of the combine kernel
// (grid-stride beyond it) over the partial rows `yw` (bf16 when `bf16_parts`,
// else fp32; nsplit2 per route) and the route flags.  Chained to the
// previous launch by programmatic dependent launch.
static int launch_combine(bool bf16_parts, const uint8_t* yw, const int32_t* flags, void* out, int T, int K,
                          int top_k, int nsplit2, int nsm, cudaStream_t stream) {
  static std::atomic<int> comb_occ[2];  // races store the same value
  int occ = comb_occ[bf16_parts ? 1 : 0].load(std::memory_order_relaxed);
  cudaError_t err;
  if (occ == 0) {
    int nb = 0;
    err = bf16_parts
              ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, moe_combine_kernel<__nv_bfloat16, 8>, 256, 0)
              : cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, moe_combine_kernel<float, 8>, 256, 0);
    if (err != cudaSuccess) return cuda_fail("fused_moe: combine occupancy query", err);
    occ = nb < 1 ? 1 : nb;
    comb_occ[bf16_parts ? 1 : 0].store(occ, std::memory_order_relaxed);
  }
  const int64_t nvec = static_cast<int64_t>(T) * (K / 8);
  const int64_t cblocks = (nvec + 255) / 256;
  const int64_t wave = static_cast<int64_t>(occ) * nsm;
  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t c3 = {};
  c3.gridDim = dim3(static_cast<unsigned>(cblocks < wave ? cblocks : wave), 1, 1);
  c3.blockDim = dim3(256, 1, 1);
  c3.stream = stream;
  c3.attrs = pdl;
  c3.numAttrs = 1;
  __nv_bfloat16* outp = static_cast<__nv_bfloat16*>(out);
  err = bf16_parts ? cudaLaunchKernelEx(&c3, moe_combine_kernel<__nv_bfloat16, 8>,
                                        reinterpret_cast<const __nv_bfloat16*>(yw), flags, outp, T, K, top_k, nsplit2)
                   : cudaLaunchKernelEx(&c3, moe_combine_kernel<float, 8>, reinterpret_cast<const float*>(yw), flags,
                                        outp, T, K, top_k, nsplit2);
  if (err != cudaSuccess) return cuda_fail("fused_moe: combine launch", err);
  return MOE_OK;
}

static int run_fused(const FusedArgs& a) {
  const char* nm = a.w_fp4 ? "fused_moe_mxfp4" : (a.fp8 ? "fused_moe_mxfp8" : "fused_moe_bf16");
  int rc0 = check_fused(a, true);
  if (rc0 != MOE_OK || a.T == 0) return rc0;
  const WsLayout L = ws_layout(a.fp8, a.T, a.K, a.N, a.E, a.top_k, a.bm);
  if (a.ws_bytes < L.total)
    return fail(MOE_ERR_WORKSPACE, "%s: workspace %lld bytes < required %lld", nm, (long long)a.ws_bytes,
                (long long)L.total);

  const int I = a.N / 2;
  uint8_t* ws = static_cast<uint8_t*>(a.ws);
  // Blocks a kernel may visit: never past the caller's sorted_token_ids /
  // expert_ids arrays, even if num_tokens_post_padded were out of range.
  const int max_blocks = static_cast<int>(std::min<int64_t>(L.cap_rows, a.capacity) / a.bm);
  static std::atomic<int*> status_ptr[kMaxDevices];  // per device; races store the same address
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cuda_fail("cudaGetDevice");
  if (dev >= kMaxDevices) return fail(MOE_ERR_UNSUPPORTED, "%s: device index %d too large", nm, dev);
  int* status = status_ptr[dev].load(std::memory_order_relaxed);
  if (!status) {
    void* sp = nullptr;
    if (cudaGetSymbolAddress(&sp, g_moe_status) != cudaSuccess) return cuda_fail("cudaGetSymbolAddress");
    status = static_cast<int*>(sp);
    status_ptr[dev].store(status, std::memory_order_relaxed);
  }

  int rc;
  const unsigned long long wait_ns =
      a.tune && a.tune->wait_timeout_ns > 0 ? static_cast<unsigned long long>(a.tune->wait_timeout_ns) : kWaitTimeoutNs;
  const int nsm = sm_count();
  if (nsm <= 0) return cuda_fail("cudaDeviceGetAttribute(SM count)");
  if (!a.fp8) {
    const int mode = a.tune ? a.tune->small_batch : 0;
    const bool small = mode >= 0 && small_batch_shapes_ok(a.T, a.K, a.N, a.top_k) &&
                       (mode > 0 || static_cast<int64_t>(a.T) * a.top_k <= kSbAutoRoutes);
    if (small) {
      SbArgs sb{};
      sb.x = a.x; sb.w1 = a.w1; sb.w2 = a.w2;
      sb.sorted_ids = a.sorted_ids; sb.expert_ids = a.expert_ids; sb.ntpp = a.ntpp;
      sb.topk_w = a.topk_w;
      sb.T = a.T; sb.K = a.K; sb.N = a.N; sb.E = a.E; sb.top_k = a.top_k; sb.bm = a.bm;
      sb.max_blocks = max_blocks;
      sb.act = ws + L.act;
      sb.yw = reinterpret_cast<float*>(ws + L.yw);
      sb.flags = reinterpret_cast<int32_t*>(ws + L.flags);
      sb.pf_all = static_cast<int64_t>(a.E) * (a.N + I) * a.K * 2 <= kPrefetchAllBytes;
      void* const* ev = a.tune ? a.tune->phase_events : nullptr;
      if ((rc = run_small_batch(sb, a.stream, ev)) != MOE_OK) return rc;
      if ((rc = launch_combine(false, ws + L.yw, sb.flags, a.out, a.T, a.K, a.top_k, 1, nsm, a.stream)) != MOE_OK)
        return rc;
      if (ev && cudaEventRecord(static_cast<cudaEvent_t>(ev[3]), a.stream) != cudaSuccess)
        return cuda_fail("fused_moe: cudaEventRecord");
      return MOE_OK;
    }
  }

  CUtensorMap tm_w1, tm_w2, tm_w2x, tm_act, tm_actx;
  const TmapKind wk = a.w_fp4 ? kTmFp4 : (a.fp8 ? kTmU8 : kTmBf16), ak = a.fp8 ? kTmU8 : kTmBf16;
  if ((rc = make_tmap(&tm_w1, a.w1, wk, static_cast<int64_t>(a.E) * a.N, a.K, 128)) != MOE_OK) return rc;
  if ((rc = make_tmap(&tm_w2, a.w2, wk, static_cast<int64_t>(a.E) * a.K, I, 128)) != MOE_OK) return rc;
  if ((rc = make_tmap(&tm_act, ws + L.act, ak, L.cap_rows, I, 16)) != MOE_OK) return rc;
  // the one-box forms are encoded only where the down phase can use them
  // (full 256-feature tiles; 128-row A regions)
  tm_w2x = tm_w2;
  tm_actx = tm_act;
  const int a_rows = a_region_rows(a.bm, static_cast<int64_t>(a.T) * a.top_k);
  if (a.K >= 2 * 128 && (rc = make_tmap(&tm_w2x, a.w2, wk, static_cast<int64_t>(a.E) * a.K, I, 256)) != MOE_OK)
    return rc;
  if (a_rows >= kM && (rc = make_tmap(&tm_actx, ws + L.act, ak, L.cap_rows, I, 128)) != MOE_OK) return rc;

  const int req_stages = a.tune ? a.tune->stages : 0;
  const int req_ctas = a.tune ? a.tune->num_ctas : 0;

  P1Params p1{};
  p1.x = static_cast<const uint8_t*>(a.x);
  p1.x_sf = a.x_sf;
  p1.w1_sf = a.w1_sf;
  p1.sorted_ids = a.sorted_ids;
  p1.expert_ids = a.expert_ids;
  p1.ntpp = a.ntpp;
  p1.act = ws + L.act;
  p1.act_sf = ws + L.act_sf;
  p1.flags = reinterpret_cast<int32_t*>(ws + L.flags);
  p1.part = reinterpret_cast<float*>(ws + L.part);
  p1.status = status;
  p1.K = a.K; p1.N = a.N; p1.I = I; p1.E = a.E; p1.top_k = a.top_k; p1.bm = a.bm;
  p1.R = a.T * a.top_k;
  p1.max_blocks = max_blocks;
  p1.w_reuse = static_cast<int64_t>(a.T) * a.top_k >= static_cast<int64_t>(a.E) * a.bm ? 1 : 0;
  p1.w_fp4 = a.w_fp4 ? 1 : 0;
  p1.n_jt = (I + kTI - 1) / kTI;
  p1.stage_bytes = stage_bytes(a.fp8, a_rows);
  p1.off_b = off_b_of(a_rows);
  p1.off_sf = off_sf_of(a_rows);
  p1.stages = pick_stages(p1.stage_bytes, kP1Ctrl, req_stages, kMaxStages);
  p1.wait_ns = wait_ns;
  {
    // L2 prefetch (see P1Params): the whole expert set when it is small, else
    // the down phase's touched w2 tiles when they are
    const int64_t wb1 = static_cast<int64_t>(a.E) * a.N * a.K * (a.fp8 ? 1 : 2) / (a.w_fp4 ? 2 : 1);
    const int64_t wb2 = static_cast<int64_t>(a.E) * a.K * I * (a.fp8 ? 1 : 2) / (a.w_fp4 ? 2 : 1);
    const int64_t sb1 = a.fp8 ? pack_scales_blocked_bytes(a.E, a.N, a.K / 32) : 0;
    const int64_t sb2 = a.fp8 ? pack_scales_blocked_bytes(a.E, a.K, I / 32) : 0;
    p1.pf_all = wb1 + wb2 + sb1 + sb2 <= kPrefetchAllBytes ? 1 : 0;
    p1.pf_src[0] = static_cast<const uint8_t*>(a.w1); p1.pf_bytes[0] = wb1;
    p1.pf_src[1] = static_cast<const uint8_t*>(a.w2); p1.pf_bytes[1] = wb2;
    p1.pf_src[2] = a.w1_sf; p1.pf_bytes[2] = a.w1_sf ? sb1 : 0;
    p1.pf_src[3] = a.w2_sf; p1.pf_bytes[3] = a.w2_sf ? sb2 : 0;
    p1.w2 = static_cast<const uint8_t*>(a.w2);
    p1.w2_sf = a.fp8 ? a.w2_sf : nullptr;
    p1.w2_row_bytes = static_cast<int64_t>(I) * (a.fp8 ? 1 : 2) / (a.w_fp4 ? 2 : 1);
    p1.pf_w2_budget = kPrefetchW2Bytes;
  }

  P2Params p2{};
  p2.w2_sf = a.w2_sf;
  p2.act_sf = ws + L.act_sf;
  p2.sorted_ids = a.sorted_ids;
  p2.expert_ids = a.expert_ids;
  p2.ntpp = a.ntpp;
  p2.topk_w = a.topk_w;
  p2.yw = ws + L.yw;
  p2.flags = p1.flags;
  p2.status = p1.status;
  p2.K = a.K; p2.I = I; p2.E = a.E; p2.top_k = a.top_k; p2.bm = a.bm; p2.R = p1.R;
  p2.max_blocks = max_blocks;
  p2.w_reuse = p1.w_reuse;
  p2.w_fp4 = p1.w_fp4;
  p2.n_ht = (a.K + kTH - 1) / kTH;
  p2.n_kc = a.fp8 ? I / 128 : (I + 63) / 64;
  p2.nsplit2 = down_splits(a.fp8, a.T, a.K, a.N, a.E, a.top_k, a.bm);
  p2.stage_bytes = stage_bytes(a.fp8, a_rows);
  p2.off_b = p1.off_b;
  p2.a_full = a_rows >= kM ? 1 : 0;
  p2.off_sf = p1.off_sf;
  p2.stages = pick_stages(p2.stage_bytes, kP2Ctrl + kP2Staging, req_stages, kMaxStages);
  p2.wait_ns = wait_ns;
  if (p1.stages < 2 || p2.stages < 2) return fail(MOE_ERR_UNSUPPORTED, "%s: shared memory too small", nm);

  const int64_t units1 = static_cast<int64_t>(max_blocks) * p1.n_jt;
  const int64_t units2 = static_cast<int64_t>(max_blocks) * p2.n_ht * p2.nsplit2;
  int ctas = req_ctas > 0 ? req_ctas : nsm;
  // one CTA per SM: small problems split their units' K range over the CTAs
  const int grid1 = ctas;
  (void)units1;
  const int grid2 = static_cast<int>(units2 < ctas ? units2 : ctas);
  // Each CTA allocates all 512 TMEM columns: request more than half of the
  // shared memory so that two CTAs never share an SM.
  const int smem1 = std::max(1024 + p1.stages * p1.stage_bytes + kP1Ctrl, kSmemLimit / 2 + 1024);
  const int smem2 = std::max(1024 + p2.stages * p2.stage_bytes + kP2Ctrl + kP2Staging, kSmemLimit / 2 + 1024);

  void* const* ev = a.tune ? a.tune->phase_events : nullptr;
  auto mark = [&](int i) -> int {
    if (ev && cudaEventRecord(static_cast<cudaEvent_t>(ev[i]), a.stream) != cudaSuccess)
      return cuda_fail("fused_moe: cudaEventRecord");
    return MOE_OK;
  };
  static std::atomic<bool> attr_done[4][kMaxDevices];
  if (a.fp8) {
    if ((rc = set_smem_attr(moe_p1_kernel<true>, smem1, attr_done[0])) != MOE_OK) return rc;
    if ((rc = set_smem_attr(moe_p2_kernel<true>, smem2, attr_done[1])) != MOE_OK) return rc;
  } else {
    if ((rc = set_smem_attr(moe_p1_kernel<false>, smem1, attr_done[2])) != MOE_OK) return rc;
    if ((rc = set_smem_attr(moe_p2_kernel<false>, smem2, attr_done[3])) != MOE_OK) return rc;
  }
  // The four launches are chained by programmatic dependent launch: each
  // kernel lets the next one be scheduled early (prologue: barriers, TMEM,
  // tensor-map prefetch) and the next one waits (griddepcontrol.wait) before
  // reading the previous one's results.
  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;
  auto config = [&](int grid, int threads, int smem) {
    cudaLaunchConfig_t c = {};
    c.gridDim = dim3(grid, 1, 1);
    c.blockDim = dim3(threads, 1, 1);
    c.dynamicSmemBytes = smem;
    c.stream = a.stream;
    c.attrs = pdl;
    c.numAttrs = 1;
    return c;
  };
  if ((rc = mark(0)) != MOE_OK) return rc;
  cudaLaunchConfig_t c1 = config(grid1, kP1Threads, smem1);
  cudaError_t err = a.fp8 ? cudaLaunchKernelEx(&c1, moe_p1_kernel<true>, tm_w1, p1)
                          : cudaLaunchKernelEx(&c1, moe_p1_kernel<false>, tm_w1, p1);
  if (err != cudaSuccess) return cuda_fail("fused_moe: gate/up phase launch", err);
  cudaLaunchConfig_t cr = config(nsm, 256, 0);
  err = a.fp8 ? cudaLaunchKernelEx(&cr, moe_p1_reduce_kernel<true>, p1, grid1)
              : cudaLaunchKernelEx(&cr, moe_p1_reduce_kernel<false>, p1, grid1);
  if (err != cudaSuccess) return cuda_fail("fused_moe: split-K reduction launch", err);
  if ((rc = mark(1)) != MOE_OK) return rc;
  cudaLaunchConfig_t c2 = config(grid2, kP2Threads, smem2);
  err = a.fp8 ? cudaLaunchKernelEx(&c2, moe_p2_kernel<true>, tm_w2, tm_w2x, tm_act, tm_actx, p2)
              : cudaLaunchKernelEx(&c2, moe_p2_kernel<false>, tm_w2, tm_w2x, tm_act, tm_actx, p2);
  if (err != cudaSuccess) return cuda_fail("fused_moe: down phase launch", err);
  if ((rc = mark(2)) != MOE_OK) return rc;
  if ((rc = launch_combine(a.fp8, ws + L.yw, static_cast<const int32_t*>(p1.flags), a.out, a.T, a.K, a.top_k,
                           p2.nsplit2, nsm, a.stream)) != MOE_OK)
    return rc;
  return mark(3);
}

}  // namespace moe

using namespace moe;

extern "C" int64_t moe_workspace_bytes(int dtype, int T, int K, int N, int E, int top_k, int block_m) {
  if (T < 0 || K <= 0 || N <= 0 || E < 1 || top_k < 1 || !valid_block_m(block_m)) return -1;
  if (dtype != MOE_DTYPE_BF16 && dtype != MOE_DTYPE_MXFP8 && dtype != MOE_DTYPE_MXFP4) return -1;
  return ws_layout(dtype != MOE_DTYPE_BF16, T, K, N, E, top_k, block_m).total;
}

extern "C" int moe_device_status(moe_stream_t stream) {
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return cuda_fail("moe_device_status: cudaStreamSynchronize");
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_moe_status, sizeof(int)) != cudaSuccess)
    return cuda_fail("moe_device_status: read");
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_moe_status, &zero, sizeof(int)) != cudaSuccess)
      return cuda_fail("moe_device_status: clear");
    return fail(v, "a device-side wait timed out");
  }
  return MOE_OK;
}

extern "C" int fused_moe_bf16(const void* x, const void* w1, const void* w2, const int32_t* sorted_token_ids,
                              const int32_t* expert_ids, const int32_t* num_tokens_post_padded,
                              const float* topk_weights, void* out, int T, int K, int N, int E, int top_k,
                              int block_m, int64_t capacity, void* workspace, int64_t workspace_bytes,
                              const moe_tuning* tune, moe_stream_t stream) {
  FusedArgs a{};
  a.fp8 = false;
  a.x = x; a.w1 = w1; a.w2 = w2;
  a.sorted_ids = sorted_token_ids; a.expert_ids = expert_ids; a.ntpp = num_tokens_post_padded;
  a.topk_w = topk_weights; a.out = out;
  a.T = T; a.K = K; a.N = N; a.E = E; a.top_k = top_k; a.bm = block_m; a.capacity = capacity;
  a.ws = workspace; a.ws_bytes = workspace_bytes; a.tune = tune;
  a.stream = reinterpret_cast<cudaStream_t>(stream);
  return run_fused(a);
}

extern "C" int fused_moe_mxfp8(const uint8_t* x_e4m3, const uint8_t* x_scales, const uint8_t* w1_e4m3,
                               const uint8_t* w1_scales_blocked, const uint8_t* w2_e4m3,
                               const uint8_t* w2_scales_blocked, const int32_t* sorted_token_ids,
                               const int32_t* expert_ids, const int32_t* num_tokens_post_padded,
                               const float* topk_weights, void* out, int T, int K, int N, int E, int top_k,
                               int block_m, int64_t capacity, void* workspace, int64_t workspace_bytes,
                               const moe_tuning* tune, moe_stream_t stream) {
  FusedArgs a{};
  a.fp8 = true;
  a.x = x_e4m3; a.x_sf = x_scales; a.w1 = w1_e4m3; a.w1_sf = w1_scales_blocked;
  a.w2 = w2_e4m3; a.w2_sf = w2_scales_blocked;
  a.sorted_ids = sorted_token_ids; a.expert_ids = expert_ids; a.ntpp = num_tokens_post_padded;
  a.topk_w = topk_weights; a.out = out;
  a.T = T; a.K = K; a.N = N; a.E = E; a.top_k = top_k; a.bm = block_m; a.capacity = capacity;
  a.ws = workspace; a.ws_bytes = workspace_bytes; a.tune = tune;
  a.stream = reinterpret_cast<cudaStream_t>(stream);
  return run_fused(a);
}

extern "C" int fused_moe_mxfp4(const uint8_t* x_e4m3, const uint8_t* x_scales, const uint8_t* w1_e2m1,
                               const uint8_t* w1_scales_blocked, const uint8_t* w2_e2m1,
                               const uint8_t* w2_scales_blocked, const int32_t* sorted_token_ids,
                               const int32_t* expert_ids, const int32_t* num_tokens_post_padded,
                               const float* topk_weights, void* out, int T, int K, int N, int E, int top_k,
                               int block_m, int64_t capacity, void* workspace, int64_t workspace_bytes,
                               const moe_tuning* tune, moe_stream_t stream) {
  FusedArgs a{};
  a.fp8 = true;
  a.w_fp4 = true;
  a.x = x_e4m3; a.x_sf = x_scales; a.w1 = w1_e2m1; a.w1_sf = w1_scales_blocked;
  a.w2 = w2_e2m1; a.w2_sf = w2_scales_blocked;
  a.sorted_ids = sorted_token_ids; a.expert_ids = expert_ids; a.ntpp = num_tokens_post_padded;
  a.topk_w = topk_weights; a.out = out;
  a.T = T; a.K = K; a.N = N; a.E = E; a.top_k = top_k; a.bm = block_m; a.capacity = capacity;
  a.ws = workspace; a.ws_bytes = workspace_bytes; a.tune = tune;
  a.stream = reinterpret_cast<cudaStream_t>(stream);
  return run_fused(a);
}

// ========================================================================
// fused_moe_bf16_noalloc: the bf16 forward with a library-owned workspace
// ========================================================================
namespace moe {

// Some callers cannot allocate device memory for the workspace: a plain C
// host program that links only this library and has no allocator of its
// own, or an application whose memory pool owns every byte of the device
// and forbids extra cudaMalloc calls.  For them the workspace lives in this
// file-scope array, which every device that loads the library keeps for the
// life of the process.
constexpr int64_t kNoAllocScratchBytes = int64_t(MOE_NOALLOC_SCRATCH_BYTES);
static __device__ __align__(256) uint8_t g_noalloc_scratch[MOE_NOALLOC_SCRATCH_BYTES];

// Device address of g_noalloc_scratch, looked up once per device (host code
// cannot use the array's name as a device pointer).
static int noalloc_scratch(void** out) {
  static void* addr[kMaxDevices] = {};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cuda_fail("fused_moe_bf16_noalloc: cudaGetDevice");
  if (dev >= kMaxDevices) return fail(MOE_ERR_UNSUPPORTED, "fused_moe_bf16_noalloc: device index %d too large", dev);
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    const cudaError_t err = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (err != cudaSuccess) return cuda_fail("fused_moe_bf16_noalloc: cudaGetSymbolAddress", err);
    addr[dev] = p;
  }
  *out = addr[dev];
  return MOE_OK;
}

}  // namespace moe

extern "C" int64_t fused_moe_bf16_noalloc_max_workspace(void) { return moe::kNoAllocScratchBytes; }

extern "C" int fused_moe_bf16_noalloc(const void* x, const void* w1, const void* w2,
                                      const int32_t* sorted_token_ids, const int32_t* expert_ids,
                                      const int32_t* num_tokens_post_padded, const float* topk_weights, void* out,
                                      int T, int K, int N, int E, int top_k, int block_m, int64_t capacity,
                                      const moe_tuning* tune, moe_stream_t stream) {
  // The same argument checks, and so the same status codes, as fused_moe_bf16;
  // only then the size limit of the built-in scratch.
  moe::FusedArgs a{};
  a.x = x; a.w1 = w1; a.w2 = w2;
  a.sorted_ids = sorted_token_ids; a.expert_ids = expert_ids; a.ntpp = num_tokens_post_padded;
  a.topk_w = topk_weights; a.out = out;
  a.T = T; a.K = K; a.N = N; a.E = E; a.top_k = top_k; a.bm = block_m; a.capacity = capacity;
  const int rc0 = moe::check_fused(a, false);
  if (rc0 != MOE_OK || T == 0) return rc0;
  const int64_t need = moe_workspace_bytes(MOE_DTYPE_BF16, T, K, N, E, top_k, block_m);
  if (need > moe::kNoAllocScratchBytes)
    return moe::fail(MOE_ERR_WORKSPACE,
                     "fused_moe_bf16_noalloc: this problem needs %lld bytes of workspace, more than the %lld-byte "
                     "built-in scratch; use fused_moe_bf16 with a caller-allocated workspace",
                     (long long)need, (long long)moe::kNoAllocScratchBytes);
  void* ws = nullptr;
  const int rc = moe::noalloc_scratch(&ws);
  if (rc != MOE_OK) return rc;
  return fused_moe_bf16(x, w1, w2, sorted_token_ids, expert_ids, num_tokens_post_padded, topk_weights, out, T, K, N,
                        E, top_k, block_m, capacity, ws, moe::kNoAllocScratchBytes, tune, stream);
}
