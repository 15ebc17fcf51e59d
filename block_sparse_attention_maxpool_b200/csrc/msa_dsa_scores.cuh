// Token-level variant: lightning-indexer scores on the 5th-generation tensor
// cores.
//
// "deepseek2 : GLM-DSA sparse attention (lightning indexer)", section "What
// this does" and review thread: every query scores every visible token's
// indexer key (one F16 key per token) with each of its indexer heads; the
// per-head products are weighted per head and summed over the heads; the
// top-k tokens are kept.  Here
//   I[t][s] = sum_h w[t][h] * act(q[t][h] . k[s]),  act = ReLU or identity,
// for s <= q_pos[t], and -inf for s > q_pos[t].
//
// Per (query, 128-token key tile) the 64 heads x 128 keys products are one
// tcgen05 MMA chain: A = the key tile (M = 128 keys, K-major, 128-byte
// swizzle, two 64-column TMA boxes), B = the query's 64 head vectors (N = 64,
// K-major), 8 K-steps of 16, fp16 inputs (their products are exact in fp32)
// and fp32 accumulation in tensor memory.  Keys sit on the TMEM lanes, so
// each epilogue thread owns one key and reduces its 64 head columns in
// registers: no cross-thread reduction.  A decode query streams its keys
// once (8 MB per 32K context) and the MMAs need only a fraction of the
// tensor pipe's rate, so the kernel's bound is HBM.
//
// Warp roles (6 warps): 0 TMA producer (query tile per query, key tiles
// into a 2-stage ring), 1 MMA issuer (two 64-column accumulators), 2-5 the
// epilogue (one TMEM lane quarter each).  Two CTAs share each SM, so one
// CTA's per-tile handshakes (barrier waits, MMA commits, the epilogue's
// TMEM round trip) overlap the other's copies; a launch-shape sweep
// measured 46.8 us per 32-stream x 32K launch this way against 51.3 us with
// one CTA of four stages per SM.  Tasks (query, tile) are split into one
// contiguous range per CTA, tile fastest, walked by a cursor with no
// division per task, so a CTA keeps a query's head vectors for many tiles.
#pragma once

#include <cuda_fp16.h>

#include "msa_common.cuh"

namespace msa {
namespace dsa {

constexpr int kDi = 128;                       // indexer dim
constexpr int kHeads = 64;                     // indexer heads (MMA N)
constexpr int kTile = 128;                     // keys per tile (MMA M)
constexpr uint32_t kKeyHalf = kTile * 128;     // [128 rows][64 fp16] = 16 KB
constexpr uint32_t kKeyBytes = 2 * kKeyHalf;   // 32 KB
constexpr uint32_t kQHalf = kHeads * 128;      // [64 rows][64 fp16] = 8 KB
constexpr uint32_t kQBytes = 2 * kQHalf;       // 16 KB
constexpr int kStages = 2;
constexpr int kEpiGroups = 1;                  // epilogue groups of 4 warps (alternate tiles when > 1)
constexpr int kAccBufs = 2;                    // 64-column accumulators in tensor memory
constexpr int kCtasPerSm = 2;                  // two independent pipelines per SM
constexpr int kThreads = (2 + 4 * kEpiGroups) * 32;
constexpr uint32_t kTmemCols = kAccBufs * kHeads;
constexpr uint32_t kIdesc = umma_idesc_f16_f32(kTile, kHeads);

struct Smem {
  static constexpr uint32_t kKey = 0;                                // kStages key tiles
  static constexpr uint32_t kQ = kKey + kStages * kKeyBytes;        // 2 query tiles
  static constexpr uint32_t kBars = kQ + 2 * kQBytes;
  static constexpr uint32_t kEnd = kBars + 256;
  static constexpr size_t kBytes = kEnd + 1024;                     // + alignment slack
};
static_assert(Smem::kBytes <= 232448, "shared memory budget");

struct Params {
  const float* weights;      // [n_q][64]
  const int32_t* q_stream;
  const int32_t* q_pos;
  float* scores;             // [n_q][cap]
  int n_q, n_streams, capacity, n_tiles;   // n_tiles = capacity / 128
  int relu;
  KvPages pages;             // block table of a paged key cache (table null: contiguous [S][cap][128])
};

// Walks this CTA's tasks (query t, key tile kt) in order, tile fastest,
// without a division per task; the query's stream and position are read
// when t changes.  row: the tile's first cache row, or -1 when the tile has
// no data to score (past the query, an invalid query, an unmapped page).
struct TaskCursor {
  int t, kt, p, s;
  long long row;
  bool query_ok;
  __device__ __forceinline__ void load_query(const Params& P) {
    s = P.q_stream[t];
    p = P.q_pos[t];
    query_ok = s >= 0 && s < P.n_streams && p >= 0 && p < P.capacity;
  }
  __device__ __forceinline__ void resolve(const Params& P) {
    row = -1;
    if (query_ok && kt <= p / kTile) row = kv_block_row(P.pages, s, 0, kt, 1, P.capacity);
  }
  __device__ __forceinline__ void start(const Params& P, long long task) {
    t = static_cast<int>(task / P.n_tiles);
    kt = static_cast<int>(task - static_cast<long long>(t) * P.n_tiles);
    load_query(P);
    resolve(P);
  }
  __device__ __forceinline__ void next(const Params& P) {
    if (++kt == P.n_tiles) {
      kt = 0;
      ++t;
      load_query(P);
    }
    resolve(P);
  }
};

__global__ void __launch_bounds__(kThreads, kCtasPerSm)
    dsa_scores_kernel(const __grid_constant__ CUtensorMap tm_key, const __grid_constant__ CUtensorMap tm_q,
                      const Params P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Smem::kBars);
  uint64_t* full = bars;                          // [kStages] key tile landed
  uint64_t* empty = full + kStages;               // [kStages] MMAs done with the key tile
  uint64_t* q_full = empty + kStages;             // [2]
  uint64_t* q_empty = q_full + 2;                 // [2]
  uint64_t* acc_full = q_empty + 2;               // [kAccBufs]
  uint64_t* acc_empty = acc_full + kAccBufs;      // [kAccBufs]
  uint64_t* mma_done = acc_empty + kAccBufs;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  int* abort_flag = reinterpret_cast<int*>(mma_done + 2);
  static_assert((2 * kStages + 4 + 2 * kAccBufs + 3) * 8 <= Smem::kEnd - Smem::kBars, "barrier slots");

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const long long T = static_cast<long long>(P.n_q) * P.n_tiles;
  const long long t0 = T * blockIdx.x / gridDim.x;
  const long long t1 = T * (blockIdx.x + 1) / gridDim.x;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1);
    }
    for (int i = 0; i < kAccBufs; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 4);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, kTmemCols);
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  volatile int* abort_v = abort_flag;
  pdl_trigger();
  pdl_wait();

  if (warp == 0) {
    // ------------------------------ TMA producer ------------------------------
    if (lane == 0) {
      int kst = 0, q_use = 0, q_t = -1;
      TaskCursor I;
      for (long long task = t0; task < t1 && !*abort_v; ++task) {
        if (task == t0) I.start(P, task); else I.next(P);
        if (I.row < 0) continue;
        if (I.t != q_t) {                    // first scored tile of a query: its head vectors
          const int slot = q_use & 1;
          if (q_use >= 2 && !mbar_wait(&q_empty[slot], ((q_use >> 1) - 1) & 1)) { *abort_v = 1; break; }
          uint8_t* qd = smem + Smem::kQ + slot * kQBytes;
          mbar_arrive_expect_tx(&q_full[slot], kQBytes);
          tma_load_2d(qd, &tm_q, 0, I.t * kHeads, &q_full[slot]);
          tma_load_2d(qd + kQHalf, &tm_q, 64, I.t * kHeads, &q_full[slot]);
          q_t = I.t;
          ++q_use;
        }
        const int st = kst % kStages;
        const int use = kst / kStages;
        if (use > 0 && !mbar_wait(&empty[st], (use - 1) & 1)) { *abort_v = 1; break; }
        uint8_t* kd = smem + Smem::kKey + st * kKeyBytes;
        mbar_arrive_expect_tx(&full[st], kKeyBytes);
        tma_load_2d(kd, &tm_key, 0, static_cast<int>(I.row), &full[st]);
        tma_load_2d(kd + kKeyHalf, &tm_key, 64, static_cast<int>(I.row), &full[st]);
        ++kst;
      }
      // no copy may still be landing when the CTA exits
      for (int j = max(0, kst - kStages); j < kst; ++j) mbar_wait(&full[j % kStages], (j / kStages) & 1);
      for (int j = max(0, q_use - 2); j < q_use; ++j) mbar_wait(&q_full[j & 1], (j >> 1) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issuer --------------------------------
    if (lane == 0) {
      int kst = 0, q_use = 0, q_t = -1, acc = 0;
      TaskCursor I;
      for (long long task = t0; task < t1 && !*abort_v; ++task) {
        if (task == t0) I.start(P, task); else I.next(P);
        if (I.row < 0) continue;
        if (I.t != q_t) {
          if (q_use > 0) umma_commit(&q_empty[(q_use - 1) & 1]);   // previous query's vectors free
          if (!mbar_wait(&q_full[q_use & 1], (q_use >> 1) & 1)) { *abort_v = 1; break; }
          q_t = I.t;
          ++q_use;
        }
        const int st = kst % kStages;
        const int buf = acc % kAccBufs;
        if (!mbar_wait(&full[st], (kst / kStages) & 1)) { *abort_v = 1; break; }
        if (acc >= kAccBufs && !mbar_wait(&acc_empty[buf], ((acc / kAccBufs) - 1) & 1)) { *abort_v = 1; break; }
        tc_fence_after();
        const uint32_t a_base = smem_addr(smem + Smem::kKey + st * kKeyBytes);
        const uint32_t b_base = smem_addr(smem + Smem::kQ + ((q_use - 1) & 1) * kQBytes);
        const uint32_t d = tmem_base + static_cast<uint32_t>(buf * kHeads);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t a_off = (kk >> 2) * kKeyHalf + (kk & 3) * 32;
          const uint32_t b_off = (kk >> 2) * kQHalf + (kk & 3) * 32;
          umma_f16_ss(d, umma_desc_sw128(a_base + a_off), umma_desc_sw128(b_base + b_off), kIdesc, kk != 0);
        }
        umma_commit(&empty[st]);
        umma_commit(&acc_full[buf]);
        ++kst;
        ++acc;
      }
      umma_commit(mma_done);
      mbar_wait(mma_done, 0);
    }
  } else {
    // ------------------------- epilogue (kEpiGroups groups of 4 warps) -------
    const int quarter = warp & 3;                 // TMEM lane quarter this warp may read
    const int group = (warp - 2) >> 2;            // takes the scored tiles with acc % kEpiGroups == group
    const int r = quarter * 32 + lane;            // key within the tile
    float w[kHeads];
    int w_t = -1, acc = 0;
    bool ok = true;
    TaskCursor I;
    for (long long task = t0; task < t1; ++task) {
      if (task == t0) I.start(P, task); else I.next(P);
      float* out = P.scores + static_cast<size_t>(I.t) * P.capacity + static_cast<size_t>(I.kt) * kTile;
      if (I.row < 0) {
        if (group != 0) continue;
        out[r] = -INFINITY;
        if (r == 0) {
          if (!I.query_ok && I.kt == 0) raise_error(MSA_DEVERR_QUERY_RANGE);
          if (I.query_ok && I.kt <= I.p / kTile) raise_error(MSA_DEVERR_PAGE_RANGE);
        }
        continue;
      }
      const int mine = acc % kEpiGroups == group;
      if (!mine) {
        ++acc;
        continue;
      }
      if (I.t != w_t) {
        const float4* wp = reinterpret_cast<const float4*>(P.weights + static_cast<size_t>(I.t) * kHeads);
#pragma unroll
        for (int i = 0; i < kHeads / 4; ++i) {
          const float4 v = __ldg(wp + i);
          w[4 * i] = v.x;
          w[4 * i + 1] = v.y;
          w[4 * i + 2] = v.z;
          w[4 * i + 3] = v.w;
        }
        w_t = I.t;
      }
      const int buf = acc % kAccBufs;
      if (ok && !*abort_v) ok = mbar_wait(&acc_full[buf], (acc / kAccBufs) & 1);
      ok = __all_sync(0xffffffffu, ok);         // the TMEM loads below are warp-collective
      if (!ok) *abort_v = 1;
      tc_fence_after();
      float score = 0.f;
      if (ok) {
        float v[64];
        tmem_ld64(tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + buf * kHeads, v);
        tmem_ld_wait();
        // four interleaved chains over the heads (h mod 4), then their sum
        float part[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int h = 0; h < kHeads; ++h) {
          const float x = P.relu ? fmaxf(v[h], 0.f) : v[h];
          part[h & 3] = fmaf(w[h], x, part[h & 3]);
        }
        score = (part[0] + part[1]) + (part[2] + part[3]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[buf]);
      const int s = I.kt * kTile + r;
      out[r] = s <= I.p ? score : -INFINITY;
      ++acc;
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace dsa
}  // namespace msa
