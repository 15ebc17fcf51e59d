// Top-k block selection: one warp per (query, group).
//
// MSA pull request "Add MiniMax-M3 (MSA) support": block scores plus the
// local bias are ranked together for top-k (section "Implementation"); the
// number kept is min(indexer_top_k, n_blocks) (RADV review comment).  Ties
// rank the lower block index first.
//
// Every visible block gets a unique 64-bit key: the float32 score mapped to
// an order-preserving unsigned integer in the high word, the complemented
// block index in the low word.  One unsigned compare then orders by score
// descending and index ascending, exactly.  Lane l owns the blocks l + 32 j
// and holds their keys in registers.
//
// With at most 16 visible blocks all of them are kept.  With more, the top
// 16 are found in one pass: the 16th largest of the 32 lanes' best keys
// bounds the 16th largest key from below; the keys at or above it
// (typically about 20) are compacted into shared memory in ascending block
// order with one ballot per column, each is ranked against the others by
// broadcast reads, and a chosen key's place in the ascending output is a
// ballot count.  When more than 32 keys pass the bound, k exact rounds run
// instead: round r takes the warp maximum of the lanes' best keys (two
// 32-bit warp reductions: the high words, then the low words of the lanes
// that hold the highest high word), the r-th ranked block; only the lane
// that owned it needs a new best, which the warp finds among that lane's
// keys (now in shared memory) in parallel.  Above 1024 blocks the keys are
// re-read from global memory every round.
#pragma once

#include "msa_common.cuh"

namespace msa {
namespace sel {

constexpr int kBlock = 128;
constexpr int kTopK = 16;

__device__ __forceinline__ uint32_t ordered_bits(float v) {
  if (v != v) v = -INFINITY;  // NaN ranks as -inf
  if (v == 0.0f) v = 0.0f;    // -0 and +0 are the same score
  const uint32_t u = __float_as_uint(v);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ uint64_t block_key(float v, int b) {
  return (static_cast<uint64_t>(ordered_bits(v)) << 32) |
         static_cast<uint64_t>(0xffffffffu - static_cast<uint32_t>(b));
}

// Largest 64-bit key over the warp: the largest high word, then the largest
// low word among the lanes holding it (keys are unique, so one lane holds it).
__device__ __forceinline__ uint64_t warp_max_key(uint64_t x) {
  const uint32_t hi = __reduce_max_sync(0xffffffffu, static_cast<uint32_t>(x >> 32));
  const uint32_t lo = __reduce_max_sync(0xffffffffu, static_cast<uint32_t>(x >> 32) == hi ? static_cast<uint32_t>(x) : 0u);
  return (static_cast<uint64_t>(hi) << 32) | lo;
}

// Shared memory of one warp's keys (kPerLane > 0): a padded row per lane,
// then 32 slots for the candidates of the threshold pass.
template <int kPerLane>
struct KeySmem {
  static constexpr int kStride = kPerLane + 1;
  static constexpr int kCandOff = 32 * kStride;
  static constexpr size_t kBytesPerWarp = (32 * kStride + 32) * sizeof(uint64_t);
};

// The top kTopK keys when more than kTopK blocks are visible, without
// kTopK serial rounds.  x: this lane's keys (block lane + 32 j, 0 when not
// visible); best: the largest of them; cand: 32 slots of this warp's shared
// memory.  The kTopK-th largest of the 32 lanes' best keys, t, bounds the
// kTopK-th largest key from below (kTopK lanes each hold a key >= t), so the
// top keys are among those >= t.  They are compacted into cand column by
// column (one ballot per column), which leaves them in ascending block
// order, then each is ranked against the others by broadcast reads; a
// chosen key's place in the ascending output is then one ballot count.
// False, with nothing written, when more than 32 keys pass the bound (the
// caller then runs the exact rounds).
template <int kPerLane>
__device__ __forceinline__ bool select_by_threshold(const uint64_t (&x)[kPerLane], uint64_t best, int lane,
                                                    uint64_t* cand, int32_t* out) {
  const uint32_t lt = (1u << lane) - 1u;
  cand[lane] = best;
  __syncwarp();
  int rb = 0;
#pragma unroll
  for (int d = 0; d < 32; ++d) rb += cand[d] > best ? 1 : 0;
  __syncwarp();
  const int tl = __ffs(__ballot_sync(0xffffffffu, rb == kTopK - 1)) - 1;
  const uint64_t t = __shfl_sync(0xffffffffu, best, tl);
  int total = 0;
#pragma unroll
  for (int j = 0; j < kPerLane; ++j) {
    const bool pass = x[j] >= t;
    const uint32_t m = __ballot_sync(0xffffffffu, pass);
    const int slot = total + __popc(m & lt);
    if (pass && slot < 32) cand[slot] = x[j];
    total += __popc(m);
  }
  __syncwarp();
  if (total > 32) return false;
  const uint64_t c = lane < total ? cand[lane] : 0ull;
  int rc = 0;
  for (int d = 0; d < total; ++d) rc += cand[d] > c ? 1 : 0;
  const bool chosen = lane < total && rc < kTopK;
  const int pos = __popc(__ballot_sync(0xffffffffu, chosen) & lt);
  if (chosen) out[pos] = static_cast<int>(0xffffffffu - static_cast<uint32_t>(c));
  __syncwarp();
  return true;
}

// The top-k of (query, group) pair `wid` into `out` (k ids, ascending, -1
// padded to kTopK) and its count into *count (nullable).
// kPerLane > 0: at most 32 * kPerLane visible blocks, keys in `wsm` (this
// warp's KeySmem<kPerLane>::kBytesPerWarp bytes of shared memory);
// kPerLane == 0: any count, re-read from global memory each round.
template <int kPerLane>
__device__ __forceinline__ void select_pair(const float* __restrict__ bs, const int32_t* __restrict__ q_pos,
                                            int G, int nblk, int capacity, int32_t* out, int32_t* count, int wid,
                                            int lane, uint64_t* wsm) {
  const int qi = wid / G;
  const float* row = bs + static_cast<size_t>(wid) * nblk;
  // the row's scores are requested before the query position arrives (the
  // two round trips overlap); blocks past the position are masked after
  float v[kPerLane > 0 ? kPerLane : 1];
  if constexpr (kPerLane > 0) {
#pragma unroll
    for (int j = 0; j < kPerLane; ++j) {
      const int b = lane + 32 * j;
      v[j] = b < nblk ? __ldcg(row + b) : 0.f;
    }
  }
  const int p = q_pos[qi];
  if (p < 0 || p >= capacity) {
    if (lane < kTopK) out[lane] = -1;
    if (lane == 0) {
      if (count != nullptr) *count = 0;
      if (wid % G == 0) raise_error(MSA_DEVERR_QUERY_RANGE);
    }
    return;
  }
  const int nvis = p / kBlock + 1;
  const int k = min(kTopK, nvis);
  if (nvis <= kTopK) {                              // every visible block is kept
    if (lane < kTopK) out[lane] = lane < nvis ? lane : -1;
    if (lane == 0 && count != nullptr) *count = nvis;
    return;
  }
  int my_id = -1;

  if constexpr (kPerLane > 0) {
    constexpr int kStride = KeySmem<kPerLane>::kStride;
    uint64_t x[kPerLane];
    uint64_t best = 0ull;                          // every real key is > 0
#pragma unroll
    for (int j = 0; j < kPerLane; ++j) {
      const int b = lane + 32 * j;
      x[j] = b < nvis ? block_key(v[j], b) : 0ull;
      best = x[j] > best ? x[j] : best;
    }
    if (select_by_threshold<kPerLane>(x, best, lane, wsm + KeySmem<kPerLane>::kCandOff, out)) {
      if (lane == 0 && count != nullptr) *count = kTopK;
      return;
    }
    // more than 32 keys at or above the bound: k exact rounds over the keys
#pragma unroll
    for (int j = 0; j < kPerLane; ++j) wsm[lane * kStride + j] = x[j];
    __syncwarp();
    for (int r = 0; r < k; ++r) {
      const uint64_t win = warp_max_key(best);
      const int b = static_cast<int>(0xffffffffu - static_cast<uint32_t>(win));
      if (lane == r) my_id = b;
      // the owner of the winner (lane b % 32) takes its largest key below it
      const int owner = b & 31;
      uint64_t y = 0ull;
      if (lane < kPerLane) {
        y = wsm[owner * kStride + lane];
        if (y >= win) y = 0ull;
      }
      const uint64_t next = warp_max_key(y);
      if (lane == owner) best = next;
    }
    __syncwarp();
  } else {
    uint64_t prev = ~0ull;
    for (int r = 0; r < k; ++r) {
      uint64_t best = 0ull;
      for (int b = lane; b < nvis; b += 32) {
        const uint64_t y = block_key(__ldcg(row + b), b);
        if (y < prev && y > best) best = y;
      }
      best = warp_max_key(best);
      prev = best;
      if (lane == r) my_id = static_cast<int>(0xffffffffu - static_cast<uint32_t>(best));
    }
  }

  int rank = 0;
#pragma unroll
  for (int j = 0; j < kTopK; ++j) {
    const int other = __shfl_sync(0xffffffffu, my_id, j);
    if (j < k && other < my_id) ++rank;
  }
  if (lane < k) {
    out[rank] = my_id;
  } else if (lane < kTopK) {
    out[lane] = -1;
  }
  if (lane == 0 && count != nullptr) *count = k;
}


// One warp per (query, group); dynamic shared memory: the warps' key rows.
template <int kPerLane>
__global__ void __launch_bounds__(256) select_topk_kernel(const float* __restrict__ bs,
                                                          const int32_t* __restrict__ q_pos,
                                                          int n_q, int G, int nblk, int capacity,
                                                          int32_t* __restrict__ sel,
                                                          int32_t* __restrict__ n_sel) {
  extern __shared__ uint64_t key_smem[];
  pdl_trigger();
  pdl_wait();
  const int wid = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (wid >= n_q * G) return;
  uint64_t* wsm = kPerLane > 0 ? key_smem + (threadIdx.x >> 5) * (KeySmem<kPerLane>::kBytesPerWarp / 8) : nullptr;
  select_pair<kPerLane>(bs, q_pos, G, nblk, capacity, sel + static_cast<size_t>(wid) * kTopK,
                        n_sel != nullptr ? n_sel + wid : nullptr, wid, threadIdx.x & 31, wsm);
}

// The warp count of a select_topk_kernel block and its dynamic shared memory.
template <int kPerLane>
struct SelectLaunch {
  static constexpr int kThreads = kPerLane > 16 ? 128 : 256;
  static constexpr size_t kSmem = kPerLane > 0 ? (kThreads / 32) * KeySmem<kPerLane>::kBytesPerWarp : 0;
};

// Shared memory one warp of select_pair_any needs for `nblk` blocks.
__host__ __device__ constexpr size_t select_smem_per_warp(int nblk) {
  return nblk <= 32 * 8 ? KeySmem<8>::kBytesPerWarp : (nblk <= 32 * 32 ? KeySmem<32>::kBytesPerWarp : 0);
}

// The same for any block count, choosing the shared-memory variant when the
// keys fit; wsm: select_smem_per_warp(nblk) bytes of this warp's shared memory.
__device__ __forceinline__ void select_pair_any(const float* bs, const int32_t* q_pos, int G, int nblk,
                                                int capacity, int32_t* out, int32_t* count, int wid, int lane,
                                                uint64_t* wsm) {
  if (nblk <= 32 * 8) {
    select_pair<8>(bs, q_pos, G, nblk, capacity, out, count, wid, lane, wsm);
  } else if (nblk <= 32 * 32) {
    select_pair<32>(bs, q_pos, G, nblk, capacity, out, count, wid, lane, wsm);
  } else {
    select_pair<0>(bs, q_pos, G, nblk, capacity, out, count, wid, lane, wsm);
  }
}

}  // namespace sel
}  // namespace msa
