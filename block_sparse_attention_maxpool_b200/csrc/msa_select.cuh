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
// and keeps its keys in shared memory and its best key in a register.
//
// With more than 16 visible blocks the top 16 are found in one pass: the
// 16th largest of the 32 lanes' best keys bounds the 16th largest key from
// below, the keys at or above it (typically about 20) are gathered and
// ranked against each other all at once (31 independent shuffles per lane),
// and the chosen ids are placed in ascending order the same way.  When more
// than 32 keys pass the bound, k exact rounds run instead: round r takes
// the warp maximum of the lanes' best keys (two 32-bit warp reductions: the
// high words, then the low words of the lanes that hold the highest high
// word), the r-th ranked block; only the lane that owned it needs a new
// best, which the warp finds among that lane's keys in parallel.  Above
// 1024 blocks the keys are re-read from global memory every round.
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

// Number of the warp's 32 values (one per lane, unique among the nonzero
// ones) that are larger than this lane's: 31 independent shuffles.
__device__ __forceinline__ int rank_in_warp(uint64_t x, int lane) {
  const uint32_t hi = static_cast<uint32_t>(x >> 32), lo = static_cast<uint32_t>(x);
  int r = 0;
#pragma unroll
  for (int d = 1; d < 32; ++d) {
    const int src = (lane + d) & 31;
    const uint32_t oh = __shfl_sync(0xffffffffu, hi, src);
    const uint32_t ol = __shfl_sync(0xffffffffu, lo, src);
    r += (oh > hi || (oh == hi && ol > lo)) ? 1 : 0;
  }
  return r;
}

// The top k = kTopK keys when more than kTopK blocks are visible, without
// k serial rounds: the kTopK-th largest of the lanes' best keys, T, is a
// lower bound of the kTopK-th largest key overall (kTopK lanes each hold a
// key >= T), so the top k are among the keys >= T.  Those candidates
// (typically about 20) are gathered into shared memory and ranked all at
// once, one per lane.  False, with nothing written, when there are more
// than 32 candidates; the caller then runs the exact rounds.
template <int kPerLane>
__device__ __forceinline__ bool select_by_threshold(uint64_t* wsm, uint64_t best, int lane, int32_t* out) {
  constexpr int kStride = KeySmem<kPerLane>::kStride;
  const int rb = rank_in_warp(best, lane);
  const int tl = __ffs(__ballot_sync(0xffffffffu, rb == kTopK - 1)) - 1;
  const uint64_t t = __shfl_sync(0xffffffffu, best, tl);
  int cnt = 0;
#pragma unroll
  for (int j = 0; j < kPerLane; ++j) cnt += wsm[lane * kStride + j] >= t ? 1 : 0;
  const int total = __reduce_add_sync(0xffffffffu, static_cast<unsigned>(cnt));
  if (total > 32) return false;
  int off = cnt;                                   // inclusive prefix of the counts
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const int o = __shfl_up_sync(0xffffffffu, off, d);
    if (lane >= d) off += o;
  }
  off -= cnt;
  uint64_t* cand = wsm + KeySmem<kPerLane>::kCandOff;
#pragma unroll
  for (int j = 0; j < kPerLane; ++j) {
    const uint64_t x = wsm[lane * kStride + j];
    if (x >= t) cand[off++] = x;
  }
  __syncwarp();
  const uint64_t c = lane < total ? cand[lane] : 0ull;
  __syncwarp();
  const int rc = rank_in_warp(c, lane);          // every lane: the shuffles take the whole warp
  const bool chosen = lane < total && rc < kTopK;
  // ascending block order: a chosen block's place is the number of chosen
  // blocks with a smaller index
  const int id = static_cast<int>(0xffffffffu - static_cast<uint32_t>(c));
  const int key = chosen ? id : 0x7fffffff;
  int pos = 0;
#pragma unroll
  for (int d = 1; d < 32; ++d) pos += __shfl_sync(0xffffffffu, key, (lane + d) & 31) < key ? 1 : 0;
  if (chosen) out[pos] = id;
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
  const float* row = bs + static_cast<size_t>(wid) * nblk;
  int my_id = -1;

  if constexpr (kPerLane > 0) {
    constexpr int kStride = KeySmem<kPerLane>::kStride;
    uint64_t best = 0ull;                          // every real key is > 0
    // all of this lane's scores in flight at once: with the shared-memory
    // stores in the same loop, the compiler (which cannot tell the two
    // pointers apart) would issue one load per store, each a full round trip
    float v[kPerLane];
#pragma unroll
    for (int j = 0; j < kPerLane; ++j) {
      const int b = lane + 32 * j;
      v[j] = b < nvis ? __ldcg(row + b) : 0.f;
    }
#pragma unroll
    for (int j = 0; j < kPerLane; ++j) {
      const int b = lane + 32 * j;
      const uint64_t x = b < nvis ? block_key(v[j], b) : 0ull;
      wsm[lane * kStride + j] = x;
      best = x > best ? x : best;
    }
    __syncwarp();
    if (nvis > kTopK && select_by_threshold<kPerLane>(wsm, best, lane, out)) {
      __syncwarp();
      if (lane == 0 && count != nullptr) *count = kTopK;
      return;
    }
    for (int r = 0; r < k; ++r) {
      const uint64_t win = warp_max_key(best);
      const int b = static_cast<int>(0xffffffffu - static_cast<uint32_t>(win));
      if (lane == r) my_id = b;
      // the owner of the winner (lane b % 32) takes its largest key below it
      const int owner = b & 31;
      uint64_t x = 0ull;
      if (lane < kPerLane) {
        x = wsm[owner * kStride + lane];
        if (x >= win) x = 0ull;
      }
      const uint64_t next = warp_max_key(x);
      if (lane == owner) best = next;
    }
    __syncwarp();
  } else {
    uint64_t prev = ~0ull;
    for (int r = 0; r < k; ++r) {
      uint64_t best = 0ull;
      for (int b = lane; b < nvis; b += 32) {
        const uint64_t x = block_key(__ldcg(row + b), b);
        if (x < prev && x > best) best = x;
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
