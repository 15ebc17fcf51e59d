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
// descending and index ascending, exactly.  Lane l owns the blocks l + 32 j;
// it keeps its keys in shared memory and its best remaining key in a
// register.  Round r takes the warp maximum of the lanes' best keys (two
// 32-bit warp reductions: the high words, then the low words of the lanes
// that hold the highest high word), which is the r-th ranked block; only the
// lane that owned it needs a new best, the largest of its keys below the
// winner, and the warp reads that lane's keys from shared memory in parallel
// (one per lane) and reduces them the same way.  k rounds give the top-k in
// rank order; the k ids are then placed in ascending order with a 16-lane
// rank count.  Above 1024 blocks the keys are re-read from global memory
// every round instead.
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

// Shared memory of one warp's keys (kPerLane > 0): a padded row per lane.
template <int kPerLane>
struct KeySmem {
  static constexpr int kStride = kPerLane + 1;
  static constexpr size_t kBytesPerWarp = 32 * kStride * sizeof(uint64_t);
};

// kPerLane > 0: at most 32 * kPerLane visible blocks, keys in `wsm` (this
// warp's KeySmem<kPerLane>::kBytesPerWarp bytes of shared memory);
// kPerLane == 0: any count, re-read from global memory each round.
template <int kPerLane>
__device__ __forceinline__ void select_pair(const float* __restrict__ bs, const int32_t* __restrict__ q_pos,
                                            int G, int nblk, int capacity, int32_t* __restrict__ sel,
                                            int32_t* __restrict__ n_sel, int wid, int lane, uint64_t* wsm) {
  const int qi = wid / G;
  const int p = q_pos[qi];
  int32_t* out = sel + static_cast<size_t>(wid) * kTopK;
  if (p < 0 || p >= capacity) {
    if (lane < kTopK) out[lane] = -1;
    if (lane == 0) {
      if (n_sel != nullptr) n_sel[wid] = 0;
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
#pragma unroll
    for (int j = 0; j < kPerLane; ++j) {
      const int b = lane + 32 * j;
      const uint64_t x = b < nvis ? block_key(__ldcg(row + b), b) : 0ull;
      wsm[lane * kStride + j] = x;
      best = x > best ? x : best;
    }
    __syncwarp();
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
  if (lane == 0 && n_sel != nullptr) n_sel[wid] = k;
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
  select_pair<kPerLane>(bs, q_pos, G, nblk, capacity, sel, n_sel, wid, threadIdx.x & 31, wsm);
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
                                                int capacity, int32_t* sel, int32_t* n_sel, int wid, int lane,
                                                uint64_t* wsm) {
  if (nblk <= 32 * 8) {
    select_pair<8>(bs, q_pos, G, nblk, capacity, sel, n_sel, wid, lane, wsm);
  } else if (nblk <= 32 * 32) {
    select_pair<32>(bs, q_pos, G, nblk, capacity, sel, n_sel, wid, lane, wsm);
  } else {
    select_pair<0>(bs, q_pos, G, nblk, capacity, sel, n_sel, wid, lane, wsm);
  }
}

}  // namespace sel
}  // namespace msa
