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
// descending and index ascending, exactly.  Round r finds the largest key
// below the one found in round r-1 (a warp max-reduction), so k rounds give
// the top-k in rank order; the k ids are then placed in ascending order with
// a 16-lane rank count.
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

__device__ __forceinline__ uint64_t warp_max_u64(uint64_t x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const uint64_t y = __shfl_xor_sync(0xffffffffu, x, o);
    x = y > x ? y : x;
  }
  return x;
}

// kPerLane > 0: the visible scores (at most 32 * kPerLane) are held in
// registers; kPerLane == 0: any count, re-read from global memory each round.
template <int kPerLane>
__device__ __forceinline__ void select_pair(const float* __restrict__ bs, const int32_t* __restrict__ q_pos,
                                            int G, int nblk, int capacity, int32_t* __restrict__ sel,
                                            int32_t* __restrict__ n_sel, int wid, int lane) {
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

  uint64_t keys[kPerLane > 0 ? kPerLane : 1];
  if constexpr (kPerLane > 0) {
#pragma unroll
    for (int j = 0; j < kPerLane; ++j) {
      const int b = lane + 32 * j;
      keys[j] = b < nvis ? block_key(__ldcg(row + b), b) : 0ull;
    }
  }

  uint64_t prev = ~0ull;
  int my_id = -1;
  for (int r = 0; r < k; ++r) {
    uint64_t best = 0ull;  // every real key is > 0
    if constexpr (kPerLane > 0) {
#pragma unroll
      for (int j = 0; j < kPerLane; ++j) {
        const uint64_t x = keys[j];
        if (x < prev && x > best) best = x;
      }
    } else {
      for (int b = lane; b < nvis; b += 32) {
        const uint64_t x = block_key(__ldcg(row + b), b);
        if (x < prev && x > best) best = x;
      }
    }
    best = warp_max_u64(best);
    prev = best;
    if (lane == r) my_id = static_cast<int>(0xffffffffu - static_cast<uint32_t>(best));
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


// One warp per (query, group).
template <int kPerLane>
__global__ void __launch_bounds__(256) select_topk_kernel(const float* __restrict__ bs,
                                                          const int32_t* __restrict__ q_pos,
                                                          int n_q, int G, int nblk, int capacity,
                                                          int32_t* __restrict__ sel,
                                                          int32_t* __restrict__ n_sel) {
  pdl_trigger();
  pdl_wait();
  const int wid = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (wid >= n_q * G) return;
  select_pair<kPerLane>(bs, q_pos, G, nblk, capacity, sel, n_sel, wid, threadIdx.x & 31);
}

// The same for any block count, choosing the register-held variant.
__device__ __forceinline__ void select_pair_any(const float* bs, const int32_t* q_pos, int G, int nblk,
                                                int capacity, int32_t* sel, int32_t* n_sel, int wid, int lane) {
  if (nblk <= 32 * 8) {
    select_pair<8>(bs, q_pos, G, nblk, capacity, sel, n_sel, wid, lane);
  } else if (nblk <= 32 * 32) {
    select_pair<32>(bs, q_pos, G, nblk, capacity, sel, n_sel, wid, lane);
  } else {
    select_pair<0>(bs, q_pos, G, nblk, capacity, sel, n_sel, wid, lane);
  }
}

}  // namespace sel
}  // namespace msa
