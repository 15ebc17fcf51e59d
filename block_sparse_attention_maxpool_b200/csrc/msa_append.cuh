// Cache append: copies new tokens' rows into a [S][G][cap][row] cache, or
// into the page its block table names for a paged cache.  Used for the F32
// indexer-key cache (row = 128 floats = 512 B) and the bf16 K/V caches
// (row = 128 bf16 = 256 B).  Pure data movement: one warp per (token, group)
// row, 16-byte vector loads and stores.
#pragma once

#include <cuda_fp16.h>

#include "msa_common.cuh"

namespace msa {

// One (token, group) row: warp `warp` of the n_tok * n_groups rows.
// rows_bytes: bytes of one row (a multiple of 16, at most 512).  Up to two
// caches (K and V) are written at once; cache1/src1 may be null.
__device__ __forceinline__ void append_row(uint8_t* __restrict__ cache0, const uint8_t* __restrict__ src0,
                                           uint8_t* __restrict__ cache1, const uint8_t* __restrict__ src1,
                                           const int32_t* __restrict__ tok_stream,
                                           const int32_t* __restrict__ tok_pos, int n_streams, int n_groups,
                                           int capacity, int row_bytes, const KvPages& pages, int warp, int lane) {
  const int t = warp / n_groups;
  const int g = warp - t * n_groups;
  const int s = tok_stream[t];
  const int p = tok_pos[t];
  if (s < 0 || s >= n_streams || p < 0 || p >= capacity) {
    if (g == 0 && lane == 0) raise_error(MSA_DEVERR_TOKEN_RANGE);
    return;
  }
  const long long blk = kv_block_row(pages, s, g, p / 128, n_groups, capacity);
  if (blk < 0) {
    if (lane == 0) raise_error(MSA_DEVERR_PAGE_RANGE);
    return;
  }
  const size_t dst_row = static_cast<size_t>(blk) + (p & 127);
  const size_t src_row = static_cast<size_t>(t) * n_groups + g;
  const int vecs = row_bytes >> 4;
  if (lane < vecs) {
    const int4* a = reinterpret_cast<const int4*>(src0 + src_row * row_bytes) + lane;
    int4* b = reinterpret_cast<int4*>(cache0 + dst_row * row_bytes) + lane;
    *b = __ldg(a);
    if (cache1 != nullptr) {
      const int4* c = reinterpret_cast<const int4*>(src1 + src_row * row_bytes) + lane;
      int4* d = reinterpret_cast<int4*>(cache1 + dst_row * row_bytes) + lane;
      *d = __ldg(c);
    }
  }
}

__global__ void __launch_bounds__(256) append_rows_kernel(
    uint8_t* __restrict__ cache0, const uint8_t* __restrict__ src0, uint8_t* __restrict__ cache1,
    const uint8_t* __restrict__ src1, const int32_t* __restrict__ tok_stream,
    const int32_t* __restrict__ tok_pos, int n_tok, int n_streams, int n_groups, int capacity,
    int row_bytes, const KvPages pages) {
  pdl_trigger();
  pdl_wait();
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (warp >= n_tok * n_groups) return;
  append_row(cache0, src0, cache1, src1, tok_stream, tok_pos, n_streams, n_groups, capacity, row_bytes, pages,
             warp, threadIdx.x & 31);
}

// All of a step's appends in one launch: one warp per (token, group) writes
// the F32 indexer key (512 B, one 16-byte vector per lane), then the K row
// (lanes 0-15) and the V row (lanes 16-31), 256 B each, at the slot the
// separate appends use, with the same checks and error bits.
__global__ void __launch_bounds__(256) append_step_kernel(
    float* __restrict__ idx_cache, const float* __restrict__ idx_src, uint8_t* __restrict__ k_cache,
    const uint8_t* __restrict__ k_src, uint8_t* __restrict__ v_cache, const uint8_t* __restrict__ v_src,
    const int32_t* __restrict__ tok_stream, const int32_t* __restrict__ tok_pos, int n_tok, int n_streams,
    int n_groups, int capacity, const KvPages pages) {
  pdl_trigger();
  pdl_wait();
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= n_tok * n_groups) return;
  const int t = warp / n_groups;
  const int g = warp - t * n_groups;
  const int s = tok_stream[t];
  const int p = tok_pos[t];
  if (s < 0 || s >= n_streams || p < 0 || p >= capacity) {
    if (g == 0 && lane == 0) raise_error(MSA_DEVERR_TOKEN_RANGE);
    return;
  }
  const long long blk = kv_block_row(pages, s, g, p / 128, n_groups, capacity);
  if (blk < 0) {
    if (lane == 0) raise_error(MSA_DEVERR_PAGE_RANGE);
    return;
  }
  const size_t dst_row = static_cast<size_t>(blk) + (p & 127);
  const size_t src_row = static_cast<size_t>(t) * n_groups + g;
  reinterpret_cast<int4*>(idx_cache + dst_row * 128)[lane] =
      __ldg(reinterpret_cast<const int4*>(idx_src + src_row * 128) + lane);
  const int h = lane & 15;
  uint8_t* cache = lane < 16 ? k_cache : v_cache;
  const uint8_t* src = lane < 16 ? k_src : v_src;
  reinterpret_cast<int4*>(cache + dst_row * 256)[h] = __ldg(reinterpret_cast<const int4*>(src + src_row * 256) + h);
}

// F16 indexer-key cache variant: each F32 key of 128 values is rounded to
// fp16 (nearest even) as it is written.  One warp per (token, group) row,
// four values per lane.
__global__ void __launch_bounds__(256) append_idx_f16_kernel(__half* __restrict__ cache,
                                                             const float* __restrict__ src,
                                                             const int32_t* __restrict__ tok_stream,
                                                             const int32_t* __restrict__ tok_pos, int n_tok,
                                                             int n_streams, int n_groups, int capacity,
                                                             const KvPages pages) {
  pdl_trigger();
  pdl_wait();
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= n_tok * n_groups) return;
  const int t = warp / n_groups;
  const int g = warp - t * n_groups;
  const int s = tok_stream[t];
  const int p = tok_pos[t];
  if (s < 0 || s >= n_streams || p < 0 || p >= capacity) {
    if (g == 0 && lane == 0) raise_error(MSA_DEVERR_TOKEN_RANGE);
    return;
  }
  const long long blk = kv_block_row(pages, s, g, p / 128, n_groups, capacity);
  if (blk < 0) {
    if (lane == 0) raise_error(MSA_DEVERR_PAGE_RANGE);
    return;
  }
  const float4 x = __ldg(reinterpret_cast<const float4*>(src + (static_cast<size_t>(t) * n_groups + g) * 128) + lane);
  const __half2 a = __floats2half2_rn(x.x, x.y);
  const __half2 b = __floats2half2_rn(x.z, x.w);
  uint2 out;
  out.x = *reinterpret_cast<const uint32_t*>(&a);
  out.y = *reinterpret_cast<const uint32_t*>(&b);
  *(reinterpret_cast<uint2*>(cache + (static_cast<size_t>(blk) + (p & 127)) * 128) + lane) = out;
}

}  // namespace msa
