// Block scores for a few queries (decode): fused indexer GEMV + causal mask
// + max-pool over 128-slot blocks + local-force bias.
//
// MSA pull request "Add MiniMax-M3 (MSA) support", section "Implementation":
// bs = maxpool_128(idx_q * idx_k^T + causal mask) plus a large bias on the
// query's local block; scores accumulate in F32 (MSA branch commit message).
//
// The work is HBM-bound: every visible indexer key (128 f32 = 512 B) is read
// once and feeds 128 FMAs.  The task space is (query, group, block); a
// persistent grid gives each CTA one contiguous range of tasks, so a CTA
// streams long runs of one (stream, group) cache region.  One producer
// thread moves 32 KB chunks (64 key rows) into a ring of shared-memory
// stages with cp.async.bulk (evict-first L2 policy); eight consumer warps
// each take 8 rows of a chunk (one 16-byte load per lane per row, so a row
// is one conflict-free 512-byte shared-memory read) and reduce the 8 partial
// dot products across the warp with a transposed butterfly (9 shuffles for
// 8 rows).  Rows past the query position are masked, the per-block maximum
// is combined across warps and the local block gets MSA_LOCAL_BIAS.
#pragma once

#include <cuda_fp16.h>

#include "msa_common.cuh"

namespace msa {
namespace gemv {

constexpr int kDi = 128;                                 // indexer dim
constexpr int kBlock = 128;                              // key block
constexpr uint32_t kStageBytes = 32 * 1024;              // one chunk of key rows
constexpr int kConsumerWarps = 8;
constexpr int kThreads = (kConsumerWarps + 1) * 32;

// KeyT: float (the F32 cache) or __half (the F16 cache variant).  A 32 KB
// chunk holds 64 F32 key rows or 128 F16 key rows (one block).
template <typename KeyT>
struct Rows {
  static constexpr int kPerStage = kStageBytes / (kDi * sizeof(KeyT));
  static constexpr int kPerWarp = kPerStage / kConsumerWarps;   // 8 (F32) or 16 (F16)
};

template <typename KeyT, int kStages>
struct Smem {
  KeyT stage[kStages][kStageBytes / sizeof(KeyT)];
  uint64_t full[kStages];
  uint64_t empty[kStages];
  float red[2][kConsumerWarps];
};

// Four consecutive key elements as float.
__device__ __forceinline__ float4 load4(const float* p) { return *reinterpret_cast<const float4*>(p); }
__device__ __forceinline__ float4 load4(const __half* p) {
  const uint2 raw = *reinterpret_cast<const uint2*>(p);
  const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&raw.x));
  const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&raw.y));
  return make_float4(a.x, a.y, b.x, b.y);
}

template <typename KeyT>
struct Params {
  const float* idx_q;    // [n_q][G][Di]
  const KeyT* idx_k;     // [S][G][cap][Di]
  const int32_t* q_stream;
  const int32_t* q_pos;
  float* bs;             // [n_q][G][nblk]
  int n_q, G, n_streams, capacity, nblk;
  long long n_tasks;     // n_q * G * nblk (ignored in list mode)
  const int32_t* q_list;   // list mode: score only these query indices ...
  const int32_t* q_count;  // ... of which there are *q_count (device memory)
};

// Task t -> (query, group, block); in list mode the query comes from q_list.
template <typename KeyT>
__device__ __forceinline__ void task_coords(const Params<KeyT>& P, long long t, int& qi, int& g, int& b) {
  b = static_cast<int>(t % P.nblk);
  const long long qg = t / P.nblk;
  g = static_cast<int>(qg % P.G);
  const int i = static_cast<int>(qg / P.G);
  qi = P.q_list != nullptr ? P.q_list[i] : i;
}

// Visible blocks of query qi (0 for an out-of-range query).
template <typename KeyT>
__device__ __forceinline__ int query_visible(const Params<KeyT>& P, int qi, int& s, int& p) {
  s = P.q_stream[qi];
  p = P.q_pos[qi];
  if (s < 0 || s >= P.n_streams || p < 0 || p >= P.capacity) return 0;
  return p / kBlock + 1;
}

// Sum over the warp of 8 per-lane partial dot products (rows 0..7); the
// result for row (lane >> 2) lands in every lane of that quad.
__device__ __forceinline__ float reduce8_rows(const float (&v)[8], int lane) {
  const bool b4 = lane & 16, b3 = lane & 8, b2 = lane & 4;
  float q[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float send = b4 ? v[i] : v[i + 4];
    const float keep = b4 ? v[i + 4] : v[i];
    q[i] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
  }
  float r[2];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const float send = b3 ? q[i] : q[i + 2];
    const float keep = b3 ? q[i + 2] : q[i];
    r[i] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
  }
  const float send = b2 ? r[0] : r[1];
  float t = (b2 ? r[1] : r[0]) + __shfl_xor_sync(0xffffffffu, send, 4);
  t += __shfl_xor_sync(0xffffffffu, t, 2);
  t += __shfl_xor_sync(0xffffffffu, t, 1);
  return t;
}

// F16 rows: each half-warp holds one row of a row pair (lane >> 4 picks the
// row), each lane 8 of its 128 values.  Sum over each half-warp of 8 per-lane
// partial dot products (row pairs 0..7); the result for pair
// 4*b3 + 2*b2 + b1 (bits of the lane index) lands in both lanes of that pair.
__device__ __forceinline__ float reduce8_pairs(const float (&v)[8], int lane) {
  const bool b3 = lane & 8, b2 = lane & 4, b1 = lane & 2;
  float q[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float send = b3 ? v[i] : v[i + 4];
    const float keep = b3 ? v[i + 4] : v[i];
    q[i] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
  }
  float r[2];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const float send = b2 ? q[i] : q[i + 2];
    const float keep = b2 ? q[i + 2] : q[i];
    r[i] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
  }
  const float send = b1 ? r[0] : r[1];
  float t = (b1 ? r[1] : r[0]) + __shfl_xor_sync(0xffffffffu, send, 2);
  t += __shfl_xor_sync(0xffffffffu, t, 1);
  return t;
}

template <typename KeyT, int kStages>
__global__ void __launch_bounds__(kThreads, 1) block_scores_gemv_kernel(const Params<KeyT> P) {
  constexpr bool kF16 = sizeof(KeyT) == 2;
  constexpr int kRowsPerStage = Rows<KeyT>::kPerStage;
  constexpr int kRowsPerWarp = Rows<KeyT>::kPerWarp;
  constexpr int kStageElems = kRowsPerStage * kDi;
  extern __shared__ __align__(128) uint8_t smem_raw[];
  Smem<KeyT, kStages>& sm = *reinterpret_cast<Smem<KeyT, kStages>*>(smem_raw);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const long long T = P.q_list != nullptr ? static_cast<long long>(*P.q_count) * P.G * P.nblk : P.n_tasks;
  const long long t_begin = T * blockIdx.x / gridDim.x;
  const long long t_end = T * (blockIdx.x + 1) / gridDim.x;

  if (threadIdx.x == 0) {
#pragma unroll
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], kConsumerWarps);
    }
    mbar_fence_init();
  }
  __syncthreads();

  if (warp == kConsumerWarps) {
    // ---------------- producer: one thread issues every chunk copy --------
    if (lane != 0) return;
    const uint64_t pol = policy_evict_first();
    bool ok = true;
    int k = 0;
    for (long long t = t_begin; t < t_end && ok; ++t) {
      int qi, g, b;
      task_coords(P, t, qi, g, b);
      int s, p;
      const int nvis = query_visible(P, qi, s, p);
      if (b >= nvis) continue;
      const int n_chunks = min(p - b * kBlock, kBlock - 1) / kRowsPerStage + 1;
      const KeyT* src =
          P.idx_k + ((static_cast<size_t>(s) * P.G + g) * P.capacity + static_cast<size_t>(b) * kBlock) * kDi;
      for (int c = 0; c < n_chunks; ++c, ++k) {
        const int st = k % kStages;
        const uint32_t use = static_cast<uint32_t>(k / kStages);
        if (use > 0 && !mbar_wait(&sm.empty[st], (use - 1) & 1)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&sm.full[st], kStageBytes);
        bulk_load(sm.stage[st], src + static_cast<size_t>(c) * kStageElems, kStageBytes, &sm.full[st], pol);
      }
    }
    // Before leaving, make sure no copy this thread issued is still landing
    // (only matters when a consumer gave up early).
    for (int j = max(0, k - kStages); j < k; ++j) mbar_wait(&sm.full[j % kStages], (j / kStages) & 1);
    return;
  }

  // ---------------- consumers ------------------------------------------------
  bool ok = true;
  long long cur_qg = -1;
  float4 qv = make_float4(0.f, 0.f, 0.f, 0.f);
  float4 qv2 = make_float4(0.f, 0.f, 0.f, 0.f);   // F16 path: the lane's second 4 dims
  int k = 0;
  int par = 0;
  for (long long t = t_begin; t < t_end; ++t) {
    int qi, g, b;
    task_coords(P, t, qi, g, b);
    const long long qg = static_cast<long long>(qi) * P.G + g;
    const size_t out = static_cast<size_t>(qg) * P.nblk + b;
    int s, p;
    const int nvis = query_visible(P, qi, s, p);
    if (b >= nvis) {
      if (warp == 0 && lane == 0) {
        P.bs[out] = -INFINITY;
        if (nvis == 0 && b == 0 && g == 0) raise_error(MSA_DEVERR_QUERY_RANGE);
      }
      continue;
    }
    if (qg != cur_qg) {
      cur_qg = qg;
      if constexpr (kF16) {   // dims 8j .. 8j+7, j = lane & 15
        const float4* qp = reinterpret_cast<const float4*>(P.idx_q + static_cast<size_t>(qg) * kDi) + 2 * (lane & 15);
        qv = __ldg(qp);
        qv2 = __ldg(qp + 1);
      } else {
        qv = __ldg(reinterpret_cast<const float4*>(P.idx_q + static_cast<size_t>(qg) * kDi) + lane);
      }
    }
    float m = -INFINITY;
    const int n_chunks = min(p - b * kBlock, kBlock - 1) / kRowsPerStage + 1;
    for (int c = 0; c < n_chunks; ++c, ++k) {
      const int st = k % kStages;
      if (ok) ok = mbar_wait(&sm.full[st], (k / kStages) & 1);
      if (ok) {
        if constexpr (kF16) {
          // 16 rows per warp as 8 row pairs; one 16-byte load covers 8 values
          const KeyT* base = sm.stage[st] + (warp * kRowsPerWarp + (lane >> 4)) * kDi + 8 * (lane & 15);
          float part[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const uint4 raw = *reinterpret_cast<const uint4*>(base + 2 * i * kDi);
            const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&raw.x));
            const float2 bb = __half22float2(*reinterpret_cast<const __half2*>(&raw.y));
            const float2 cc = __half22float2(*reinterpret_cast<const __half2*>(&raw.z));
            const float2 dd = __half22float2(*reinterpret_cast<const __half2*>(&raw.w));
            float acc = qv.x * a.x;
            acc = fmaf(qv.y, a.y, acc);
            acc = fmaf(qv.z, bb.x, acc);
            acc = fmaf(qv.w, bb.y, acc);
            acc = fmaf(qv2.x, cc.x, acc);
            acc = fmaf(qv2.y, cc.y, acc);
            acc = fmaf(qv2.z, dd.x, acc);
            part[i] = fmaf(qv2.w, dd.y, acc);
          }
          const float dot = reduce8_pairs(part, lane);
          const int ip = ((lane >> 3) & 1) * 4 + ((lane >> 2) & 1) * 2 + ((lane >> 1) & 1);
          const int j = b * kBlock + c * kRowsPerStage + warp * kRowsPerWarp + 2 * ip + (lane >> 4);
          if (j <= p) m = fmaxf(m, dot);
        } else {
          const KeyT* base = sm.stage[st] + warp * kRowsPerWarp * kDi + lane * 4;
          float part[kRowsPerWarp];
#pragma unroll
          for (int r = 0; r < kRowsPerWarp; ++r) {
            const float4 kv = load4(base + r * kDi);
            part[r] = fmaf(qv.w, kv.w, fmaf(qv.z, kv.z, fmaf(qv.y, kv.y, qv.x * kv.x)));
          }
          const float dot = reduce8_rows(part, lane);
          const int j = b * kBlock + c * kRowsPerStage + warp * kRowsPerWarp + (lane >> 2);
          if (j <= p) m = fmaxf(m, dot);  // fmaxf drops NaN: a NaN score ranks as -inf
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.empty[st]);
    }
    if constexpr (kF16) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 4));
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 8));
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 16));
    if (lane == 0) sm.red[par][warp] = m;
    named_barrier_sync(1, kConsumerWarps * 32);
    if (warp == 0 && lane == 0) {
      float mm = sm.red[par][0];
#pragma unroll
      for (int w = 1; w < kConsumerWarps; ++w) mm = fmaxf(mm, sm.red[par][w]);
      if (b == p / kBlock) mm += MSA_LOCAL_BIAS;
      P.bs[out] = mm;
    }
    par ^= 1;
  }
}

}  // namespace gemv
}  // namespace msa
