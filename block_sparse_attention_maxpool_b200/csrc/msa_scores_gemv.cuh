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

#include "msa_common.cuh"

namespace msa {
namespace gemv {

constexpr int kDi = 128;                                 // indexer dim
constexpr int kBlock = 128;                              // key block
constexpr int kRowsPerStage = 64;                        // key rows per chunk
constexpr int kStageFloats = kRowsPerStage * kDi;
constexpr uint32_t kStageBytes = kStageFloats * 4;       // 32 KB
constexpr int kChunksPerBlock = kBlock / kRowsPerStage;  // 2
constexpr int kConsumerWarps = 8;
constexpr int kRowsPerWarp = kRowsPerStage / kConsumerWarps;  // 8
constexpr int kThreads = (kConsumerWarps + 1) * 32;

template <int kStages>
struct Smem {
  float stage[kStages][kStageFloats];
  uint64_t full[kStages];
  uint64_t empty[kStages];
  float red[2][kConsumerWarps];
};

struct Params {
  const float* idx_q;    // [n_q][G][Di]
  const float* idx_k;    // [S][G][cap][Di]
  const int32_t* q_stream;
  const int32_t* q_pos;
  float* bs;             // [n_q][G][nblk]
  int n_q, G, n_streams, capacity, nblk;
  long long n_tasks;     // n_q * G * nblk (ignored in list mode)
  const int32_t* q_list;   // list mode: score only these query indices ...
  const int32_t* q_count;  // ... of which there are *q_count (device memory)
};

// Task t -> (query, group, block); in list mode the query comes from q_list.
__device__ __forceinline__ void task_coords(const Params& P, long long t, int& qi, int& g, int& b) {
  b = static_cast<int>(t % P.nblk);
  const long long qg = t / P.nblk;
  g = static_cast<int>(qg % P.G);
  const int i = static_cast<int>(qg / P.G);
  qi = P.q_list != nullptr ? P.q_list[i] : i;
}

// Visible blocks of query qi (0 for an out-of-range query).
__device__ __forceinline__ int query_visible(const Params& P, int qi, int& s, int& p) {
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

template <int kStages>
__global__ void __launch_bounds__(kThreads, 1) block_scores_gemv_kernel(const Params P) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  Smem<kStages>& sm = *reinterpret_cast<Smem<kStages>*>(smem_raw);
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
      const float* src =
          P.idx_k + ((static_cast<size_t>(s) * P.G + g) * P.capacity + static_cast<size_t>(b) * kBlock) * kDi;
      for (int c = 0; c < n_chunks; ++c, ++k) {
        const int st = k % kStages;
        const uint32_t use = static_cast<uint32_t>(k / kStages);
        if (use > 0 && !mbar_wait(&sm.empty[st], (use - 1) & 1)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&sm.full[st], kStageBytes);
        bulk_load(sm.stage[st], src + static_cast<size_t>(c) * kStageFloats, kStageBytes, &sm.full[st], pol);
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
      qv = __ldg(reinterpret_cast<const float4*>(P.idx_q + static_cast<size_t>(qg) * kDi) + lane);
    }
    float m = -INFINITY;
    const int n_chunks = min(p - b * kBlock, kBlock - 1) / kRowsPerStage + 1;
    for (int c = 0; c < n_chunks; ++c, ++k) {
      const int st = k % kStages;
      if (ok) ok = mbar_wait(&sm.full[st], (k / kStages) & 1);
      if (ok) {
        const float* base = sm.stage[st] + warp * kRowsPerWarp * kDi + lane * 4;
        float part[kRowsPerWarp];
#pragma unroll
        for (int r = 0; r < kRowsPerWarp; ++r) {
          const float4 kv = *reinterpret_cast<const float4*>(base + r * kDi);
          part[r] = fmaf(qv.w, kv.w, fmaf(qv.z, kv.z, fmaf(qv.y, kv.y, qv.x * kv.x)));
        }
        const float dot = reduce8_rows(part, lane);
        const int j = b * kBlock + c * kRowsPerStage + warp * kRowsPerWarp + (lane >> 2);
        if (j <= p) m = fmaxf(m, dot);  // fmaxf drops NaN: a NaN score ranks as -inf
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.empty[st]);
    }
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
