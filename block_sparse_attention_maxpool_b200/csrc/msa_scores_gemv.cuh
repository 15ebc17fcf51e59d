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
// 8 rows).  The F16 cache variant runs two CTAs per SM, each with a 3-stage
// ring, and reduces half-warp row pairs the same way.  Rows past the query position are masked, the per-block maximum
// is combined across warps and the local block gets MSA_LOCAL_BIAS.
#pragma once

#include <cuda_fp16.h>

#include "msa_common.cuh"

namespace msa {
namespace gemv {

constexpr int kDi = 128;                                 // indexer dim
constexpr int kBlock = 128;                              // key block
constexpr uint32_t kStageBytes = 32 * 1024;              // one chunk of key rows

// Launch shape per key type: consumer warps, ring stages and resident CTAs
// per SM (the grid is that many CTAs per SM, each with the ring in shared
// memory).
template <typename KeyT>
struct Config;
template <>
struct Config<float> {
  static constexpr int kWarps = 8, kStages = 4, kCtasPerSm = 1;
};
template <>
struct Config<__half> {   // twice the blocks per byte: two independent rings per SM hide the per-block joins
  static constexpr int kWarps = 8, kStages = 3, kCtasPerSm = 2;
};

// KeyT: float (the F32 cache) or __half (the F16 cache variant).  A 32 KB
// chunk holds 64 F32 key rows or 128 F16 key rows (one block).  An F32 row
// spans the warp (4 values per lane); an F16 row spans a half-warp (8 values
// per lane), so one 16-byte load per lane covers two rows.
template <typename KeyT, int kWarps>
struct Rows {
  static constexpr int kPerStage = kStageBytes / (kDi * sizeof(KeyT));
  static constexpr int kPerWarp = kPerStage / kWarps;
  static constexpr int kPerLoad = sizeof(KeyT) == 2 ? 2 : 1;
  static constexpr int kPartials = kPerWarp / kPerLoad;   // dot products per lane per chunk
  static constexpr int kLanesPerRow = 32 / kPerLoad;
  static_assert(kPerWarp * kWarps == kPerStage && kPartials >= 1, "rows must split evenly over warps");
};

template <typename KeyT, int kStages, int kWarps>
struct Smem {
  KeyT stage[kStages][kStageBytes / sizeof(KeyT)];
  uint64_t full[kStages];
  uint64_t empty[kStages];
  float red[2][kWarps];
};

template <typename KeyT>
struct Params {
  const float* idx_q;    // [n_q][G][Di]
  const KeyT* idx_k;     // [S][G][cap][Di], or pages [n_pages][G][128][Di]
  const int32_t* q_stream;
  const int32_t* q_pos;
  float* bs;             // [n_q][G][nblk]
  int n_q, G, n_streams, capacity, nblk;
  long long n_tasks;     // n_q * G * nblk (ignored in list mode)
  const int32_t* q_list;   // list mode: score only these query indices ...
  const int32_t* q_count;  // ... of which there are *q_count (device memory)
  KvPages pages;           // block table of a paged cache (table null: contiguous)
};

// Walks the task space (query slot, group, block) in order, block fastest,
// without a division per task; the query's stream, position and visible
// block count are re-read only when the query slot changes.
template <typename KeyT>
struct Cursor {
  int i, g, b;      // query slot (index into q_list in list mode), group, block
  int qi, s, p, nvis;
  __device__ __forceinline__ void load_query(const Params<KeyT>& P) {
    qi = P.q_list != nullptr ? P.q_list[i] : i;
    s = P.q_stream[qi];
    p = P.q_pos[qi];
    nvis = (s < 0 || s >= P.n_streams || p < 0 || p >= P.capacity) ? 0 : p / kBlock + 1;
  }
  __device__ __forceinline__ void start(const Params<KeyT>& P, long long t, long long t_end) {
    b = static_cast<int>(t % P.nblk);
    const long long qg = t / P.nblk;
    g = static_cast<int>(qg % P.G);
    i = static_cast<int>(qg / P.G);
    if (t < t_end) load_query(P);
  }
  // Advance to task t + 1 (t + 1 < t_end).
  __device__ __forceinline__ void next(const Params<KeyT>& P) {
    if (++b < P.nblk) return;
    b = 0;
    if (++g < P.G) return;
    g = 0;
    ++i;
    load_query(P);
  }
};

// Sum over groups of kLanes lanes of kN per-lane partials (kN <= kLanes, both
// powers of two).  Each halving step trades half of the partials with the
// lane kLanes/2, kLanes/4, ... away, so after log2(kN) steps every lane holds
// one partially summed index; the remaining steps finish the sum.  Partial
// partial_index<kN, kLanes>(lane) ends in the lane (every lane of the group
// whose bits select that index holds it).
template <int kN, int kLanes>
__device__ __forceinline__ float transposed_sum(float (&v)[kN], int lane) {
  static_assert(kN >= 1 && kN <= kLanes && (kN & (kN - 1)) == 0 && (kLanes & (kLanes - 1)) == 0, "bad shape");
  int off = kLanes / 2;
#pragma unroll
  for (int n = kN; n > 1; n /= 2, off /= 2) {
    const bool upper = lane & off;
#pragma unroll
    for (int i = 0; i < n / 2; ++i) {
      const float send = upper ? v[i] : v[i + n / 2];
      const float keep = upper ? v[i + n / 2] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
    }
  }
  float t = v[0];
#pragma unroll
  for (; off >= 1; off /= 2) t += __shfl_xor_sync(0xffffffffu, t, off);
  return t;
}

template <int kN, int kLanes>
__device__ __forceinline__ int partial_index(int lane) {
  int idx = 0, off = kLanes / 2;
#pragma unroll
  for (int n = kN; n > 1; n /= 2, off /= 2)
    if (lane & off) idx += n / 2;
  return idx;
}

// Dot product of 8 F16 key values (one 16-byte word) with 8 query values.
__device__ __forceinline__ float dot8_f16(const uint4 raw, const float4 qa, const float4 qb) {
  const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&raw.x));
  const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&raw.y));
  const float2 c = __half22float2(*reinterpret_cast<const __half2*>(&raw.z));
  const float2 d = __half22float2(*reinterpret_cast<const __half2*>(&raw.w));
  float acc = qa.x * a.x;
  acc = fmaf(qa.y, a.y, acc);
  acc = fmaf(qa.z, b.x, acc);
  acc = fmaf(qa.w, b.y, acc);
  acc = fmaf(qb.x, c.x, acc);
  acc = fmaf(qb.y, c.y, acc);
  acc = fmaf(qb.z, d.x, acc);
  return fmaf(qb.w, d.y, acc);
}

// The kernel body: CTA `cta` of `n_cta` takes its contiguous share of the
// tasks.  smem_raw: at least sizeof(Smem<...>) bytes, 128-byte aligned.
// Warps past the producer warp (when a caller's CTA has more) only join the
// initial barrier.
template <typename KeyT, int kStages, int kWarps>
__device__ __forceinline__ void block_scores_gemv_body(const Params<KeyT>& P, uint8_t* smem_raw, int cta, int n_cta) {
  constexpr bool kF16 = sizeof(KeyT) == 2;
  using R = Rows<KeyT, kWarps>;
  constexpr int kStageElems = R::kPerStage * kDi;
  Smem<KeyT, kStages, kWarps>& sm = *reinterpret_cast<Smem<KeyT, kStages, kWarps>*>(smem_raw);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const long long T = P.q_list != nullptr ? static_cast<long long>(*P.q_count) * P.G * P.nblk : P.n_tasks;
  const long long t_begin = T * cta / n_cta;
  const long long t_end = T * (cta + 1) / n_cta;

  if (threadIdx.x == 0) {
#pragma unroll
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], kWarps);
    }
    mbar_fence_init();
  }
  __syncthreads();
  if (warp > kWarps) return;

  Cursor<KeyT> cur;
  cur.start(P, t_begin, t_end);

  if (warp == kWarps) {
    // ---------------- producer: one thread issues every chunk copy --------
    if (lane != 0) return;
    const uint64_t pol = policy_evict_first();
    bool ok = true;
    int k = 0;
    for (long long t = t_begin; t < t_end && ok; ++t) {
      if (t > t_begin) cur.next(P);
      if (cur.b >= cur.nvis) continue;
      const long long row = kv_block_row(P.pages, cur.s, cur.g, cur.b, P.G, P.capacity);
      if (row < 0) continue;
      const int n_chunks = min(cur.p - cur.b * kBlock, kBlock - 1) / R::kPerStage + 1;
      const KeyT* src = P.idx_k + static_cast<size_t>(row) * kDi;
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
  // Lane layout within a chunk: this warp owns rows [warp * kPerWarp, +kPerWarp);
  // partial r of a lane covers row r * kPerLoad + (lane / kLanesPerRow) of them.
  const int part_row = partial_index<R::kPartials, R::kLanesPerRow>(lane) * R::kPerLoad + lane / R::kLanesPerRow;
  const int lane_in_row = lane % R::kLanesPerRow;
  bool ok = true;
  long long cur_qg = -1;
  float4 qv = make_float4(0.f, 0.f, 0.f, 0.f);
  float4 qv2 = make_float4(0.f, 0.f, 0.f, 0.f);   // F16 path: the lane's second 4 dims
  int k = 0;
  int par = 0;
  for (long long t = t_begin; t < t_end; ++t) {
    if (t > t_begin) cur.next(P);
    const int b = cur.b, p = cur.p;
    const long long qg = static_cast<long long>(cur.qi) * P.G + cur.g;
    const size_t out = static_cast<size_t>(qg) * P.nblk + b;
    if (b >= cur.nvis) {
      if (warp == 0 && lane == 0) {
        P.bs[out] = -INFINITY;
        if (cur.nvis == 0 && b == 0 && cur.g == 0) raise_error(MSA_DEVERR_QUERY_RANGE);
      }
      continue;
    }
    if (P.pages.table != nullptr && kv_block_row(P.pages, cur.s, cur.g, b, P.G, P.capacity) < 0) {
      if (warp == 0 && lane == 0) {   // the producer skipped this block too
        P.bs[out] = -INFINITY;
        raise_error(MSA_DEVERR_PAGE_RANGE);
      }
      continue;
    }
    if (qg != cur_qg) {
      cur_qg = qg;
      const float4* qp = reinterpret_cast<const float4*>(P.idx_q + static_cast<size_t>(qg) * kDi);
      if constexpr (kF16) {   // dims 8j .. 8j+7, j = lane_in_row
        qv = __ldg(qp + 2 * lane_in_row);
        qv2 = __ldg(qp + 2 * lane_in_row + 1);
      } else {                // dims 4 * lane .. +3
        qv = __ldg(qp + lane_in_row);
      }
    }
    float m = -INFINITY;
    const int n_chunks = min(p - b * kBlock, kBlock - 1) / R::kPerStage + 1;
    for (int c = 0; c < n_chunks; ++c, ++k) {
      const int st = k % kStages;
      if (ok) ok = mbar_wait(&sm.full[st], (k / kStages) & 1);
      ok = __all_sync(0xffffffffu, ok);   // warp-uniform: the row sums below shuffle across the warp
      if (ok) {
        const KeyT* base = sm.stage[st] + (warp * R::kPerWarp + lane / R::kLanesPerRow) * kDi;
        float part[R::kPartials];
#pragma unroll
        for (int r = 0; r < R::kPartials; ++r) {
          const KeyT* row = base + r * R::kPerLoad * kDi;
          if constexpr (kF16) {
            part[r] = dot8_f16(*reinterpret_cast<const uint4*>(row + 8 * lane_in_row), qv, qv2);
          } else {
            const float4 kv = *reinterpret_cast<const float4*>(row + 4 * lane_in_row);
            part[r] = fmaf(qv.w, kv.w, fmaf(qv.z, kv.z, fmaf(qv.y, kv.y, qv.x * kv.x)));
          }
        }
        const float dot = transposed_sum<R::kPartials, R::kLanesPerRow>(part, lane);
        const int j = b * kBlock + c * R::kPerStage + warp * R::kPerWarp + part_row;
        if (j <= p) m = fmaxf(m, dot);  // fmaxf drops NaN: a NaN score ranks as -inf
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.empty[st]);
    }
    // lanes that differ only below bit kSame hold the same row
    constexpr int kSame = R::kLanesPerRow / R::kPartials;
#pragma unroll
    for (int off = kSame; off < 32; off *= 2) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    if (lane == 0) sm.red[par][warp] = m;
    named_barrier_sync(1, kWarps * 32);
    if (warp == 0 && lane == 0) {
      float mm = sm.red[par][0];
#pragma unroll
      for (int w = 1; w < kWarps; ++w) mm = fmaxf(mm, sm.red[par][w]);
      if (b == p / kBlock) mm += MSA_LOCAL_BIAS;
      P.bs[out] = mm;
    }
    par ^= 1;
  }
}

template <typename KeyT, int kStages, int kWarps, int kMinCtas>
__global__ void __launch_bounds__((kWarps + 1) * 32, kMinCtas) block_scores_gemv_kernel(const Params<KeyT> P) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  pdl_trigger();
  pdl_wait();
  block_scores_gemv_body<KeyT, kStages, kWarps>(P, smem_raw, blockIdx.x, gridDim.x);
}

// Invalidate the body's mbarriers (one thread, after every thread of the CTA
// is past its last use) so that the shared memory can be used for other data.
template <typename KeyT, int kStages, int kWarps>
__device__ __forceinline__ void block_scores_gemv_release(uint8_t* smem_raw) {
  Smem<KeyT, kStages, kWarps>& sm = *reinterpret_cast<Smem<KeyT, kStages, kWarps>*>(smem_raw);
#pragma unroll
  for (int s = 0; s < kStages; ++s) {
    mbar_inval(&sm.full[s]);
    mbar_inval(&sm.empty[s]);
  }
}

}  // namespace gemv
}  // namespace msa
