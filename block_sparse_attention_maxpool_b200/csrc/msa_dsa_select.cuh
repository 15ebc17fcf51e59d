// Token-level variant: keep the top-k tokens of each query.
//
// "deepseek2 : GLM-DSA sparse attention (lightning indexer)", section "What
// this does": the top-k highest-scoring keys of each query are kept (GLM-5.2
// keeps 2048); with at most k visible tokens every visible token is kept
// (the page's "no-op-exact" check).  Equal scores keep the lower token index;
// NaN ranks as -inf; -0 equals +0.
//
// One CTA of 1024 threads per query.  Each visible score becomes an
// order-preserving 32-bit key, staged in shared memory (contexts up to 48K
// tokens; longer ones are re-read from global memory, where they stay in
// L2).  The k-th largest key T comes from a sample-select: the keys of 2048
// evenly spaced tokens bracket the rank k/n quantile (two exact radix
// selects on the sample), one ballot-compacted pass keeps the few thousand
// keys inside the bracket and counts those above it, and an exact radix
// select among the kept keys gives T and how many keys equal to T are still
// needed.  If the bracket misses (rare), the radix select runs over all
// keys, so the result is always exact.  A final pass walks the tokens in
// index order, one contiguous range per warp, and writes every token with
// key > T plus the first needed tokens with key == T: the output is
// ascending with no sort.
//
// The radix select is most-significant-digit first, 8 bits per pass, with
// shared-memory atomic histograms; the filter and emit passes take four
// keys per lane per step and place them with warp scans.
//
// A batch with fewer queries than SMs (a decode step) would leave most SMs
// idle with one CTA per query, so it runs on clusters of four CTAs per query
// instead (dsa_select_topk_cluster_kernel, rows up to 192K tokens): the
// quarters of a row are staged by the four CTAs, and the radix select and
// the emit offsets are combined through distributed shared memory.
#pragma once

#include <cooperative_groups.h>
#include <cstddef>

#include "msa_common.cuh"

namespace msa {
namespace dsa {

constexpr int kSelThreads = 1024;
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kMaxTopK = 2048;                 // width of a selection row
constexpr int kSmemKeys = 48 * 1024;           // scores staged in shared memory up to this context
constexpr int kSamples = 2048;                 // sample of the sample-select
constexpr int kMaxCands = 4096;                // keys kept inside the sample bracket
constexpr int kSampleMin = 8192;               // shorter contexts take the plain radix select

struct SelSmem {
  unsigned int hist[256];
  int warp_gt[kSelWarps];
  int warp_eq[kSelWarps];
  uint32_t prefix;
  int need;
  int n_above;                 // sample-select: keys above the bracket
  int n_cand;                  // sample-select: keys kept inside it
  uint32_t samples[kSamples];
  uint32_t cands[kMaxCands];
  uint32_t keys[kSmemKeys];    // last: the unstaged kernel is launched without it
};
static_assert(offsetof(SelSmem, keys) % 16 == 0 && offsetof(SelSmem, cands) % 16 == 0 &&
                  offsetof(SelSmem, samples) % 16 == 0,
              "key vectors must be 16-byte aligned");
constexpr size_t kSelSmemStaged = sizeof(SelSmem);
constexpr size_t kSelSmemUnstaged = sizeof(SelSmem) - sizeof(uint32_t) * kSmemKeys;
static_assert(kSelSmemStaged <= 232448, "shared memory budget");

// Order-preserving key of a score: larger score, larger key.  NaN maps to
// the key of -inf and -0 to the key of +0.
__device__ __forceinline__ uint32_t score_key(float x) {
  uint32_t u = __float_as_uint(x);
  if (x != x) u = 0xff800000u;
  if (x == 0.f) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Keys read from a shared-memory array (16-byte aligned).  get4(i): keys
// i .. i+3 for i a multiple of 4, in one vector load; callers ignore keys at
// or past n, and every array is long enough for the whole vector.
struct SmemKeys {
  const uint32_t* a;
  __device__ __forceinline__ uint32_t operator()(int i) const { return a[i]; }
  __device__ __forceinline__ uint4 get4(int i) const { return *reinterpret_cast<const uint4*>(a + i); }
};
// Keys computed from a score row in global memory (rows are whole multiples
// of 128 floats, 16-byte aligned).
struct RowKeys {
  const float* row;
  __device__ __forceinline__ uint32_t operator()(int i) const { return score_key(__ldg(row + i)); }
  __device__ __forceinline__ uint4 get4(int i) const {
    const float4 v = __ldg(reinterpret_cast<const float4*>(row + i));
    return make_uint4(score_key(v.x), score_key(v.y), score_key(v.z), score_key(v.w));
  }
};

// The k-th largest (1 <= k <= n) of the n keys get(0..n-1): *T receives it
// and *need how many keys equal to it rank within the first k.  Called by
// the whole CTA; ends with a barrier.
template <typename Get>
__device__ void radix_kth(SelSmem& sm, Get get, int n, int k, uint32_t* T, int* need_out) {
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  if (tid == 0) {
    sm.prefix = 0;
    sm.need = k;
  }
  uint32_t mask = 0;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int b = tid; b < 256; b += kSelThreads) sm.hist[b] = 0;
    __syncthreads();
    const uint32_t prefix = sm.prefix;
    for (int i = tid; i < n; i += kSelThreads) {
      const uint32_t key = get(i);
      if ((key & mask) == prefix) atomicAdd(&sm.hist[(key >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (warp == 0) {
      // lane l holds bins 255-8l .. 248-8l (descending); find the bin where
      // the count from the top reaches `need`
      const int need = sm.need;
      unsigned int c[8];
      unsigned int local = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        c[j] = sm.hist[255 - 8 * lane - j];
        local += c[j];
      }
      unsigned int incl = local;                      // inclusive scan over lanes (from the top bins)
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const unsigned int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      const unsigned int excl = incl - local;
      if (excl < static_cast<unsigned int>(need) && incl >= static_cast<unsigned int>(need)) {
        unsigned int cum = excl;
        int bin = 255 - 8 * lane;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (cum + c[j] >= static_cast<unsigned int>(need)) {
            bin = 255 - 8 * lane - j;
            break;
          }
          cum += c[j];
        }
        sm.prefix = prefix | (static_cast<uint32_t>(bin) << shift);
        sm.need = need - static_cast<int>(cum);
      }
    }
    mask |= 255u << shift;
    __syncthreads();
  }
  *T = sm.prefix;
  *need_out = sm.need;
  __syncthreads();
}

// Sample-select of the k-th largest of the n keys get(0..n-1) (n >= 4 *
// kSamples): false when the sample bracket misses the k-th key or keeps too
// many keys, in which case nothing is returned.  Called by the whole CTA.
template <typename Get>
__device__ bool sample_kth(SelSmem& sm, Get get, int n, int k, uint32_t* T, int* need) {
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  for (int j = tid; j < kSamples; j += kSelThreads)
    sm.samples[j] = get(static_cast<int>(static_cast<long long>(j) * n / kSamples));
  if (tid == 0) {
    sm.n_above = 0;
    sm.n_cand = 0;
  }
  __syncthreads();
  // the k-th key's expected rank in the sample, +- three binomial standard deviations
  const float r = static_cast<float>(k) * kSamples / n;
  const int delta = static_cast<int>(3.f * sqrtf(r) + 8.f);
  const int r_hi = static_cast<int>(r) - delta;                  // 1-based ranks
  const int r_lo = min(kSamples, static_cast<int>(r) + delta + 1);
  const bool has_hi = r_hi >= 1;
  uint32_t t_hi = 0xffffffffu, t_lo = 0u;
  int unused;
  if (has_hi) radix_kth(sm, SmemKeys{sm.samples}, kSamples, r_hi, &t_hi, &unused);
  radix_kth(sm, SmemKeys{sm.samples}, kSamples, r_lo, &t_lo, &unused);

  // one pass: count the keys above the bracket, keep the keys inside it
  // (four keys per lane per iteration; order inside the kept list is free)
  int above = 0;
  for (int base0 = 0; base0 < n; base0 += 4 * kSelThreads) {      // same trip count in every lane
    const int base = base0 + 4 * tid;
    const uint4 kv = base < n ? get.get4(base) : make_uint4(0u, 0u, 0u, 0u);
    const uint32_t key[4] = {kv.x, kv.y, kv.z, kv.w};
    int keep_n = 0;
    bool keep[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const bool in = base + j < n;
      const bool up = in && has_hi && key[j] > t_hi;
      keep[j] = in && !up && key[j] >= t_lo;
      above += up ? 1 : 0;
      keep_n += keep[j] ? 1 : 0;
    }
    int incl = keep_n;                                   // warp inclusive scan of the kept counts
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    const int total = __shfl_sync(0xffffffffu, incl, 31);
    int slot0 = 0;
    if (lane == 31 && total > 0) slot0 = atomicAdd(&sm.n_cand, total);
    int slot = __shfl_sync(0xffffffffu, slot0, 31) + incl - keep_n;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      if (keep[j]) {
        if (slot < kMaxCands) sm.cands[slot] = key[j];
        ++slot;
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) above += __shfl_xor_sync(0xffffffffu, above, o);
  if (lane == 0 && above != 0) atomicAdd(&sm.n_above, above);
  __syncthreads();
  const int n_above = sm.n_above;
  const int n_cand = sm.n_cand;
  __syncthreads();
  if (n_cand > kMaxCands || n_above >= k || n_above + n_cand < k) return false;
  radix_kth(sm, SmemKeys{sm.cands}, n_cand, k - n_above, T, need);
  return true;
}

// Per-warp key counts of the emit pass: warp w owns the contiguous range
// [w0, w1) of the n keys (whole spans of 128) and counts its keys above T
// and equal to T into warp_gt[w] / warp_eq[w].  Called by the whole CTA;
// ends with a barrier.
constexpr int kEmitSpan = 4 * 32;

__device__ __forceinline__ void warp_range(int n, int warp, int& w0, int& w1) {
  const int per_warp = (n + kSelWarps * kEmitSpan - 1) / (kSelWarps * kEmitSpan) * kEmitSpan;
  w0 = min(n, warp * per_warp);
  w1 = min(n, w0 + per_warp);
}

template <typename Get>
__device__ void count_gt_eq(Get get, int n, uint32_t T, int* warp_gt, int* warp_eq) {
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  int w0, w1;
  warp_range(n, warp, w0, w1);
  int gt = 0, eq = 0;
  for (int b0 = w0; b0 < w1; b0 += kEmitSpan) {
    const int i0 = b0 + 4 * lane;
    const uint4 kv = i0 < w1 ? get.get4(i0) : make_uint4(0u, 0u, 0u, 0u);
    const uint32_t key[4] = {kv.x, kv.y, kv.z, kv.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      gt += (i0 + j < w1 && key[j] > T) ? 1 : 0;
      eq += (i0 + j < w1 && key[j] == T) ? 1 : 0;
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    gt += __shfl_xor_sync(0xffffffffu, gt, o);
    eq += __shfl_xor_sync(0xffffffffu, eq, o);
  }
  if (lane == 0) {
    warp_gt[warp] = gt;
    warp_eq[warp] = eq;
  }
  __syncthreads();
}

// Write, in index order, every token with key > T and the first need_eq
// tokens with key == T.  Key i is token tok0 + i; gt0 / eq0 keys above /
// equal to T come before key 0 (other CTAs' ranges).  Each warp walks its
// range 128 keys at a time, four consecutive keys per lane, placing them
// with one warp scan per 128 keys after the counts of count_gt_eq.
template <typename Get>
__device__ void emit_counted(Get get, int n, uint32_t T, int need_eq, int32_t* out, const int* warp_gt,
                             const int* warp_eq, int tok0, int gt0, int eq0) {
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  int w0, w1;
  warp_range(n, warp, w0, w1);
  int gt_before = gt0, eq_before = eq0;
  for (int w = 0; w < warp; ++w) {
    gt_before += warp_gt[w];
    eq_before += warp_eq[w];
  }
  for (int b0 = w0; b0 < w1; b0 += kEmitSpan) {
    bool is_gt[4], is_eq[4];
    int packed = 0;                                   // gt count | eq count << 16
    const int i0 = b0 + 4 * lane;
    const uint4 kv = i0 < w1 ? get.get4(i0) : make_uint4(0u, 0u, 0u, 0u);
    const uint32_t key[4] = {kv.x, kv.y, kv.z, kv.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int i = i0 + j;
      is_gt[j] = i < w1 && key[j] > T;
      is_eq[j] = i < w1 && key[j] == T;
      packed += (is_gt[j] ? 1 : 0) + (is_eq[j] ? 1 << 16 : 0);
    }
    int incl = packed;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    const int excl = incl - packed;
    int g = gt_before + (excl & 0xffff);
    int e = eq_before + (excl >> 16);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int i = tok0 + b0 + 4 * lane + j;
      if (is_gt[j]) {
        out[g + min(e, need_eq)] = i;
        ++g;
      } else if (is_eq[j]) {
        if (e < need_eq) out[g + e] = i;
        ++e;
      }
    }
    const int tot = __shfl_sync(0xffffffffu, incl, 31);
    gt_before += tot & 0xffff;
    eq_before += tot >> 16;
  }
}

// The emit pass of one CTA over all n keys.
template <typename Get>
__device__ void emit_topk(SelSmem& sm, Get get, int n, uint32_t T, int need_eq, int32_t* out) {
  count_gt_eq(get, n, T, sm.warp_gt, sm.warp_eq);
  emit_counted(get, n, T, need_eq, out, sm.warp_gt, sm.warp_eq, 0, 0, 0);
}

template <bool kStaged>
__global__ void __launch_bounds__(kSelThreads, 1)
    dsa_select_topk_kernel(const float* __restrict__ scores, const int32_t* __restrict__ q_pos, int n_q,
                           int capacity, int top_k, int32_t* __restrict__ sel, int32_t* __restrict__ n_sel) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  SelSmem& sm = *reinterpret_cast<SelSmem*>(smem_raw);
  const int t = blockIdx.x;
  const int tid = threadIdx.x;
  pdl_trigger();
  pdl_wait();
  if (t >= n_q) return;
  const int p = q_pos[t];
  int32_t* out = sel + static_cast<size_t>(t) * kMaxTopK;
  if (p < 0 || p >= capacity) {
    for (int i = tid; i < kMaxTopK; i += kSelThreads) out[i] = -1;
    if (tid == 0) {
      if (n_sel != nullptr) n_sel[t] = 0;
      raise_error(MSA_DEVERR_QUERY_RANGE);
    }
    return;
  }
  const int n = p + 1;
  if (n <= top_k) {                                   // every visible token is kept
    for (int i = tid; i < kMaxTopK; i += kSelThreads) out[i] = i < n ? i : -1;
    if (tid == 0 && n_sel != nullptr) n_sel[t] = n;
    return;
  }
  const float* row = scores + static_cast<size_t>(t) * capacity;
  uint32_t T;
  int need;
  if constexpr (kStaged) {
#pragma unroll 8
    for (int i = tid; i < n; i += kSelThreads) sm.keys[i] = score_key(__ldg(row + i));   // loads in flight
    __syncthreads();
    const SmemKeys get{sm.keys};
    if (n < kSampleMin || !sample_kth(sm, get, n, top_k, &T, &need)) radix_kth(sm, get, n, top_k, &T, &need);
    emit_topk(sm, get, n, T, need, out);
  } else {
    const RowKeys get{row};
    if (!sample_kth(sm, get, n, top_k, &T, &need)) radix_kth(sm, get, n, top_k, &T, &need);
    emit_topk(sm, get, n, T, need, out);
  }
  for (int i = top_k + tid; i < kMaxTopK; i += kSelThreads) out[i] = -1;
  if (tid == 0 && n_sel != nullptr) n_sel[t] = top_k;
}

// ---- the same selection on a cluster of CTAs per query ----------------------
// One query's keys split into kClusterCtas contiguous quarters, one per CTA
// of a thread-block cluster (so a small batch of long rows uses four times
// the SMs).  Each CTA stages its quarter in shared memory.  The radix select
// of the k-th key runs over the whole row: per 8-bit digit, every CTA
// counts its own keys into a local histogram and adds it into rank 0's
// histogram through distributed shared memory; after a cluster barrier rank
// 0 picks the digit (as radix_kth does) and clears its histogram; after a
// second barrier every CTA reads the decided prefix.  The emit pass then
// counts each CTA's keys above and equal to T, exchanges the four totals
// through rank 0, and each CTA writes its quarter's tokens at their global
// places: the output is the same ascending list as the one-CTA kernels'.
constexpr int kClusterCtas = 4;
constexpr int kClusterKeys = kClusterCtas * kSmemKeys;   // longest row the cluster path stages

struct ClusterSmem {
  unsigned int hist[256];          // this CTA's digit histogram
  unsigned int chist[256];         // rank 0: the cluster's histogram
  int warp_gt[kSelWarps];
  int warp_eq[kSelWarps];
  uint32_t prefix;                 // rank 0: the decided key prefix
  int need;                        // rank 0: how many keys of that prefix are still needed
  int cta_gt[kClusterCtas];        // rank 0: each CTA's keys above T
  int cta_eq[kClusterCtas];        // rank 0: each CTA's keys equal to T
  alignas(16) uint32_t keys[kSmemKeys];   // read four at a time (16-byte vectors)
};
constexpr size_t kClusterSmemBytes = sizeof(ClusterSmem);
static_assert(kClusterSmemBytes <= 232448, "shared memory budget");
static_assert(offsetof(ClusterSmem, keys) % 16 == 0, "key vectors must be 16-byte aligned");

__global__ void __launch_bounds__(kSelThreads, 1)
    dsa_select_topk_cluster_kernel(const float* __restrict__ scores, const int32_t* __restrict__ q_pos, int n_q,
                                   int capacity, int top_k, int32_t* __restrict__ sel, int32_t* __restrict__ n_sel) {
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  extern __shared__ __align__(16) uint8_t smem_raw[];
  ClusterSmem& sm = *reinterpret_cast<ClusterSmem*>(smem_raw);
  const int rank = static_cast<int>(cluster.block_rank());
  const int t = blockIdx.x / kClusterCtas;
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  pdl_trigger();
  pdl_wait();
  // every branch below that returns before the cluster barriers is taken by
  // the whole cluster (it depends on the query only)
  if (t >= n_q) return;
  const int p = q_pos[t];
  int32_t* out = sel + static_cast<size_t>(t) * kMaxTopK;
  if (p < 0 || p >= capacity) {
    if (rank == 0) {
      for (int i = tid; i < kMaxTopK; i += kSelThreads) out[i] = -1;
      if (tid == 0) {
        if (n_sel != nullptr) n_sel[t] = 0;
        raise_error(MSA_DEVERR_QUERY_RANGE);
      }
    }
    return;
  }
  const int n = p + 1;
  if (n <= top_k) {                                   // every visible token is kept
    if (rank == 0) {
      for (int i = tid; i < kMaxTopK; i += kSelThreads) out[i] = i < n ? i : -1;
      if (tid == 0 && n_sel != nullptr) n_sel[t] = n;
    }
    return;
  }
  const int lo = static_cast<int>(static_cast<long long>(n) * rank / kClusterCtas);
  const int hi = static_cast<int>(static_cast<long long>(n) * (rank + 1) / kClusterCtas);
  const int m = hi - lo;
  const float* row = scores + static_cast<size_t>(t) * capacity + lo;
#pragma unroll 8
  for (int i = tid; i < m; i += kSelThreads) sm.keys[i] = score_key(__ldg(row + i));
  for (int i = m + tid; i < ((m + 3) & ~3); i += kSelThreads) sm.keys[i] = 0u;   // whole vectors for get4
  if (rank == 0) {
    for (int b = tid; b < 256; b += kSelThreads) sm.chist[b] = 0;
    if (tid == 0) {
      sm.prefix = 0;
      sm.need = top_k;
    }
  }
  cluster.sync();                                     // keys staged; rank 0's histogram and decision ready
  unsigned int* chist0 = cluster.map_shared_rank(sm.chist, 0);
  uint32_t prefix = 0, mask = 0;
  int need = top_k;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int b = tid; b < 256; b += kSelThreads) sm.hist[b] = 0;
    __syncthreads();
    for (int i = tid; i < m; i += kSelThreads) {
      const uint32_t key = sm.keys[i];
      if ((key & mask) == prefix) atomicAdd(&sm.hist[(key >> shift) & 255u], 1u);
    }
    __syncthreads();
    for (int b = tid; b < 256; b += kSelThreads) {
      const unsigned int c = sm.hist[b];
      if (c != 0u) atomicAdd(chist0 + b, c);
    }
    cluster.sync();                                   // every CTA's counts are in rank 0's histogram
    if (rank == 0) {
      if (warp == 0) {
        // lane l holds bins 255-8l .. 248-8l (descending); find the bin where
        // the count from the top reaches `need`
        const int need0 = sm.need;
        unsigned int c[8];
        unsigned int local = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          c[j] = sm.chist[255 - 8 * lane - j];
          local += c[j];
        }
        unsigned int incl = local;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const unsigned int v = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += v;
        }
        const unsigned int excl = incl - local;
        if (excl < static_cast<unsigned int>(need0) && incl >= static_cast<unsigned int>(need0)) {
          unsigned int cum = excl;
          int bin = 255 - 8 * lane;
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            if (cum + c[j] >= static_cast<unsigned int>(need0)) {
              bin = 255 - 8 * lane - j;
              break;
            }
            cum += c[j];
          }
          sm.prefix = sm.prefix | (static_cast<uint32_t>(bin) << shift);
          sm.need = need0 - static_cast<int>(cum);
        }
      }
      __syncthreads();                                // the decision is made: clear for the next digit
      for (int b = tid; b < 256; b += kSelThreads) sm.chist[b] = 0;
    }
    cluster.sync();                                   // the decided prefix is visible to every CTA
    prefix = *cluster.map_shared_rank(&sm.prefix, 0);
    need = *cluster.map_shared_rank(&sm.need, 0);
    mask |= 255u << shift;
  }
  const uint32_t T = prefix;
  const SmemKeys get{sm.keys};
  count_gt_eq(get, m, T, sm.warp_gt, sm.warp_eq);
  if (tid == 0) {
    int gt = 0, eq = 0;
    for (int w = 0; w < kSelWarps; ++w) {
      gt += sm.warp_gt[w];
      eq += sm.warp_eq[w];
    }
    *cluster.map_shared_rank(&sm.cta_gt[rank], 0) = gt;
    *cluster.map_shared_rank(&sm.cta_eq[rank], 0) = eq;
  }
  cluster.sync();                                     // every CTA's totals are at rank 0
  int gt0 = 0, eq0 = 0;
  for (int r = 0; r < rank; ++r) {
    gt0 += *cluster.map_shared_rank(&sm.cta_gt[r], 0);
    eq0 += *cluster.map_shared_rank(&sm.cta_eq[r], 0);
  }
  emit_counted(get, m, T, need, out, sm.warp_gt, sm.warp_eq, lo, gt0, eq0);
  if (rank == 0) {
    for (int i = top_k + tid; i < kMaxTopK; i += kSelThreads) out[i] = -1;
    if (tid == 0 && n_sel != nullptr) n_sel[t] = top_k;
  }
  cluster.sync();                                     // no CTA leaves while another reads its shared memory
}

}  // namespace dsa
}  // namespace msa
