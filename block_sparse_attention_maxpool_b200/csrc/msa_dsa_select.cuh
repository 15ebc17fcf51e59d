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
// L2).  A most-significant-digit-first radix select (4 passes of 8 bits,
// warp-aggregated shared-memory histograms) finds the k-th largest key T and
// how many keys equal to T are still needed.  A final pass walks the tokens
// in index order, one contiguous range per warp, and writes every token with
// key > T plus the first needed tokens with key == T, so the output is
// ascending with no sort.
#pragma once

#include "msa_common.cuh"

namespace msa {
namespace dsa {

constexpr int kSelThreads = 1024;
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kMaxTopK = 2048;                 // width of a selection row
constexpr int kSmemKeys = 48 * 1024;           // scores staged in shared memory up to this context

struct SelSmem {
  unsigned int hist[256];
  int warp_gt[kSelWarps];
  int warp_eq[kSelWarps];
  uint32_t prefix;
  int need;
  uint32_t keys[kSmemKeys];    // last: the unstaged kernel is launched without it
};
constexpr size_t kSelSmemStaged = sizeof(SelSmem);
constexpr size_t kSelSmemUnstaged = sizeof(SelSmem) - sizeof(uint32_t) * kSmemKeys;

// Order-preserving key of a score: larger score, larger key.  NaN maps to
// the key of -inf and -0 to the key of +0.
__device__ __forceinline__ uint32_t score_key(float x) {
  uint32_t u = __float_as_uint(x);
  if (x != x) u = 0xff800000u;
  if (x == 0.f) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

template <bool kStaged>
__device__ __forceinline__ uint32_t key_at(const SelSmem& sm, const float* row, int i) {
  if constexpr (kStaged) return sm.keys[i];
  return score_key(__ldg(row + i));
}

template <bool kStaged>
__global__ void __launch_bounds__(kSelThreads, 1)
    dsa_select_topk_kernel(const float* __restrict__ scores, const int32_t* __restrict__ q_pos, int n_q,
                           int capacity, int top_k, int32_t* __restrict__ sel, int32_t* __restrict__ n_sel) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  SelSmem& sm = *reinterpret_cast<SelSmem*>(smem_raw);
  const int t = blockIdx.x;
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
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
  if constexpr (kStaged) {
    for (int i = tid; i < n; i += kSelThreads) sm.keys[i] = score_key(__ldg(row + i));
  }
  if (tid == 0) {
    sm.prefix = 0;
    sm.need = top_k;
  }
  __syncthreads();

  // ---- radix select: the top_k-th largest key, 8 bits per pass ------------
  uint32_t mask = 0;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int b = tid; b < 256; b += kSelThreads) sm.hist[b] = 0;
    __syncthreads();
    const uint32_t prefix = sm.prefix;
    for (int base = 0; base < n; base += kSelThreads) {
      const int i = base + tid;
      const bool in = i < n;
      const uint32_t key = in ? key_at<kStaged>(sm, row, i) : 0u;
      const bool cand = in && (key & mask) == prefix;
      const unsigned int digit = cand ? (key >> shift) & 255u : 256u + lane;   // unique dummy digit
      const unsigned int peers = __match_any_sync(0xffffffffu, digit);
      if (cand && (__ffs(peers) - 1) == lane) atomicAdd(&sm.hist[digit], __popc(peers));
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
      const bool here = excl < static_cast<unsigned int>(need) && incl >= static_cast<unsigned int>(need);
      if (here) {
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
  const uint32_t T = sm.prefix;
  const int need_eq = sm.need;                        // keys equal to T still to keep (>= 1)

  // ---- emit in index order: one contiguous range of tokens per warp --------
  const int per_warp = (n + kSelWarps - 1) / kSelWarps;
  const int w0 = min(n, warp * per_warp);
  const int w1 = min(n, w0 + per_warp);
  int gt = 0, eq = 0;
  for (int base = w0; base < w1; base += 32) {
    const int i = base + lane;
    const uint32_t key = i < w1 ? key_at<kStaged>(sm, row, i) : 0u;
    gt += __popc(__ballot_sync(0xffffffffu, i < w1 && key > T));
    eq += __popc(__ballot_sync(0xffffffffu, i < w1 && key == T));
  }
  if (lane == 0) {
    sm.warp_gt[warp] = gt;
    sm.warp_eq[warp] = eq;
  }
  __syncthreads();
  int gt_before = 0, eq_before = 0;
  for (int w = 0; w < warp; ++w) {
    gt_before += sm.warp_gt[w];
    eq_before += sm.warp_eq[w];
  }
  const unsigned int lt_mask = (1u << lane) - 1u;
  for (int base = w0; base < w1; base += 32) {
    const int i = base + lane;
    const uint32_t key = i < w1 ? key_at<kStaged>(sm, row, i) : 0u;
    const bool is_gt = i < w1 && key > T;
    const bool is_eq = i < w1 && key == T;
    const unsigned int bgt = __ballot_sync(0xffffffffu, is_gt);
    const unsigned int beq = __ballot_sync(0xffffffffu, is_eq);
    const int my_eq = eq_before + __popc(beq & lt_mask);          // equal keys before token i
    const int my_gt = gt_before + __popc(bgt & lt_mask);
    if (is_gt || (is_eq && my_eq < need_eq)) out[my_gt + min(my_eq, need_eq)] = i;
    gt_before += __popc(bgt);
    eq_before += __popc(beq);
  }
  for (int i = top_k + tid; i < kMaxTopK; i += kSelThreads) out[i] = -1;
  if (tid == 0 && n_sel != nullptr) n_sel[t] = top_k;
}

}  // namespace dsa
}  // namespace msa
