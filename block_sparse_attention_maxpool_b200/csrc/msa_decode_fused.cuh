// The whole decode step as one persistent kernel.
//
// MSA pull request "Add MiniMax-M3 (MSA) support": a decode step appends the
// new token's indexer key and K/V rows, scores the blocks
// (maxpool_128(idx_q * idx_k^T + causal mask) + local bias), keeps the
// top-16 per group and attends over the selected blocks.  The same step
// runs here as three or four phases of one cooperative launch (one CTA per SM, all
// resident), separated by grid-wide barriers instead of kernel boundaries:
//
//   1. append      one warp per (token, group) row, grid-stride
//   2. scores      the streaming block-score body (F32 keys), every CTA
//   3. select      each attention CTA ranks the pairs its units touch, at
//                  the start of phase 4 (no barrier); for batches whose
//                  CTA shares touch more than 8 pairs, one warp per
//                  (query, group), grid-stride, then a barrier
//   4. attention   the stream-K decode body over (pair, block) units, pairs
//                  cut between CTAs merged by the CTA holding their first unit
//
// Each phase computes exactly what its standalone kernel computes, with the
// same launch shape where it matters (the score body's task split and the
// attention's unit split use every CTA of the grid, as the standalone
// launches do), so the results are bit-identical.  The grid barrier is a
// counter and a generation word in the caller's workspace (zeroed before
// the launch); a CTA waiting on it gives up after MSA's bounded wait,
// records MSA_DEVERR_TIMEOUT and returns, so no phase can hang the GPU.
#pragma once

#include "msa_append.cuh"
#include "msa_attn_decode_sk.cuh"
#include "msa_common.cuh"
#include "msa_scores_gemv.cuh"
#include "msa_select.cuh"

namespace msa {
namespace fused {

using ScoreKey = float;
constexpr int kScoreStages = 4;
constexpr int kScoreWarps = 8;
constexpr int kThreads = dattn::kThreads;                      // the widest phase (attention)
constexpr size_t kScoreSmem = sizeof(gemv::Smem<ScoreKey, kScoreStages, kScoreWarps>);
constexpr size_t kSmemBytes = dattn::Layout::kBytes > kScoreSmem + 1024 ? dattn::Layout::kBytes : kScoreSmem + 1024;
static_assert(kThreads >= (kScoreWarps + 1) * 32, "the score body needs its producer warp");
static_assert((kThreads / 32) * sel::KeySmem<32>::kBytesPerWarp <= kSmemBytes, "the top-16 keys of every warp");

struct Params {
  // phase 1: appends of the new tokens
  float* idx_k_cache;
  const float* idx_k_new;
  uint8_t* k_cache;
  uint8_t* v_cache;
  const uint8_t* k_new;
  const uint8_t* v_new;
  const int32_t* tok_stream;
  const int32_t* tok_pos;
  int n_tok;
  // phases 2-4
  gemv::Params<ScoreKey> scores;     // writes block_scores
  int32_t* sel;
  int32_t* n_sel;
  dattn::Params attn;                // reads sel, writes out and the partials
  // grid barrier words (workspace, zeroed before the launch)
  unsigned int* bar_count;
  unsigned int* bar_gen;
  long long wait_cycles;             // give-up limit of a grid-barrier wait (SM clock cycles)
};

__device__ __forceinline__ unsigned int ld_acquire_gpu(const unsigned int* p) {
  unsigned int v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Orders this thread's generic-proxy global writes before later async-proxy
// (bulk copy, TMA) reads of the same memory by any CTA.
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// Arrival on the barrier counter: releases this CTA's writes and acquires
// those of the CTAs that arrived before (the last arriver passes them on).
__device__ __forceinline__ unsigned int atom_add_acq_rel_gpu(unsigned int* p, unsigned int v) {
  unsigned int old;
  asm volatile("atom.add.acq_rel.gpu.global.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}
__device__ __forceinline__ void st_release_gpu(unsigned int* p, unsigned int v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ void st_relaxed_gpu(unsigned int* p, unsigned int v) {
  asm volatile("st.relaxed.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Grid-wide barrier over `expected` arrivals (the n_cta resident CTAs).
// The CTA's threads meet at __syncthreads, then thread 0 arrives with an
// acquire-release add on the counter; the arrival that completes the count
// resets the counter and publishes the next generation with a release
// store, the others poll it with acquire loads for at most `limit` SM clock
// cycles.  gen: the generation this CTA last saw.  proxy_fence: the phase
// wrote global memory that async copies (bulk, TMA) read afterwards.  False,
// for every thread of the CTA, when the wait timed out (MSA_DEVERR_TIMEOUT
// recorded).
__device__ __forceinline__ bool grid_barrier(unsigned int* bar_count, unsigned int* bar_gen, unsigned int expected,
                                             long long limit, unsigned int& gen, int* flag, bool proxy_fence) {
  if (proxy_fence) fence_proxy_async_global();
  __syncthreads();
  if (threadIdx.x == 0) {
    bool ok = true;
    const unsigned int target = gen + 1;
    if (atom_add_acq_rel_gpu(bar_count, 1u) == expected - 1) {
      st_relaxed_gpu(bar_count, 0u);
      st_release_gpu(bar_gen, target);
    } else {
      const long long t0 = clock64();
      while (ld_acquire_gpu(bar_gen) < target) {
        if (clock64() - t0 > limit) {
          raise_error(MSA_DEVERR_TIMEOUT);
          ok = false;
          break;
        }
      }
    }
    gen = target;
    *flag = ok ? 1 : 0;
  }
  __syncthreads();
  return *flag != 0;
}

__device__ __forceinline__ bool grid_barrier(const Params& F, unsigned int n_cta, unsigned int& gen, int* flag,
                                             bool proxy_fence) {
  return grid_barrier(F.bar_count, F.bar_gen, n_cta, F.wait_cycles, gen, flag, proxy_fence);
}

__global__ void __launch_bounds__(kThreads, 1)
    decode_step_fused_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                             const __grid_constant__ CUtensorMap tm_q, const Params F) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ int barrier_flag;
  const int cta = blockIdx.x;
  const unsigned int n_cta = gridDim.x;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const long long gwarp = static_cast<long long>(cta) * (kThreads / 32) + warp;
  const long long n_gwarps = static_cast<long long>(n_cta) * (kThreads / 32);
  const int G = F.scores.G;
  unsigned int gen = 0;

  // ---- 1. append the new tokens' indexer keys and K/V rows ----------------
  for (long long w = gwarp; w < static_cast<long long>(F.n_tok) * G; w += n_gwarps) {
    const KvPages none{nullptr, 0};
    append_row(reinterpret_cast<uint8_t*>(F.idx_k_cache), reinterpret_cast<const uint8_t*>(F.idx_k_new), nullptr,
               nullptr, F.tok_stream, F.tok_pos, F.scores.n_streams, G, F.scores.capacity, 128 * 4, none,
               static_cast<int>(w), lane);
    append_row(F.k_cache, F.k_new, F.v_cache, F.v_new, F.tok_stream, F.tok_pos, F.scores.n_streams, G,
               F.scores.capacity, 128 * 2, none, static_cast<int>(w), lane);
  }
  if (!grid_barrier(F, n_cta, gen, &barrier_flag, true)) return;

  // ---- 2. block scores -------------------------------------------------------
  gemv::block_scores_gemv_body<ScoreKey, kScoreStages, kScoreWarps>(F.scores, smem, cta, static_cast<int>(n_cta));
  fence_proxy_async_smem();
  __syncthreads();
  if (threadIdx.x == 0) gemv::block_scores_gemv_release<ScoreKey, kScoreStages, kScoreWarps>(smem);
  if (!grid_barrier(F, n_cta, gen, &barrier_flag, false)) return;

  // ---- 3 + 4. top-16 and attention over the selected blocks ---------------
  // (pairs cut between CTAs are merged inside the attention body)
  if (F.attn.bs != nullptr) {
    // every CTA ranks the pairs its units touch, as the attention kernel
    // of msa_select_attn_decode does: no grid barrier between the two
    if (cta < F.attn.n_cta) dattn::sparse_attn_decode_sk_body<false, true>(&tm_k, &tm_v, &tm_q, F.attn, smem, cta);
    return;
  }
  const int n_pairs = F.scores.n_q * G;
  uint64_t* wsm = reinterpret_cast<uint64_t*>(smem + warp * sel::select_smem_per_warp(F.scores.nblk));
  for (long long w = gwarp; w < n_pairs; w += n_gwarps)
    sel::select_pair_any(F.scores.bs, F.scores.q_pos, G, F.scores.nblk, F.scores.capacity,
                         F.sel + static_cast<size_t>(w) * sel::kTopK, F.n_sel != nullptr ? F.n_sel + w : nullptr,
                         static_cast<int>(w), lane, wsm);
  if (!grid_barrier(F, n_cta, gen, &barrier_flag, false)) return;
  if (cta < F.attn.n_cta) dattn::sparse_attn_decode_sk_body<false, false>(&tm_k, &tm_v, &tm_q, F.attn, smem, cta);
}

// The library's bounded waits driven to their limit: every CTA of a
// cooperative grid (one per SM) meets at the grid barrier above with one
// more arrival expected than the grid gives, so no CTA sees the next
// generation; then thread 0 of each CTA waits on an mbarrier nothing
// arrives on.  Each wait gives up after `limit` cycles, records
// MSA_DEVERR_TIMEOUT, and the kernel returns.  No copy or MMA is in flight
// at either wait.  bar: two zeroed words (counter, generation).
__global__ void __launch_bounds__(32, 1) wait_selftest_kernel(unsigned int* bar, long long limit) {
  __shared__ int barrier_flag;
  __shared__ __align__(8) uint64_t never;
  unsigned int gen = 0;
  const bool passed = grid_barrier(bar, bar + 1, gridDim.x + 1, limit, gen, &barrier_flag, false);
  if (threadIdx.x == 0) {
    mbar_init(&never, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    const bool arrived = mbar_wait(&never, 0, limit);
    mbar_inval(&never);
    if (passed || arrived) bar[2] = 1u;          // a wait that should have run out did not
  }
}

}  // namespace fused
}  // namespace msa
