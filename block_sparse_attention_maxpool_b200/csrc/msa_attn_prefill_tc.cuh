// Block-sparse GQA attention for prefill batches on the tcgen05 tensor cores.
//
// MSA pull request "Add MiniMax-M3 (MSA) support", section "Overview": each
// query attends to the rows of its selected blocks only (16 x 128 = 2048
// keys), shared by the 16 heads of its GQA group; the token-level causal mask
// applies inside the local block.
//
// Each (query, group) pair is one unit of work, computed transposed so that
// the 128 keys of a block sit on the MMA's M dimension and the group's 16
// heads on N:
//   S^T[keys][heads] = K_b . Q^T     (kind::f16, bf16, M=128 N=16 K=128)
// for all selected blocks at once (16 x 16 columns of tensor memory), then a
// softmax over the pair's 2048 keys per head (one max and one sum reduction
// across the 128 key lanes per pair, not per block), then
//   O^T[dims][heads] += V_b^T . P_b^T   (A = V_b, MN-major in shared memory)
// block by block as each P_b is written.  Every K and V element is read once
// per pair from L2/HBM (TMA, 128-byte swizzle) and once by the tensor cores.
//
// One persistent CTA per SM, warp-specialised so that no role waits on
// another's unrelated work: warp 0 loads Q and the K blocks (own ring of 32 KB
// stages), warp 2 loads the V blocks (own ring), warp 1 issues the score MMAs
// and warp 3 the PV MMAs (each tracks its own completions), warps 4-7 run the
// softmax and write the output.  Two 256-column tensor-memory slots alternate
// between consecutive pairs, so the scores of the next pair are computed while
// the softmax of the current one runs and its V blocks stream in.  Consecutive pairs of a CTA (and of
// neighbouring CTAs) are consecutive queries of one group, so their K/V
// blocks are shared in L2.
#pragma once

#include "msa_common.cuh"

namespace msa {
namespace pattn {

constexpr int kD = 128;
constexpr int kBlock = 128;
constexpr int kHpg = 16;
constexpr int kTopK = 16;
constexpr int kKRing = 2;                      // K block stages (scores consume them at once)
constexpr int kVRing = 4;                      // V block stages (wait on the softmax: deeper)
constexpr uint32_t kHalf = 128 * 128;          // [128 rows][64 bf16] = 16 KB
constexpr uint32_t kTile = 2 * kHalf;          // one K or V block
constexpr uint32_t kQHalf = 16 * 128;          // [16 heads][64 bf16] = 2 KB
constexpr uint32_t kQBytes = 2 * kQHalf;
constexpr int kPR = 3;                          // P tiles in flight per slot
constexpr uint32_t kPBytes = 2 * kQHalf;       // [16 heads][128 keys] bf16
constexpr int kThreads = 8 * 32;                // K loader, S MMA, V loader, PV MMA, 4 softmax warps
constexpr uint32_t kTmemCols = 512;            // two slots of 256 columns
constexpr uint32_t kIdescS = umma_idesc_bf16_f32(128, 16, false, false);
constexpr uint32_t kIdescPV = umma_idesc_bf16_f32(128, 16, true, false);

struct Layout {
  static constexpr uint32_t kKOff = 0;
  static constexpr uint32_t kVOff = kKOff + kKRing * kTile;
  static constexpr uint32_t kQOff = kVOff + kVRing * kTile;
  static constexpr uint32_t kPOff = kQOff + 2 * kQBytes;
  static constexpr uint32_t kRedOff = kPOff + 2 * kPR * kPBytes;
  static constexpr uint32_t kBarOff = kRedOff + 2 * 4 * 16 * 4;
  static constexpr uint32_t kEnd = kBarOff + 48 * 8;
  static constexpr size_t kBytes = kEnd + 1024;
};
static_assert(Layout::kBytes <= 232448, "shared memory budget");

struct Params {
  const int32_t* sel;        // [n_q][G][16]
  const int32_t* q_stream;
  const int32_t* q_pos;
  __nv_bfloat16* out;        // [n_q][Hq][D]
  int n_q, G, n_streams, capacity;
  float scale_log2;
  KvPages pages;             // block table of paged K/V caches (table null: contiguous)
};

struct PairInfo {
  int qi, g, p, s, nb;
  int blocks[kTopK];         // selected visible blocks (with a page, when paged), ascending
};

// Pair t -> (group, query); the selected blocks that are visible (and, for
// a paged cache, mapped to a page).
template <bool kPaged>
__device__ __forceinline__ void pair_info(const Params& P, int t, PairInfo& I, bool report) {
  I.g = t / P.n_q;
  I.qi = t - I.g * P.n_q;
  const int s = P.q_stream[I.qi];
  I.s = s;
  I.p = P.q_pos[I.qi];
  I.nb = 0;
  if (s < 0 || s >= P.n_streams || I.p < 0 || I.p >= P.capacity) {
    if (report && I.g == 0) raise_error(MSA_DEVERR_QUERY_RANGE);
    return;
  }
  const int nvis = I.p / kBlock + 1;
  const int32_t* sl = P.sel + (static_cast<size_t>(I.qi) * P.G + I.g) * kTopK;
#pragma unroll
  for (int j = 0; j < kTopK; ++j) {
    const int b = __ldg(sl + j);
    if (b < 0) continue;
    if (b >= nvis) {
      if (report) raise_error(MSA_DEVERR_SEL_RANGE);
      continue;
    }
    if (kPaged && kv_block_row(P.pages, s, I.g, b, P.G, P.capacity) < 0) {
      if (report) raise_error(MSA_DEVERR_PAGE_RANGE);
      continue;
    }
    I.blocks[I.nb++] = b;
  }
}

// Next pair (from *t on, stride gridDim.x) that has at least one block to
// attend; false at the end of this CTA's pairs.
template <bool kPaged>
__device__ __forceinline__ bool next_pair(const Params& P, int n_pairs, int& t, PairInfo& I) {
  while (t < n_pairs) {
    pair_info<kPaged>(P, t, I, false);
    t += gridDim.x;
    if (I.nb > 0) return true;
  }
  return false;
}

// kPaged: K/V are page pools addressed through P.pages (a separate
// instantiation, so the contiguous path carries no page-table code).
template <bool kPaged>
__global__ void __launch_bounds__(kThreads, 1)
    sparse_attn_prefill_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                                  const __grid_constant__ CUtensorMap tm_v, const Params P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Layout::kBarOff);
  static_assert(kKRing <= 4 && kVRing <= 4 && kPR <= 4, "barrier slots");
  uint64_t* kfull = bars;                // [kKRing]
  uint64_t* kempty = bars + 4;           // [kKRing]
  uint64_t* vfull = bars + 8;            // [kVRing]
  uint64_t* vempty = bars + 12;          // [kVRing]
  uint64_t* q_full = bars + 16;          // [2]
  uint64_t* q_empty = bars + 18;         // [2]
  uint64_t* s_full = bars + 20;          // [2]
  uint64_t* o_full = bars + 22;          // [2]
  uint64_t* slot_free = bars + 24;       // [2]
  uint64_t* p_full = bars + 26;          // [2][kPR]
  uint64_t* p_empty = bars + 34;         // [2][kPR]
  uint64_t* s_done = bars + 42;
  uint64_t* pv_done = bars + 43;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 44);
  float* red = reinterpret_cast<float*>(smem + Layout::kRedOff);   // [max|sum][4 warps][16]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_pairs = P.n_q * P.G;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kKRing; ++i) {
      mbar_init(&kfull[i], 1);
      mbar_init(&kempty[i], 1);
    }
    for (int i = 0; i < kVRing; ++i) {
      mbar_init(&vfull[i], 1);
      mbar_init(&vempty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&o_full[i], 1);
      mbar_init(&slot_free[i], 4);
    }
    for (int i = 0; i < 2 * kPR; ++i) {
      mbar_init(&p_full[i], 4);
      mbar_init(&p_empty[i], 1);
    }
    mbar_init(s_done, 1);
    mbar_init(pv_done, 1);
    mbar_fence_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, kTmemCols);
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const uint32_t k_base = smem_addr(smem + Layout::kKOff);
  const uint32_t v_base = smem_addr(smem + Layout::kVOff);
  const uint32_t q_base = smem_addr(smem + Layout::kQOff);
  const uint32_t p_base = smem_addr(smem + Layout::kPOff);
  pdl_trigger();
  pdl_wait();

  if (warp == 0 || warp == 2) {
    // --------------------- TMA loaders: warp 0 Q and K, warp 2 V --------------------
    if (lane == 0) {
      const bool is_k = warp == 0;
      const int ring_n = is_k ? kKRing : kVRing;
      uint64_t* rfull = is_k ? kfull : vfull;
      uint64_t* rempty = is_k ? kempty : vempty;
      uint8_t* rbase = smem + (is_k ? Layout::kKOff : Layout::kVOff);
      const CUtensorMap* map = is_k ? &tm_k : &tm_v;
      int t = blockIdx.x, u = 0, ring = 0;
      bool ok = true;
      PairInfo I;
      while (ok && next_pair<kPaged>(P, n_pairs, t, I)) {
        if (is_k) {
          const int slot = u & 1;
          if (u >= 2) ok = mbar_wait(&q_empty[slot], ((u >> 1) - 1) & 1);
          if (!ok) break;
          uint8_t* qdst = smem + Layout::kQOff + slot * kQBytes;
          const int qrow = I.qi * P.G * kHpg + I.g * kHpg;
          mbar_arrive_expect_tx(&q_full[slot], kQBytes);
          tma_load_2d(qdst, &tm_q, 0, qrow, &q_full[slot]);
          tma_load_2d(qdst + kQHalf, &tm_q, 64, qrow, &q_full[slot]);
        }
        for (int j = 0; j < I.nb && ok; ++j) {
          const int st = ring % ring_n;
          const int use = ring / ring_n;
          if (use > 0) ok = mbar_wait(&rempty[st], (use - 1) & 1);
          if (!ok) break;
          uint8_t* dst = rbase + st * kTile;
          // the host checks that every row fits 31 bits
          const int row = kPaged ? static_cast<int>(kv_block_row(P.pages, I.s, I.g, I.blocks[j], P.G, P.capacity))
                                 : (I.s * P.G + I.g) * P.capacity + I.blocks[j] * kBlock;
          mbar_arrive_expect_tx(&rfull[st], kTile);
          tma_load_2d(dst, map, 0, row, &rfull[st]);
          tma_load_2d(dst + kHalf, map, 64, row, &rfull[st]);
          ++ring;
        }
        ++u;
      }
      // no copy may still be landing when the CTA exits
      for (int j = max(0, ring - ring_n); j < ring; ++j) mbar_wait(&rfull[j % ring_n], (j / ring_n) & 1);
      if (is_k)
        for (int i = max(0, u - 2); i < u; ++i) mbar_wait(&q_full[i & 1], (i >> 1) & 1);
    }
  } else if (warp == 1) {
    // ------------------------- S^T = K Q^T for every selected block ----------------
    if (lane == 0) {
      int t = blockIdx.x, u = 0, ring = 0;
      bool ok = true;
      PairInfo I;
      while (ok && next_pair<kPaged>(P, n_pairs, t, I)) {
        const int slot = u & 1;
        if (u >= 2) ok = mbar_wait(&slot_free[slot], ((u >> 1) - 1) & 1);
        if (ok) ok = mbar_wait(&q_full[slot], (u >> 1) & 1);
        if (!ok) break;
        tc_fence_after();
        const uint32_t qb = q_base + slot * kQBytes;
        for (int j = 0; j < I.nb && ok; ++j) {
          const int st = ring % kKRing;
          ok = mbar_wait(&kfull[st], (ring / kKRing) & 1);
          if (!ok) break;
          tc_fence_after();
          const uint32_t kb = k_base + st * kTile;
          const uint32_t d = tmem_base + static_cast<uint32_t>(slot * 256 + 16 * j);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = (kk >> 2) * kHalf + (kk & 3) * 32;
            const uint32_t qoff = (kk >> 2) * kQHalf + (kk & 3) * 32;
            umma_f16_ss(d, umma_desc_sw128(kb + off), umma_desc_sw128(qb + qoff), kIdescS, kk != 0);
          }
          umma_commit(&kempty[st]);
          ++ring;
        }
        umma_commit(&s_full[slot]);
        umma_commit(&q_empty[slot]);
        ++u;
      }
      umma_commit(s_done);
      mbar_wait(s_done, 0);
    }
  } else if (warp == 3) {
    // ------------------------- O^T += V^T P^T block by block ----------------------
    if (lane == 0) {
      int t = blockIdx.x, u = 0, ring = 0;
      int pcnt[2] = {0, 0};
      bool ok = true;
      PairInfo I;
      while (ok && next_pair<kPaged>(P, n_pairs, t, I)) {
        const int sl = u & 1;
        const uint32_t d = tmem_base + static_cast<uint32_t>(sl * 256);
        for (int j = 0; j < I.nb && ok; ++j) {
          const int pr = pcnt[sl] % kPR;
          ok = mbar_wait(&p_full[sl * kPR + pr], (pcnt[sl] / kPR) & 1);
          const int st = ring % kVRing;
          if (ok) ok = mbar_wait(&vfull[st], (ring / kVRing) & 1);
          if (!ok) break;
          tc_fence_after();
          const uint32_t vb = v_base + st * kTile;
          const uint32_t pb = p_base + (sl * kPR + pr) * kPBytes;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            umma_f16_ss(d, umma_desc_sw128_mn(vb + kk * 2048, kHalf),
                        umma_desc_sw128(pb + (kk >> 2) * kQHalf + (kk & 3) * 32), kIdescPV, (j | kk) != 0);
          }
          umma_commit(&vempty[st]);
          umma_commit(&p_empty[sl * kPR + pr]);
          ++ring;
          ++pcnt[sl];
        }
        if (ok) umma_commit(&o_full[sl]);
        ++u;
      }
      umma_commit(pv_done);
      mbar_wait(pv_done, 0);
    }
  } else if (warp >= 4) {
    // --------------------------- softmax + output (warps 4-7) ---------------------
    const int q4 = warp & 3;                      // TMEM lane quarter of this warp
    const int row = q4 * 32 + lane;               // key row of a block / dim row of O
    const uint32_t lane_addr = static_cast<uint32_t>(q4 * 32) << 16;
    int u = 0;
    int pcnt[2] = {0, 0};
    bool ok = true;
    PairInfo I;
    for (int t = blockIdx.x; t < n_pairs; t += gridDim.x) {
      pair_info<kPaged>(P, t, I, q4 == 0 && lane == 0);
      __nv_bfloat16* out = P.out + (static_cast<size_t>(I.qi) * P.G * kHpg + I.g * kHpg) * kD + row;
      if (I.nb == 0) {
#pragma unroll
        for (int h = 0; h < kHpg; ++h) out[h * kD] = __float2bfloat16_rn(0.f);
        continue;
      }
      const int slot = u & 1;
      if (ok) ok = mbar_wait(&s_full[slot], (u >> 1) & 1);
      ok = __all_sync(0xffffffffu, ok);
      tc_fence_after();
      const uint32_t sbase = tmem_base + lane_addr + static_cast<uint32_t>(slot * 256);
      // pass 1: per-head maximum over this lane's keys of every block
      float mx[kHpg];
#pragma unroll
      for (int h = 0; h < kHpg; ++h) mx[h] = -INFINITY;
      for (int c = 0; c * 2 < I.nb; ++c) {
        float v[32];
        if (ok) {
          tmem_ld32(sbase + 32 * c, v);
          tmem_ld_wait();
        }
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const int j = c * 2 + i;
          if (ok && j < I.nb && I.blocks[j] * kBlock + row <= I.p) {
#pragma unroll
            for (int h = 0; h < kHpg; ++h) mx[h] = fmaxf(mx[h], v[i * 16 + h] * P.scale_log2);
          }
        }
      }
#pragma unroll
      for (int h = 0; h < kHpg; ++h) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], o));
      }
      if (lane < kHpg) {
        float m = mx[0];
#pragma unroll
        for (int h = 1; h < kHpg; ++h) m = lane == h ? mx[h] : m;
        red[q4 * 16 + lane] = m;
      }
      named_barrier_sync(1, 128);
#pragma unroll
      for (int h = 0; h < kHpg; ++h)
        mx[h] = fmaxf(fmaxf(red[h], red[16 + h]), fmaxf(red[32 + h], red[48 + h]));
      // pass 2: probabilities, their sums, and P tiles for the PV MMAs
      float sm[kHpg];
#pragma unroll
      for (int h = 0; h < kHpg; ++h) sm[h] = 0.f;
      const int half = row >> 6;
      const int chunk = (row & 63) >> 3;
      for (int c = 0; c * 2 < I.nb; ++c) {
        float v[32];
        if (ok) {
          tmem_ld32(sbase + 32 * c, v);
          tmem_ld_wait();
        }
        tc_fence_before();                        // these scores are read (block 0's columns take O next)
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const int j = c * 2 + i;
          if (j >= I.nb) break;
          const bool valid = ok && I.blocks[j] * kBlock + row <= I.p;
          const int pr = pcnt[slot] % kPR;
          if (ok && pcnt[slot] >= kPR) ok = mbar_wait(&p_empty[slot * kPR + pr], ((pcnt[slot] / kPR) - 1) & 1);
          ok = __all_sync(0xffffffffu, ok);
          uint8_t* pt = smem + Layout::kPOff + (slot * kPR + pr) * kPBytes + half * kQHalf + (row & 7) * 2;
#pragma unroll
          for (int h = 0; h < kHpg; ++h) {
            const float pe = valid ? exp2f(v[i * 16 + h] * P.scale_log2 - mx[h]) : 0.f;
            sm[h] += pe;
            *reinterpret_cast<__nv_bfloat16*>(pt + h * 128 + ((chunk ^ (h & 7)) << 4)) = __float2bfloat16_rn(pe);
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(&p_full[slot * kPR + pr]);
          ++pcnt[slot];
        }
      }
#pragma unroll
      for (int h = 0; h < kHpg; ++h) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sm[h] += __shfl_xor_sync(0xffffffffu, sm[h], o);
      }
      if (lane < kHpg) {
        float m = sm[0];
#pragma unroll
        for (int h = 1; h < kHpg; ++h) m = lane == h ? sm[h] : m;
        red[64 + q4 * 16 + lane] = m;
      }
      named_barrier_sync(1, 128);
      float inv[kHpg];
#pragma unroll
      for (int h = 0; h < kHpg; ++h) {
        const float L = red[64 + h] + red[80 + h] + red[96 + h] + red[112 + h];
        inv[h] = L > 0.f ? 1.f / L : 0.f;
      }
      // output: O^T[dim][head] / L
      if (ok) ok = mbar_wait(&o_full[slot], (u >> 1) & 1);
      ok = __all_sync(0xffffffffu, ok);
      tc_fence_after();
      float o[kHpg];
      if (ok) {
        tmem_ld16(tmem_base + lane_addr + static_cast<uint32_t>(slot * 256), o);
        tmem_ld_wait();
      }
#pragma unroll
      for (int h = 0; h < kHpg; ++h) out[h * kD] = __float2bfloat16_rn(ok ? o[h] * inv[h] : 0.f);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&slot_free[slot]);
      ++u;
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace pattn
}  // namespace msa
