// Block-sparse GQA attention over the selected key blocks.
//
// MSA pull request "Add MiniMax-M3 (MSA) support", section "Overview": the
// main attention runs only over the selected blocks (16 x 128 = 2048 K/V
// rows per query), shared by the 16 query heads of a GQA group; the
// token-level causal mask applies inside the local block.
//
// One CTA handles one (query, group) and a contiguous slice of its selected
// blocks (split-K across CTAs when there are few queries).  Each selected
// block's K and V rows (128 x 128 bf16 = 32 KB each) arrive by TMA as four
// 16 KB tiles with 128-byte swizzling, into a two-stage ring, so the next
// block streams in while the current one is used.  Eight warps each own 16
// key rows of the block: S = Q K^T (16 heads x 16 rows) and O += P V run as
// bf16 m16n8k16 tensor-core MMAs with fp32 accumulation; the softmax is the
// streaming (online) form in fp32 with base-2 exponentials.  Warps are merged
// through shared memory at the end; with several splits the CTA writes an
// unnormalised partial (max, sum, O) and attn_combine_kernel merges them.
#pragma once

#include "msa_common.cuh"

namespace msa {
namespace attn {

constexpr int kD = 128;
constexpr int kBlock = 128;
constexpr int kHpg = 16;                    // query heads per group
constexpr int kTopK = 16;
constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kRowsPerWarp = kBlock / kWarps;   // 16
constexpr uint32_t kTileBytes = kBlock * 64 * 2;   // [128 rows][64 dims] bf16 = 16 KB
constexpr uint32_t kStageBytes = 4 * kTileBytes;   // K lo, K hi, V lo, V hi
constexpr int kStages = 2;
constexpr int kOStride = kD + 4;                   // padded fp32 row in the merge buffer
constexpr size_t kSmemBytes = kStages * kStageBytes + 1024 /*align*/ + 64 /*barriers*/;

struct Params {
  const __nv_bfloat16* q;     // [n_q][Hq][D]
  const int32_t* sel;         // [n_q][G][16]
  const int32_t* q_stream;
  const int32_t* q_pos;
  __nv_bfloat16* out;         // [n_q][Hq][D]
  float* ws_o;                // [n_q*G][n_split][16][D]   (n_split > 1)
  float* ws_ml;               // [n_q*G][n_split][16][2]
  int n_q, G, n_streams, capacity, n_split, blocks_per_split;
  float scale_log2;           // softmax_scale * log2(e)
};

__device__ __forceinline__ float fast_exp2(float x) { return exp2f(x); }

__global__ void __launch_bounds__(kThreads, 1)
    sparse_attn_kernel(const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const Params P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int pair = blockIdx.x / P.n_split;
  const int split = blockIdx.x - pair * P.n_split;
  const int qi = pair / P.G;
  const int g = pair - qi * P.G;

  // ---- which blocks this CTA attends -------------------------------------
  const int s = P.q_stream[qi];
  const int p = P.q_pos[qi];
  const bool q_ok = s >= 0 && s < P.n_streams && p >= 0 && p < P.capacity;
  const int nvis = q_ok ? p / kBlock + 1 : 0;
  int blocks[kTopK];
  int nb = 0;
  if (q_ok) {
    const int32_t* sl = P.sel + static_cast<size_t>(pair) * kTopK;
    const int j0 = split * P.blocks_per_split;
    const int j1 = min(kTopK, j0 + P.blocks_per_split);
#pragma unroll
    for (int j = 0; j < kTopK; ++j) {
      if (j < j0 || j >= j1) continue;
      const int b = __ldg(sl + j);
      if (b < 0) continue;
      if (b >= nvis) {
        if (tid == 0) raise_error(MSA_DEVERR_SEL_RANGE);
        continue;
      }
      blocks[nb++] = b;
    }
  } else if (tid == 0 && split == 0 && g == 0) {
    raise_error(MSA_DEVERR_QUERY_RANGE);
  }
  const int row0 = q_ok ? (s * P.G + g) * P.capacity : 0;   // first cache row of (stream, group)

  if (tid == 0) {
    for (int st = 0; st < kStages; ++st) mbar_init(&full[st], 1);
    mbar_fence_init();
  }
  __syncthreads();
  auto issue = [&](int i) {
    const int st = i % kStages;
    uint8_t* dst = smem + st * kStageBytes;
    const int y = row0 + blocks[i] * kBlock;
    mbar_arrive_expect_tx(&full[st], kStageBytes);
    tma_load_2d(dst, &tm_k, 0, y, &full[st]);
    tma_load_2d(dst + kTileBytes, &tm_k, 64, y, &full[st]);
    tma_load_2d(dst + 2 * kTileBytes, &tm_v, 0, y, &full[st]);
    tma_load_2d(dst + 3 * kTileBytes, &tm_v, 64, y, &full[st]);
  };
  int issued = 0;   // copies started (thread 0 only)
  if (tid == 0) {
    for (; issued < min(nb, kStages); ++issued) issue(issued);
  }

  // ---- Q fragments (A operand, 16 heads x 128 dims) straight from global ----
  const int gr = lane >> 2;   // fragment row group
  const int tq = lane & 3;    // thread in quad
  uint32_t qa[8][4];
  {
    const __nv_bfloat16* qb = P.q + (static_cast<size_t>(qi) * P.G * kHpg + g * kHpg) * kD;
    const uint32_t* r0 = reinterpret_cast<const uint32_t*>(qb + gr * kD);
    const uint32_t* r1 = reinterpret_cast<const uint32_t*>(qb + (gr + 8) * kD);
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      const int c = ks * 8 + tq;   // 32-bit word index of dims (16ks + 2tq)
      qa[ks][0] = __ldg(r0 + c);
      qa[ks][1] = __ldg(r1 + c);
      qa[ks][2] = __ldg(r0 + c + 4);
      qa[ks][3] = __ldg(r1 + c + 4);
    }
  }

  float o[16][4];
#pragma unroll
  for (int n = 0; n < 16; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
  float m_run[2] = {-INFINITY, -INFINITY};
  float l_run[2] = {0.f, 0.f};
  bool ok = true;

  for (int i = 0; i < nb; ++i) {
    const int st = i % kStages;
    if (ok) ok = mbar_wait(&full[st], (i / kStages) & 1);
    if (ok) {
      const uint32_t kbase = smem_addr(smem + st * kStageBytes);
      const uint32_t vbase = kbase + 2 * kTileBytes;
      const int wr = warp * kRowsPerWarp;     // first key row of this warp in the block

      // S = Q K^T : two n-tiles of 8 key rows
      float sacc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const int half = ks >> 2;
        const int c0 = (ks & 3) * 2;
        const int mi = lane >> 3;
        const int r = wr + (mi >> 1) * 8 + (lane & 7);
        const int ch = c0 + (mi & 1);
        uint32_t b[4];
        ldmatrix_x4(b, kbase + half * kTileBytes + swz128(r, ch));
        mma_bf16_16816(sacc[0], qa[ks], b[0], b[1]);
        mma_bf16_16816(sacc[1], qa[ks], b[2], b[3]);
      }

      // causal mask inside the block, scale to base 2
      const int jb = blocks[i] * kBlock + wr;
      float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int j = jb + nt * 8 + tq * 2 + (e & 1);
          const float x = j <= p ? sacc[nt][e] * P.scale_log2 : -INFINITY;
          sacc[nt][e] = x;
          mx[e >> 1] = fmaxf(mx[e >> 1], x);
        }
      }
      float alpha[2], m_use[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 1));
        mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 2));
        const float m_new = fmaxf(m_run[h], mx[h]);
        m_use[h] = m_new == -INFINITY ? 0.f : m_new;
        alpha[h] = fast_exp2(m_run[h] - m_use[h]);   // 0 when m_run is -inf
        m_run[h] = m_new;
      }
      float rs[2] = {0.f, 0.f};
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float pe = fast_exp2(sacc[nt][e] - m_use[e >> 1]);
          sacc[nt][e] = pe;
          rs[e >> 1] += pe;
        }
      }
      l_run[0] = l_run[0] * alpha[0] + rs[0];
      l_run[1] = l_run[1] * alpha[1] + rs[1];
#pragma unroll
      for (int n = 0; n < 16; ++n) {
        o[n][0] *= alpha[0];
        o[n][1] *= alpha[0];
        o[n][2] *= alpha[1];
        o[n][3] *= alpha[1];
      }

      // O += P V : P (16 heads x 16 rows) is the A operand of one k-step
      uint32_t pa[4];
      pa[0] = pack_bf16(sacc[0][0], sacc[0][1]);
      pa[1] = pack_bf16(sacc[0][2], sacc[0][3]);
      pa[2] = pack_bf16(sacc[1][0], sacc[1][1]);
      pa[3] = pack_bf16(sacc[1][2], sacc[1][3]);
#pragma unroll
      for (int jn = 0; jn < 8; ++jn) {
        const int half = jn >> 2;
        const int c = (jn & 3) * 2;
        const int mi = lane >> 3;
        const int r = wr + (mi & 1) * 8 + (lane & 7);
        const int ch = c + (mi >> 1);
        uint32_t v[4];
        ldmatrix_x4_trans(v, vbase + half * kTileBytes + swz128(r, ch));
        const int nt = half * 8 + c;
        mma_bf16_16816(o[nt], pa, v[0], v[1]);
        mma_bf16_16816(o[nt + 1], pa, v[2], v[3]);
      }
    }
    __syncthreads();                       // every warp is done with stage st
    if (tid == 0 && ok && i + kStages < nb) issue(issued++);
  }
  if (tid == 0 && !ok) {
    // a wait gave up: let any copy still landing finish before the stage
    // memory is reused (bounded as well)
    for (int j = max(0, issued - kStages); j < issued; ++j) mbar_wait(&full[j % kStages], (j / kStages) & 1);
  }
  __syncthreads();

  // ---- merge the eight warps ----------------------------------------------
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    l_run[h] += __shfl_xor_sync(0xffffffffu, l_run[h], 1);
    l_run[h] += __shfl_xor_sync(0xffffffffu, l_run[h], 2);
  }
  float* so = reinterpret_cast<float*>(smem);                       // [8][16][kOStride]
  float* sml = so + kWarps * kHpg * kOStride;                       // [8][16][2]
  {
    float* ow = so + warp * kHpg * kOStride;
#pragma unroll
    for (int n = 0; n < 16; ++n) {
      const int col = n * 8 + tq * 2;
      *reinterpret_cast<float2*>(ow + gr * kOStride + col) = make_float2(o[n][0], o[n][1]);
      *reinterpret_cast<float2*>(ow + (gr + 8) * kOStride + col) = make_float2(o[n][2], o[n][3]);
    }
    if (tq == 0) {
      sml[(warp * kHpg + gr) * 2 + 0] = m_run[0];
      sml[(warp * kHpg + gr) * 2 + 1] = l_run[0];
      sml[(warp * kHpg + gr + 8) * 2 + 0] = m_run[1];
      sml[(warp * kHpg + gr + 8) * 2 + 1] = l_run[1];
    }
  }
  __syncthreads();
  {
    const int head = tid >> 4;            // 16 heads x 16 threads
    const int d0 = (tid & 15) * 8;        // 8 dims per thread
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) M = fmaxf(M, sml[(w * kHpg + head) * 2]);
    const float Mu = M == -INFINITY ? 0.f : M;
    float L = 0.f;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const float sc = fast_exp2(sml[(w * kHpg + head) * 2] - Mu);
      L += sml[(w * kHpg + head) * 2 + 1] * sc;
      const float* src = so + (w * kHpg + head) * kOStride + d0;
#pragma unroll
      for (int d = 0; d < 8; ++d) acc[d] += src[d] * sc;
    }
    if (P.n_split == 1) {
      const float inv = L > 0.f ? 1.f / L : 0.f;
      uint32_t pk[4];
#pragma unroll
      for (int d = 0; d < 4; ++d) pk[d] = pack_bf16(acc[2 * d] * inv, acc[2 * d + 1] * inv);
      __nv_bfloat16* dst = P.out + (static_cast<size_t>(pair) * kHpg + head) * kD + d0;
      *reinterpret_cast<uint4*>(dst) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
    } else {
      const size_t slot = (static_cast<size_t>(pair) * P.n_split + split) * kHpg + head;
      float* dst = P.ws_o + slot * kD + d0;
      *reinterpret_cast<float4*>(dst) = make_float4(acc[0], acc[1], acc[2], acc[3]);
      *reinterpret_cast<float4*>(dst + 4) = make_float4(acc[4], acc[5], acc[6], acc[7]);
      if ((tid & 15) == 0) {
        P.ws_ml[slot * 2 + 0] = M;
        P.ws_ml[slot * 2 + 1] = L;
      }
    }
  }
}

// Merge the split partials of every (query, head): one warp per head row,
// four dims per lane.
__global__ void __launch_bounds__(256) attn_combine_kernel(const float* __restrict__ ws_o,
                                                           const float* __restrict__ ws_ml,
                                                           __nv_bfloat16* __restrict__ out,
                                                           int n_pairs, int n_split) {
  const int w = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (w >= n_pairs * kHpg) return;
  const int pair = w / kHpg;
  const int head = w - pair * kHpg;
  float M = -INFINITY;
  for (int sp = 0; sp < n_split; ++sp)
    M = fmaxf(M, ws_ml[((static_cast<size_t>(pair) * n_split + sp) * kHpg + head) * 2]);
  const float Mu = M == -INFINITY ? 0.f : M;
  float L = 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int sp = 0; sp < n_split; ++sp) {
    const size_t slot = (static_cast<size_t>(pair) * n_split + sp) * kHpg + head;
    const float sc = exp2f(ws_ml[slot * 2] - Mu);
    L += ws_ml[slot * 2 + 1] * sc;
    const float4 v = *reinterpret_cast<const float4*>(ws_o + slot * kD + lane * 4);
    acc.x += v.x * sc;
    acc.y += v.y * sc;
    acc.z += v.z * sc;
    acc.w += v.w * sc;
  }
  const float inv = L > 0.f ? 1.f / L : 0.f;
  __nv_bfloat16* dst = out + (static_cast<size_t>(pair) * kHpg + head) * kD + lane * 4;
  *reinterpret_cast<uint2*>(dst) = make_uint2(pack_bf16(acc.x * inv, acc.y * inv), pack_bf16(acc.z * inv, acc.w * inv));
}

}  // namespace attn
}  // namespace msa
