// Block scores for prefill batches on the 5th-generation tensor cores.
//
// MSA pull request "Add MiniMax-M3 (MSA) support", section "Implementation":
// bs = maxpool_128(idx_q * idx_k^T + causal mask) plus the local bias, the
// same semantics for batch (prefill) and decode; scores accumulate in F32
// (MSA branch commit message).  For a prefill batch the score matrix of
// consecutive queries against the stream's keys is a dense contraction, so
// it runs as tcgen05 MMAs with the max-pool fused into the epilogue; the
// token-level score matrix is never written to memory.
//
// Precision.  The inputs are float32.  Every row (one query or one key, 128
// values) is scaled by an exact power of two 2^e so that its largest entry
// lies in [2^14, 2^15), then split as x * 2^e = hi + lo with hi = fp16(x*2^e)
// and lo = fp16(x*2^e - hi) (round to nearest even).  Three kind::f16 MMAs
// accumulate hi_q.hi_k + hi_q.lo_k + lo_q.hi_k in float32 tensor memory; the
// dropped lo_q.lo_k term and the fp16 rounding of lo leave a relative error
// near 2^-22 of sum |q_d k_d|, the same order as a float32 dot product.  The
// epilogue multiplies each score by 2^-(e_q + e_k) (exact) before pooling.
// The split kernels flag every 128-row tile with a nonzero lo part; a tile
// whose lo half is all zero (rows that fit fp16 after scaling: keys of the
// F16 cache, values on a coarse grid) is neither loaded nor multiplied, as
// its products add exactly zero.
//
// Launch sequence (all on the caller's stream):
//   tc_init_kernel         zero the per-call counters
//   tc_tile_info_kernel    per 128-query tile: its stream, visible blocks;
//                          queries of other streams go to a leftover list
//   tc_split_queries_kernel  hi/lo/scale of every (query, group) row, -inf
//                          for the blocks a query cannot see
//   tc_split_keys_kernel   hi/lo/scale of the keys the tiles will read
//   block_scores_tc_kernel persistent, warp-specialised tile kernel (one
//                          TMA producer with a ring of five 32 KB key
//                          slots, one MMA issuer, four epilogue warps)
//   block_scores_gemv_kernel (list mode) for the leftover queries
#pragma once

#include <cuda_fp16.h>

#include "msa_common.cuh"

namespace msa {
namespace tc {

constexpr int kDi = 128;
constexpr int kBlock = 128;
constexpr int kTileQ = 128;                 // queries per tile (MMA M)
constexpr int kChunk = 32;                  // key blocks per task
constexpr uint32_t kHalfBytes = 128 * 128;  // [128 rows][64 fp16] = 16 KB (one swizzle-128B box)
constexpr uint32_t kOperandBytes = 4 * kHalfBytes;   // hi (2 halves) + lo (2 halves) = 64 KB
constexpr uint32_t kSlotBytes = 2 * kHalfBytes;      // the hi or the lo half of a key block = 32 KB
constexpr int kSlots = 5;                            // key ring: a block takes 1 slot (hi) or 2 (hi, lo)
constexpr int kEpiGroups = 1;               // epilogue groups (group e drains accumulators acc % kEpiGroups == e)
constexpr int kThreads = (2 + 4 * kEpiGroups) * 32;   // producer, MMA, 2 x 4 epilogue warps
constexpr uint32_t kTmemCols = 256;         // two 128-column fp32 accumulators
constexpr uint32_t kIdesc = umma_idesc_f16_f32(128, 128);

struct SmemLayout {
  // all operand tiles 1024-byte aligned (swizzle atom)
  static constexpr uint32_t kA = 0;                                     // q hi|lo
  static constexpr uint32_t kB = kA + kOperandBytes;                    // key ring: kSlots x 32 KB
  static constexpr uint32_t kBars = kB + kSlots * kSlotBytes;
  static constexpr uint32_t kEnd = kBars + 256;
  static constexpr size_t kBytes = kEnd + 1024;                         // + alignment slack
};

static_assert(SmemLayout::kBytes <= 232448, "shared memory budget");
static_assert(2 * kSlots + 7 <= 32, "barrier slots");

// Workspace carve-up of the prefill block-score path (byte offsets).
struct Workspace {
  size_t counters, tile_stream, tile_nb, leftover, qscale, qhi, qlo, kscale, khi, klo, qlo_nz, klo_mask, total;
  int n_tiles, n_q_pad;
};

__host__ __device__ inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

__host__ inline Workspace workspace_layout(int n_q, int G, int S, int cap) {
  Workspace w;
  w.n_tiles = (n_q + kTileQ - 1) / kTileQ;
  w.n_q_pad = w.n_tiles * kTileQ;
  size_t o = 0;
  w.counters = o;    o = align256(o + sizeof(int) * (1 + S));
  w.tile_stream = o; o = align256(o + sizeof(int) * w.n_tiles);
  w.tile_nb = o;     o = align256(o + sizeof(int) * w.n_tiles);
  w.leftover = o;    o = align256(o + sizeof(int) * n_q);
  w.qscale = o;      o = align256(o + sizeof(float) * G * w.n_q_pad);
  w.qhi = o;         o = align256(o + sizeof(__half) * G * w.n_q_pad * kDi);
  w.qlo = o;         o = align256(o + sizeof(__half) * G * w.n_q_pad * kDi);
  w.kscale = o;      o = align256(o + sizeof(float) * static_cast<size_t>(S) * G * cap);
  w.khi = o;         o = align256(o + sizeof(__half) * static_cast<size_t>(S) * G * cap * kDi);
  w.klo = o;         o = align256(o + sizeof(__half) * static_cast<size_t>(S) * G * cap * kDi);
  w.qlo_nz = o;      o = align256(o + sizeof(int) * static_cast<size_t>(G) * w.n_tiles);
  w.klo_mask = o;    o = align256(o + sizeof(uint32_t) * static_cast<size_t>(S) * G * ((cap / kBlock + kChunk - 1) / kChunk));
  w.total = o;
  return w;
}

struct Params {
  const float* idx_q;       // [n_q][G][Di]
  const float* idx_k;       // [S][G][cap][Di] F32 cache, or its pages (null when idx_k16 is used)
  const __half* idx_k16;    // the same for the F16 cache variant (null for the F32 cache)
  const int32_t* q_stream;
  const int32_t* q_pos;
  float* bs;                // [n_q][G][nblk]
  int n_q, G, n_streams, capacity, nblk, n_tiles, n_q_pad, n_chunks;
  int* counters;            // [0] leftover count, [1 + s] visible blocks of stream s to convert
  int* tile_stream;         // [n_tiles]
  int* tile_nb;             // [n_tiles]
  int* leftover;            // [n_q]
  float* qscale;            // [G][n_q_pad]  2^-e_q
  __half* qhi;              // [G][n_q_pad][Di]
  __half* qlo;
  float* kscale;            // [S][G][cap]   2^-e_k
  __half* khi;              // [S][G][cap][Di]
  __half* klo;
  int* qlo_nz;              // [G][n_tiles]       some query row of the tile has a nonzero lo part
  uint32_t* klo_mask;       // [S][G][n_chunks]   bit b % 32: some key row of block b has a nonzero lo part
  int n_flags;              // entries of qlo_nz and klo_mask together (zeroed by tc_init_kernel)
  KvPages pages;            // block table of a paged key cache (table null: contiguous)
};

// Packed f32x2 multiply (sm_100 and later): two lanes per instruction.
__device__ __forceinline__ float2 fmul2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}

// max(a, b, c) in one instruction (three-input max.f32, sm_100 and later).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

__device__ __forceinline__ bool query_ok(const Params& P, int q, int& s, int& p) {
  s = P.q_stream[q];
  p = P.q_pos[q];
  return s >= 0 && s < P.n_streams && p >= 0 && p < P.capacity;
}

__global__ void tc_init_kernel(int* counters, int n, const Params P) {
  pdl_trigger();
  pdl_wait();
  for (int i = threadIdx.x; i < n; i += blockDim.x) counters[i] = 0;
  const int nq = P.G * P.n_tiles;
  for (int i = threadIdx.x; i < P.n_flags; i += blockDim.x) {
    if (i < nq) P.qlo_nz[i] = 0;
    else P.klo_mask[i - nq] = 0u;
  }
}

// Sets `bit` of *flags when this warp's split row has a lo part that is not
// all zero: the products with that 128-row tile's lo half are then needed
// (an all-zero lo half adds exactly zero, so its products are skipped).
__device__ __forceinline__ void flag_lo(const __half2 (&lo)[2], uint32_t* flags, uint32_t bit) {
  const uint32_t a = *reinterpret_cast<const uint32_t*>(&lo[0]) | *reinterpret_cast<const uint32_t*>(&lo[1]);
  if (__any_sync(0xffffffffu, (a & 0x7fff7fffu) != 0u) && (threadIdx.x & 31) == 0 && (*flags & bit) == 0u)
    atomicOr(flags, bit);
}

// One warp per tile of 128 consecutive queries.  The tile's stream is the
// stream of its first valid query; its visible-block count is the largest
// among that stream's queries in the tile.  Valid queries of any other
// stream are appended to the leftover list (scored by the streaming kernel).
__global__ void __launch_bounds__(256) tc_tile_info_kernel(const Params P) {
  pdl_trigger();
  pdl_wait();
  const int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (t >= P.n_tiles) return;
  int first = 0x7fffffff;
  for (int r = lane; r < kTileQ; r += 32) {
    const int q = t * kTileQ + r;
    int s, p;
    if (q < P.n_q && query_ok(P, q, s, p)) first = min(first, r);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) first = min(first, __shfl_xor_sync(0xffffffffu, first, o));
  if (first == 0x7fffffff) {
    if (lane == 0) {
      P.tile_stream[t] = -1;
      P.tile_nb[t] = 0;
    }
    return;
  }
  const int ts = P.q_stream[t * kTileQ + first];
  int nb = 0;
  for (int r = lane; r < kTileQ; r += 32) {
    const int q = t * kTileQ + r;
    int s, p;
    if (q < P.n_q && query_ok(P, q, s, p)) {
      if (s == ts) {
        nb = max(nb, p / kBlock + 1);
      } else {
        const int slot = atomicAdd(&P.counters[0], 1);
        P.leftover[slot] = q;
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) nb = max(nb, __shfl_xor_sync(0xffffffffu, nb, o));
  if (lane == 0) {
    P.tile_stream[t] = ts;
    P.tile_nb[t] = nb;
    atomicMax(&P.counters[1 + ts], nb);
  }
}

// Scale exponent of a row whose largest magnitude is m: 2^e * m in [2^14, 2^15).
__device__ __forceinline__ int row_exponent(float m) {
  if (!(m > 0.f) || !isfinite(m)) return 0;
  int E;
  frexpf(m, &E);                      // m = f * 2^E, f in [0.5, 1)
  return max(-126, min(126, 15 - E));
}

__device__ __forceinline__ float pow2f(int e) { return __int_as_float((127 + e) << 23); }

// Split 4 values of a row (this lane's share) into fp16 hi/lo with the row's
// power-of-two scale; returns the scale exponent.
__device__ __forceinline__ int split_row4(float4 x, __half2* hi, __half2* lo) {
  float m = fmaxf(fmaxf(fabsf(x.x), fabsf(x.y)), fmaxf(fabsf(x.z), fabsf(x.w)));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  const int e = row_exponent(m);
  const float sc = pow2f(e);
  const float a = x.x * sc, b = x.y * sc, c = x.z * sc, d = x.w * sc;
  const __half ha = __float2half_rn(a), hb = __float2half_rn(b), hc = __float2half_rn(c), hd = __float2half_rn(d);
  hi[0] = __halves2half2(ha, hb);
  hi[1] = __halves2half2(hc, hd);
  lo[0] = __halves2half2(__float2half_rn(a - __half2float(ha)), __float2half_rn(b - __half2float(hb)));
  lo[1] = __halves2half2(__float2half_rn(c - __half2float(hc)), __float2half_rn(d - __half2float(hd)));
  return e;
}

// One warp per (padded query, group) row.  Also writes -inf for the blocks
// past the query's position and flags invalid queries.
__global__ void __launch_bounds__(256) tc_split_queries_kernel(const Params P) {
  pdl_trigger();
  pdl_wait();
  const int w = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (w >= P.n_q_pad * P.G) return;
  const int q = w / P.G;
  const int g = w - q * P.G;
  int s = 0, p = 0;
  const bool real = q < P.n_q;
  const bool ok = real && query_ok(P, q, s, p);
  float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
  if (real) x = __ldg(reinterpret_cast<const float4*>(P.idx_q + (static_cast<size_t>(q) * P.G + g) * kDi) + lane);
  __half2 hi[2], lo[2];
  const int e = split_row4(x, hi, lo);
  const size_t row = static_cast<size_t>(g) * P.n_q_pad + q;
  *reinterpret_cast<uint2*>(P.qhi + row * kDi + lane * 4) =
      make_uint2(*reinterpret_cast<uint32_t*>(&hi[0]), *reinterpret_cast<uint32_t*>(&hi[1]));
  *reinterpret_cast<uint2*>(P.qlo + row * kDi + lane * 4) =
      make_uint2(*reinterpret_cast<uint32_t*>(&lo[0]), *reinterpret_cast<uint32_t*>(&lo[1]));
  if (lane == 0) P.qscale[row] = pow2f(-e);
  flag_lo(lo, reinterpret_cast<uint32_t*>(&P.qlo_nz[g * P.n_tiles + q / kTileQ]), 1u);
  if (!real) return;
  const int nvis = ok ? p / kBlock + 1 : 0;
  float* out = P.bs + (static_cast<size_t>(q) * P.G + g) * P.nblk;
  for (int b = nvis + lane; b < P.nblk; b += 32) out[b] = -INFINITY;
  if (!ok && lane == 0 && g == 0) raise_error(MSA_DEVERR_QUERY_RANGE);
}

// One warp per key row (stream, group, slot) that some tile will read.  The
// split rows are laid out by logical slot whatever the cache layout, so the
// tile kernel never sees the page table.  A row of a paged block with no
// valid page gets scale NaN: its scores drop out of the max-pool (the block
// scores -inf) and MSA_DEVERR_PAGE_RANGE is set.
__global__ void __launch_bounds__(256) tc_split_keys_kernel(const Params P) {
  pdl_trigger();
  pdl_wait();
  const long long w = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const long long rows = static_cast<long long>(P.n_streams) * P.G * P.capacity;
  if (w >= rows) return;
  const int j = static_cast<int>(w % P.capacity);
  const long long sg = w / P.capacity;
  const int s = static_cast<int>(sg / P.G);
  if (j >= P.counters[1 + s] * kBlock) return;
  long long src = w;
  if (P.pages.table != nullptr) {
    const int g = static_cast<int>(sg - static_cast<long long>(s) * P.G);
    const long long blk = kv_block_row(P.pages, s, g, j / kBlock, P.G, P.capacity);
    if (blk < 0) {
      *reinterpret_cast<uint2*>(P.khi + w * kDi + lane * 4) = make_uint2(0u, 0u);
      *reinterpret_cast<uint2*>(P.klo + w * kDi + lane * 4) = make_uint2(0u, 0u);
      if (lane == 0) {
        P.kscale[w] = __int_as_float(0x7fc00000);
        if ((j & (kBlock - 1)) == 0) raise_error(MSA_DEVERR_PAGE_RANGE);
      }
      return;
    }
    src = blk + (j & (kBlock - 1));
  }
  float4 x;
  if (P.idx_k16 != nullptr) {
    const uint2 raw = __ldcs(reinterpret_cast<const uint2*>(P.idx_k16 + src * kDi) + lane);
    const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&raw.x));
    const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&raw.y));
    x = make_float4(a.x, a.y, b.x, b.y);
  } else {
    x = __ldcs(reinterpret_cast<const float4*>(P.idx_k + src * kDi) + lane);
  }
  __half2 hi[2], lo[2];
  const int e = split_row4(x, hi, lo);
  *reinterpret_cast<uint2*>(P.khi + w * kDi + lane * 4) =
      make_uint2(*reinterpret_cast<uint32_t*>(&hi[0]), *reinterpret_cast<uint32_t*>(&hi[1]));
  *reinterpret_cast<uint2*>(P.klo + w * kDi + lane * 4) =
      make_uint2(*reinterpret_cast<uint32_t*>(&lo[0]), *reinterpret_cast<uint32_t*>(&lo[1]));
  if (lane == 0) P.kscale[w] = pow2f(-e);
  {
    const int blk = j / kBlock;
    flag_lo(lo, &P.klo_mask[sg * P.n_chunks + blk / kChunk], 1u << (blk % kChunk));
  }
}

// Task t -> (group, key chunk, query tile); consecutive tasks share a key
// chunk so the CTAs reading it run together and hit in L2.
__device__ __forceinline__ void task_coords(const Params& P, int t, int& g, int& chunk, int& tile) {
  tile = t % P.n_tiles;
  const int gc = t / P.n_tiles;
  chunk = gc % P.n_chunks;
  g = gc / P.n_chunks;
}

// Blocks [b0, b1) of one task (empty when the tile sees fewer blocks).
__device__ __forceinline__ void task_range(const Params& P, int tile, int chunk, int& b0, int& b1) {
  const int nb = P.tile_nb[tile];
  b0 = chunk * kChunk;
  b1 = min(nb, b0 + kChunk);
}

__global__ void __launch_bounds__(kThreads, 1)
    block_scores_tc_kernel(const __grid_constant__ CUtensorMap tm_qhi, const __grid_constant__ CUtensorMap tm_qlo,
                           const __grid_constant__ CUtensorMap tm_khi, const __grid_constant__ CUtensorMap tm_klo,
                           const Params P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SmemLayout::kBars);
  uint64_t* full = bars;                  // [kSlots]  key half-tile landed
  uint64_t* empty = full + kSlots;        // [kSlots]  MMAs done reading it
  uint64_t* a_full = empty + kSlots;      // query tile landed
  uint64_t* a_empty = a_full + 1;         // MMAs done reading the query tile
  uint64_t* acc_full = a_empty + 1;       // [2] accumulator ready
  uint64_t* acc_empty = acc_full + 2;     // [2] accumulator drained
  uint64_t* mma_done = acc_empty + 2;     // every MMA of this CTA finished
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  int* abort_flag = reinterpret_cast<int*>(mma_done + 2);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_tasks = P.G * P.n_chunks * P.n_tiles;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kSlots; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(a_full, 1);
    mbar_init(a_empty, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 4);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, kTmemCols);
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  volatile int* abort_v = abort_flag;
  pdl_trigger();
  pdl_wait();

  if (warp == 0) {
    // ------------------------------ TMA producer ------------------------------
    if (lane == 0) {
      int slot = 0, a_use = 0;
      for (int t = blockIdx.x; t < n_tasks && !*abort_v; t += gridDim.x) {
        int g, chunk, tile, b0, b1;
        task_coords(P, t, g, chunk, tile);
        task_range(P, tile, chunk, b0, b1);
        if (b0 >= b1) continue;
        const int s = P.tile_stream[tile];
        // the task's lo flags, loaded before the wait so their latency hides behind it
        const bool q_lo = __ldcg(&P.qlo_nz[g * P.n_tiles + tile]) != 0;
        const uint32_t kmask = __ldcg(P.klo_mask + (static_cast<size_t>(s) * P.G + g) * P.n_chunks + chunk);
        if (a_use > 0 && !mbar_wait(a_empty, (a_use - 1) & 1)) { *abort_v = 1; break; }
        const int qrow = g * P.n_q_pad + tile * kTileQ;
        mbar_arrive_expect_tx(a_full, q_lo ? kOperandBytes : kOperandBytes / 2);
        tma_load_2d(smem + SmemLayout::kA, &tm_qhi, 0, qrow, a_full);
        tma_load_2d(smem + SmemLayout::kA + kHalfBytes, &tm_qhi, 64, qrow, a_full);
        if (q_lo) {
          tma_load_2d(smem + SmemLayout::kA + 2 * kHalfBytes, &tm_qlo, 0, qrow, a_full);
          tma_load_2d(smem + SmemLayout::kA + 3 * kHalfBytes, &tm_qlo, 64, qrow, a_full);
        }
        ++a_use;
        const size_t krow0 = (static_cast<size_t>(s) * P.G + g) * P.capacity;
        bool stop = false;
        for (int b = b0; b < b1 && !stop; ++b) {
          const int krow = static_cast<int>(krow0) + b * kBlock;
          const bool k_lo = ((kmask >> (b - b0)) & 1u) != 0u;
          // the hi half of the key block, then (when nonzero) its lo half, one slot each
          for (int h = 0; h < (k_lo ? 2 : 1); ++h, ++slot) {
            const int st = slot % kSlots;
            const int use = slot / kSlots;
            if (use > 0 && !mbar_wait(&empty[st], (use - 1) & 1)) { *abort_v = 1; stop = true; break; }
            uint8_t* dst = smem + SmemLayout::kB + st * kSlotBytes;
            const CUtensorMap* map = h == 0 ? &tm_khi : &tm_klo;
            mbar_arrive_expect_tx(&full[st], kSlotBytes);
            tma_load_2d(dst, map, 0, krow, &full[st]);
            tma_load_2d(dst + kHalfBytes, map, 64, krow, &full[st]);
          }
        }
        if (stop) break;
      }
      // let copies still landing finish before the CTA can exit
      for (int j = max(0, slot - kSlots); j < slot; ++j) mbar_wait(&full[j % kSlots], (j / kSlots) & 1);
      if (a_use > 0) mbar_wait(a_full, (a_use - 1) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issuer --------------------------------
    if (lane == 0) {
      int slot = 0, a_use = 0, acc = 0;
      const uint32_t a_base = smem_addr(smem + SmemLayout::kA);
      for (int t = blockIdx.x; t < n_tasks && !*abort_v; t += gridDim.x) {
        int g, chunk, tile, b0, b1;
        task_coords(P, t, g, chunk, tile);
        task_range(P, tile, chunk, b0, b1);
        if (b0 >= b1) continue;
        const int s = P.tile_stream[tile];
        const bool q_lo = __ldcg(&P.qlo_nz[g * P.n_tiles + tile]) != 0;
        const uint32_t kmask = __ldcg(P.klo_mask + (static_cast<size_t>(s) * P.G + g) * P.n_chunks + chunk);
        if (!mbar_wait(a_full, a_use & 1)) { *abort_v = 1; break; }
        tc_fence_after();
        for (int b = b0; b < b1; ++b, ++acc) {
          const bool k_lo = ((kmask >> (b - b0)) & 1u) != 0u;
          const int st_hi = slot % kSlots;
          const int st_lo = (slot + 1) % kSlots;
          const int buf = acc & 1;
          if (!mbar_wait(&full[st_hi], (slot / kSlots) & 1)) { *abort_v = 1; break; }
          if (k_lo && !mbar_wait(&full[st_lo], ((slot + 1) / kSlots) & 1)) { *abort_v = 1; break; }
          if (acc >= 2 && !mbar_wait(&acc_empty[buf], ((acc >> 1) - 1) & 1)) { *abort_v = 1; break; }
          tc_fence_after();
          const uint32_t b_hi = smem_addr(smem + SmemLayout::kB + st_hi * kSlotBytes);
          const uint32_t b_lo = smem_addr(smem + SmemLayout::kB + st_lo * kSlotBytes);
          const uint32_t d = tmem_base + static_cast<uint32_t>(buf * 128);
          // three products: hi.hi, hi.lo, lo.hi; 8 K-steps of 16 each; a
          // product whose lo operand is all zero adds exactly zero and is skipped
#pragma unroll
          for (int pass = 0; pass < 3; ++pass) {
            if ((pass == 1 && !k_lo) || (pass == 2 && !q_lo)) continue;
            const uint32_t a_off = pass == 2 ? 2 * kHalfBytes : 0;   // q lo for the last pass
            const uint32_t bb = pass == 1 ? b_lo : b_hi;              // k lo for the second pass
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint32_t koff = (kk >> 2) * kHalfBytes + (kk & 3) * 32;
              umma_f16_ss(d, umma_desc_sw128(a_base + a_off + koff), umma_desc_sw128(bb + koff), kIdesc,
                          (pass | kk) != 0);
            }
          }
          umma_commit(&empty[st_hi]);    // key slots may be overwritten once these MMAs finish
          if (k_lo) umma_commit(&empty[st_lo]);
          umma_commit(&acc_full[buf]);   // accumulator ready for the epilogue
          slot += k_lo ? 2 : 1;
        }
        umma_commit(a_empty);            // query tile free after the task's last MMA
        ++a_use;
      }
      // tensor memory is released below: wait until no MMA is in flight
      umma_commit(mma_done);
      mbar_wait(mma_done, 0);
    }
  } else {
    // ---------------- epilogue: kEpiGroups groups of 4 warps ----------------
    // Group e drains the accumulators of blocks acc with acc % kEpiGroups == e.
    const int quarter = warp & 3;                 // TMEM lane quarter this warp may read
    const int group = (warp - 2) >> 2;
    const int row = quarter * 32 + lane;          // query row within the tile
    int acc = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < n_tasks; t += gridDim.x) {
      int g, chunk, tile, b0, b1;
      task_coords(P, t, g, chunk, tile);
      task_range(P, tile, chunk, b0, b1);
      if (b0 >= b1) continue;
      const int ts = P.tile_stream[tile];
      const int q = tile * kTileQ + row;
      int s = -1, p = -1;
      const bool active = q < P.n_q && query_ok(P, q, s, p) && s == ts;
      const int nvis = active ? p / kBlock + 1 : 0;
      const float qs = P.qscale[static_cast<size_t>(g) * P.n_q_pad + q];
      float* out = P.bs + (static_cast<size_t>(q) * P.G + g) * P.nblk;
      const float* ksc_base = P.kscale + (static_cast<size_t>(ts < 0 ? 0 : ts) * P.G + g) * P.capacity;
      for (int b = b0; b < b1; ++b, ++acc) {
        const int buf = acc & 1;
        if (kEpiGroups > 1 && (acc % kEpiGroups) != group) continue;
        if (ok && !*abort_v) ok = mbar_wait(&acc_full[buf], (acc >> 1) & 1);
        ok = __all_sync(0xffffffffu, ok);   // the TMEM loads below are warp-collective
        if (!ok) *abort_v = 1;
        tc_fence_after();
        float m = -INFINITY;
        const float4* ksc = reinterpret_cast<const float4*>(ksc_base + static_cast<size_t>(b) * kBlock);
        const int jmax = p - b * kBlock;   // last visible key of this block (row-local)
        if (ok) {
          float v[4][32];
#pragma unroll
          for (int c = 0; c < 4; ++c)
            tmem_ld32(tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + buf * 128 + c * 32, v[c]);
          tmem_ld_wait();
          // scale each key's score by its exact power of two, then the max over
          // the visible keys (only a row's local block is cut)
          const bool cut = __any_sync(0xffffffffu, active && jmax < kBlock - 1);
          float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
          for (int c = 0; c < 4; ++c) {
#pragma unroll
            for (int i4 = 0; i4 < 8; ++i4) {
              const float4 k4 = __ldg(ksc + c * 8 + i4);
              const float2 x01 = fmul2(make_float2(v[c][i4 * 4], v[c][i4 * 4 + 1]), make_float2(k4.x, k4.y));
              const float2 x23 = fmul2(make_float2(v[c][i4 * 4 + 2], v[c][i4 * 4 + 3]), make_float2(k4.z, k4.w));
              float x[4] = {x01.x, x01.y, x23.x, x23.y};
              if (cut) {
#pragma unroll
                for (int u = 0; u < 4; ++u) x[u] = c * 32 + i4 * 4 + u <= jmax ? x[u] : -INFINITY;
              }
              m4[i4 & 3] = fmax3(m4[i4 & 3], fmaxf(x[0], x[1]), fmaxf(x[2], x[3]));
            }
          }
          m = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[buf]);
        if (active && b < nvis) {
          float r = m * qs;
          if (b == nvis - 1) r += MSA_LOCAL_BIAS;
          out[b] = r;
        }
      }
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace tc
}  // namespace msa
