// Block-sparse GQA attention for prefill batches: query tiles over the union
// of their selected blocks (tcgen05, flash-style).
//
// MSA pull request "Add MiniMax-M3 (MSA) support", section "Overview": each
// query attends to the rows of its selected blocks only, shared by the 16
// heads of its GQA group; the token-level causal mask applies inside the
// local block.
//
// A tile is 8 consecutive queries of one group: 8 x 16 = 128 query-head
// rows, the M dimension of every MMA.  plan_tiles_kernel, launched just
// before, builds each tile's union of the 8 queries' selected blocks, each
// with an 8-bit mask of the queries that selected it (queries of different
// streams form separate segments of the union).  For every block b of the
// union:
//   S = Q . K_b^T          M=128 rows, N=128 keys, K=128 dims (TMEM, f32)
//   P = exp2(S - m)        masked: a row keeps only keys of blocks its query
//                          selected and j <= its position; one thread per
//                          row; bf16, written back over S in tensor memory
//   O += P . V_b           M=128 rows, N=128 dims, K=128 keys: A (P) from
//                          tensor memory, B (V) from shared memory
// with an online softmax per row whose reference max m is raised (and O
// rescaled in tensor memory) only when a block's max exceeds it by more than
// 2^8, so P stays below 256 and the rescale is rare.  Each K and V block is
// read once per tile instead of once per (query, group).
//
// Pipelining: three S/P buffers in tensor memory; S of block b needs only
// the P . V of block b - 3 done, so the S MMAs run up to two blocks ahead of
// P . V and the softmax warps can drift two blocks apart.  A warp whose two
// queries did not select a block writes zeros without reading S or
// computing exponentials.  The Q tile is released after the tile's last S
// MMA, so the next tile's Q loads while the last blocks' softmax runs.
//
// S and P . V are issued by two threads (warps 1 and 3).  On B200 the
// tensor pipe drains, ~300 cycles, whenever one issuing thread changes
// operand configuration (S: both operands from shared memory, K-major;
// P . V: A from tensor memory, B MN-major), but streams of two threads
// interleave at full rate.  What remains is the hand-off latency: a commit
// or an mbarrier arrive reaches its waiter after ~230 cycles, and three S
// buffers hide it only in part.
//
// Paged caches (kPaged): the loaders address blocks through the block table;
// the planner leaves out a selected block whose page is missing (and sets
// MSA_DEVERR_PAGE_RANGE), as if the query had not selected it.
//
// Warp roles: 0 loads the Q tile and the K blocks, 1 issues S, 2 loads the
// V blocks, 3 issues P . V, 4-7 run the softmax and write the output (one
// TMEM lane quarter each).  Shared memory: Q 32 KB, K ring 3 x 32 KB, V ring
// 2 x 32 KB.  Tensor memory: three S/P buffers and O (all 512 columns).
//
// Per block, a softmax warp whose queries selected it loads S, takes the
// row max and computes 128 exponentials per row; one whose queries did not
// writes zeros.  The
// quarters are busy on about half the blocks each, at random, and three S
// buffers let them drift at most two blocks apart, so the slowest quarter
// sets the pace when it is slower than the tensor pipe.
#pragma once

#include "msa_common.cuh"

namespace msa {
namespace uattn {

constexpr int kD = 128;
constexpr int kBlock = 128;
constexpr int kHpg = 16;
constexpr int kTopK = 16;
constexpr int kTileQ = 8;                           // queries per tile
constexpr int kMaxUnion = kTileQ * kTopK;           // 128 blocks at most
constexpr uint32_t kHalf = 128 * 128;               // [128 rows][64 bf16] = 16 KB
constexpr uint32_t kTile = 2 * kHalf;               // 32 KB
constexpr int kKRing = 3;
constexpr int kVRing = 2;
constexpr int kSBufs = 3;                           // S/P buffers in tensor memory
constexpr int kThreads = 8 * 32;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSCol = 0;                       // S/P buffer i: columns 128 i .. 128 i + 127
constexpr uint32_t kOCol = 128 * kSBufs;            // O: 128 columns after the S buffers
constexpr uint32_t kIdescS = umma_idesc_bf16_f32(128, 128, false, false);
constexpr uint32_t kIdescPV = umma_idesc_bf16_f32(128, 128, false, true);
constexpr float kRescale = 8.f;                     // raise the reference max past this (log2 units)
static_assert(kOCol + 128 <= kTmemCols, "tensor memory budget");

struct Plan {
  int n;                          // blocks in the union
  int pos[kTileQ];                // query positions (-1: no query / invalid)
  int seg_stream[kTileQ];         // stream of the segment whose id is this query index
  uint8_t seg_rows[kTileQ];       // queries of that segment
  int blocks[kMaxUnion];          // segments in order; within one, the order order_plan picks
  uint8_t masks[kMaxUnion];       // queries that selected the block
  uint8_t segs[kMaxUnion];        // segment id (index of its first query)
};

struct Layout {
  static constexpr uint32_t kQOff = 0;
  static constexpr uint32_t kKOff = kQOff + kTile;
  static constexpr uint32_t kVOff = kKOff + kKRing * kTile;
  static constexpr uint32_t kBarOff = kVOff + kVRing * kTile;
  static constexpr uint32_t kEnd = kBarOff + 40 * 8;
  static constexpr size_t kBytes = kEnd + 1024;
};
static_assert(Layout::kBytes <= 232448, "shared memory budget");

struct Params {
  const int32_t* sel;        // [n_q][G][16]
  const int32_t* q_stream;
  const int32_t* q_pos;
  __nv_bfloat16* out;        // [n_q][Hq][D]
  int n_q, G, n_streams, capacity, n_tiles;
  float scale_log2;
  KvPages pages;             // kPaged: K/V are page pools addressed through the block table
  Plan* plans;               // [G * n_tiles]: written by plan_tiles_kernel, read by the attention kernel
};

// Barrier slots (uint64 each, from Layout::kBarOff).
struct Bars {
  uint64_t *q_full, *q_empty, *kfull, *kempty, *vfull, *vempty;
  uint64_t *s_full, *p_full, *pv_done, *o_empty, *mma_done;
  uint32_t* tmem_slot;
  __device__ explicit Bars(uint8_t* smem) {
    uint64_t* b = reinterpret_cast<uint64_t*>(smem + Layout::kBarOff);
    q_full = b;
    q_empty = q_full + 1;
    kfull = q_empty + 1;           // [kKRing]
    kempty = kfull + kKRing;
    vfull = kempty + kKRing;       // [kVRing]
    vempty = vfull + kVRing;
    s_full = vempty + kVRing;      // [kSBufs]: S of the buffer's block is in tensor memory
    p_full = s_full + kSBufs;      // [kSBufs]: its P is written (4 softmax warps)
    pv_done = p_full + kSBufs;     // [kSBufs]: its P . V finished (buffer free, O updated)
    o_empty = pv_done + kSBufs;
    mma_done = o_empty + 1;        // [2]: the S issuer's and the P . V issuer's last MMAs
    tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 2);
  }
};
static_assert(2 + 2 * kKRing + 2 * kVRing + 3 * kSBufs + 3 + 1 <= 40, "barrier slots");

// exp2 on the special-function unit (ex2.approx.ftz: ~2 ulp; 2^-inf = 0).
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Two floats rounded to bf16 (nearest even) and packed: `lo` into the low
// half (the lower K index of a P pair), `hi` into the high half.
__device__ __forceinline__ uint32_t cvt_bf16x2(float lo, float hi) {
  uint32_t d;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
  return d;
}

// acc + both bf16 halves of `p`, in float32.
__device__ __forceinline__ float add_bf16x2_f32(uint32_t p, float acc) {
  float d;
  asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %1;\n\tadd.rn.f32.bf16 %0, lo, %2;\n\t"
      "add.rn.f32.bf16 %0, hi, %0;\n}"
      : "=f"(d)
      : "r"(p), "f"(acc));
  return d;
}

// Packed f32x2 arithmetic (sm_100 and later): two lanes per instruction.
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "mov.b64 rc, {%6, %7};\n\tfma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}
// max(a, b, c) in one instruction (three-input max.f32, sm_100 and later).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Tile t -> (group, first query).  Group-major, so the CTAs running at the
// same time work on nearby queries of one group and share its blocks in L2.
__device__ __forceinline__ void tile_coords(const Params& P, int t, int& g, int& q0) {
  g = t / P.n_tiles;
  q0 = (t - g * P.n_tiles) * kTileQ;
}

// Order of the union within each segment.  The softmax warp of TMEM lane
// quarter k serves queries 2k and 2k+1: on a block neither selected it only
// writes zeros (~400 cycles), otherwise it computes a row of exponentials
// (~1900), and with three S buffers the four quarters can drift only two
// blocks apart, so runs of blocks busy on one quarter stall the others.
// Greedily, the next block is one whose busy quarters overlap least with the
// previous block's (ties: the lower block).  Any order gives the same
// attention up to rounding (the online softmax does not depend on it).
__device__ __forceinline__ void order_plan(Plan& pl, int n, int lane) {
  constexpr uint32_t kFull = 0xffffffffu;
  auto quarters = [](uint32_t m) { return (m | (m >> 1)) & 0x55u; };   // quarter k busy: bit 2k
  uint32_t cm[4];
  int cb[4], cs[4];
  bool live[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int e = lane + 32 * k;
    live[k] = e < n;
    cb[k] = live[k] ? pl.blocks[e] : 0;
    cm[k] = live[k] ? pl.masks[e] : 0u;
    cs[k] = live[k] ? pl.segs[e] : -1;
  }
  __syncwarp();
  uint32_t prev = 0u;
  for (int pos = 0; pos < n; ++pos) {
    const int sg = pl.segs[pos];                   // segment ranges do not move
    uint32_t best = 0xffffffffu;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      if (live[k] && cs[k] == sg) {
        const uint32_t key = (static_cast<uint32_t>(__popc(quarters(cm[k]) & prev)) << 8) | static_cast<uint32_t>(lane + 32 * k);
        best = min(best, key);
      }
    }
    best = __reduce_min_sync(kFull, best);
    const int c = static_cast<int>(best & 0xffu);
    uint32_t wq = 0u;
    if ((c & 31) == lane) {
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        if (k == (c >> 5)) {
          live[k] = false;
          pl.blocks[pos] = cb[k];
          pl.masks[pos] = static_cast<uint8_t>(cm[k]);
          wq = quarters(cm[k]);
        }
      }
    }
    prev = __shfl_sync(kFull, wq, c & 31);
  }
  __syncwarp();
}

// One warp of plan_tiles_kernel: union of the tile's selections, by segment, into `pl`.
// The 128 (query, slot) entries become sortable keys (segment << 24 |
// block; ~0 for an empty or invalid entry), each carrying its query's bit;
// lane l holds entries 4l .. 4l+3.  A bitonic sort of the 128 keys (28
// compare-exchange steps, shuffles across lanes) puts equal keys side by
// side, a segmented OR over each run of equal keys gives the run's query
// mask, and a prefix count of run heads gives each distinct key its place
// in the union.  So the union comes out ascending within each segment
// whatever the order of a query's list, and a -1 or out-of-range entry
// anywhere in it is simply left out.  With paged caches a selected block
// whose page is missing is left out too (and MSA_DEVERR_PAGE_RANGE set), as
// if the query had not selected it.  order_plan then reorders each segment.
template <bool kPaged>
__device__ __forceinline__ void build_plan(const Params& P, int t, Plan& pl, int lane) {
  constexpr uint32_t kFull = 0xffffffffu;
  constexpr uint32_t kNone = 0xffffffffu;
  int g, q0;
  tile_coords(P, t, g, q0);
  // per query: position (or -1) and stream
  int pos = -1, stream = -1;
  if (lane < kTileQ) {
    const int qi = q0 + lane;
    if (qi < P.n_q) {
      const int s = P.q_stream[qi];
      const int p = P.q_pos[qi];
      if (s >= 0 && s < P.n_streams && p >= 0 && p < P.capacity) {
        pos = p;
        stream = s;
      } else if (g == 0) {
        raise_error(MSA_DEVERR_QUERY_RANGE);
      }
    }
  }
  // segment id: the first query of the tile with the same stream
  int seg = -1;
#pragma unroll
  for (int q = 0; q < kTileQ; ++q) {
    const int sq = __shfl_sync(kFull, stream, q);
    if (seg < 0 && stream >= 0 && sq == stream) seg = q;
  }
  if (lane < kTileQ) {
    pl.pos[lane] = pos;
    pl.seg_stream[lane] = stream;
  }
  uint32_t rows = 0;
#pragma unroll
  for (int q = 0; q < kTileQ; ++q) {
    const int sq = __shfl_sync(kFull, seg, q);
    if (sq == lane) rows |= 1u << q;
  }
  if (lane < kTileQ) pl.seg_rows[lane] = static_cast<uint8_t>(rows);
  // entries 4 lane + i: query lane / 4, slots 4 (lane % 4) + i
  const int q = lane >> 2;
  const int qpos = __shfl_sync(kFull, pos, q);
  const int qseg = __shfl_sync(kFull, seg, q);
  const int qstream = __shfl_sync(kFull, stream, q);
  uint32_t key[4], val[4];
  {
    int4 sel4 = make_int4(-1, -1, -1, -1);
    if (qpos >= 0)
      sel4 = __ldg(reinterpret_cast<const int4*>(P.sel + (static_cast<size_t>(q0 + q) * P.G + g) * kTopK) + (lane & 3));
    const int b4[4] = {sel4.x, sel4.y, sel4.z, sel4.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int b = b4[i];
      key[i] = kNone;
      val[i] = 1u << q;
      if (qpos >= 0) {
        if (b >= 0 && b <= qpos / kBlock) {
          if (kPaged && kv_block_row(P.pages, qstream, g, b, P.G, P.capacity) < 0)
            raise_error(MSA_DEVERR_PAGE_RANGE);
          else
            key[i] = (static_cast<uint32_t>(qseg) << 24) | static_cast<uint32_t>(b);
        } else if (b > qpos / kBlock) {
          raise_error(MSA_DEVERR_SEL_RANGE);
        }
      }
    }
  }
  // bitonic sort, ascending by key (element e = 4 lane + i)
#pragma unroll
  for (int k = 2; k <= 128; k <<= 1) {
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1) {
      if (j >= 4) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int e = 4 * lane + i;
          const uint32_t ok2 = __shfl_xor_sync(kFull, key[i], j >> 2);
          const uint32_t ov2 = __shfl_xor_sync(kFull, val[i], j >> 2);
          const bool up = (e & k) == 0;
          const bool lower = (e & j) == 0;
          if (lower == up ? ok2 < key[i] : ok2 > key[i]) {
            key[i] = ok2;
            val[i] = ov2;
          }
        }
      } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          if ((i & j) != 0) continue;
          const int i2 = i | j;
          const bool up = ((4 * lane + i) & k) == 0;
          if ((key[i] > key[i2]) == up && key[i] != key[i2]) {
            const uint32_t tk = key[i], tv = val[i];
            key[i] = key[i2];
            val[i] = val[i2];
            key[i2] = tk;
            val[i2] = tv;
          }
        }
      }
    }
  }
  // run heads, and each run's OR of query bits (a segmented scan towards the
  // run's end; bit 31 of acc marks "a run end lies in the scanned range")
  const uint32_t next0 = __shfl_down_sync(kFull, key[0], 1);
  const uint32_t prev3 = __shfl_up_sync(kFull, key[3], 1);
  uint32_t acc[4];
  bool head[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t nxt = i < 3 ? key[i + 1] : (lane < 31 ? next0 : kNone - 1);
    const uint32_t prv = i > 0 ? key[i - 1] : (lane > 0 ? prev3 : kNone - 1);
    const bool end = (i == 3 && lane == 31) || nxt != key[i];
    head[i] = (i == 0 && lane == 0) || prv != key[i];
    acc[i] = val[i] | (end ? 0x80000000u : 0u);
  }
#pragma unroll
  for (int d = 1; d < 128; d <<= 1) {
    uint32_t far[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int tt = i + d;                          // element e + d, in lane + tt / 4
      if (tt < 4) {
        far[i] = acc[tt];
      } else {
        const uint32_t x = __shfl_down_sync(kFull, acc[tt & 3], tt >> 2);
        far[i] = lane + (tt >> 2) < 32 ? x : 0x80000000u;
      }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
      if ((acc[i] & 0x80000000u) == 0u) acc[i] |= far[i];
  }
  // places of the distinct valid keys
  int mine = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) mine += (head[i] && key[i] != kNone) ? 1 : 0;
  int before = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int x = __shfl_up_sync(kFull, before, o);
    if (lane >= o) before += x;
  }
  const int n = __shfl_sync(kFull, before, 31);
  before -= mine;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    if (head[i] && key[i] != kNone) {
      pl.blocks[before] = static_cast<int>(key[i] & 0xffffffu);
      pl.segs[before] = static_cast<uint8_t>(key[i] >> 24);
      pl.masks[before] = static_cast<uint8_t>(acc[i] & 0xffu);
      ++before;
    }
  }
  if (lane == 0) pl.n = n;
  __syncwarp();
  order_plan(pl, n, lane);
}

// The plan of every tile, one warp per tile, ahead of the attention kernel
// (which reads them after its programmatic-dependent-launch wait): planning
// inside the attention kernel starved for issue slots next to the softmax
// warps (~50K cycles per tile).
template <bool kPaged>
__global__ void __launch_bounds__(256) plan_tiles_kernel(const Params P) {
  pdl_trigger();
  pdl_wait();                                          // the selections come from the kernel before
  const int t = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (t < P.G * P.n_tiles) build_plan<kPaged>(P, t, P.plans[t], threadIdx.x & 31);
}

template <bool kPaged>
__global__ void __launch_bounds__(kThreads, 1)
    sparse_attn_prefill_union_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                                     const __grid_constant__ CUtensorMap tm_v, const Params P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const Bars B(smem);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_tasks = P.G * P.n_tiles;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kSBufs; ++i) {
      mbar_init(&B.s_full[i], 1);
      mbar_init(&B.p_full[i], 4);
      mbar_init(&B.pv_done[i], 1);
    }
    mbar_init(B.q_full, 1);
    mbar_init(B.q_empty, 1);
    for (int i = 0; i < kKRing; ++i) {
      mbar_init(&B.kfull[i], 1);
      mbar_init(&B.kempty[i], 1);
    }
    for (int i = 0; i < kVRing; ++i) {
      mbar_init(&B.vfull[i], 1);
      mbar_init(&B.vempty[i], 1);
    }
    mbar_init(B.o_empty, 4);
    mbar_init(&B.mma_done[0], 1);
    mbar_init(&B.mma_done[1], 1);
    mbar_fence_init();
  }
  if (warp == 1) tmem_alloc(B.tmem_slot, kTmemCols);
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *B.tmem_slot;
  pdl_trigger();
  pdl_wait();

  if (warp == 0) {
    // ------------------------ the Q tile and the K blocks (lane 0) ---------------------
    if (lane == 0) {
      int ring = 0, q_use = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < n_tasks && ok; t += gridDim.x) {
        const Plan& pl = P.plans[t];
        int g, q0;
        tile_coords(P, t, g, q0);
        if (pl.n > 0) {
          // the previous tile's S MMAs have finished with the Q tile
          if (q_use > 0) ok = mbar_wait(B.q_empty, (q_use - 1) & 1);
          if (!ok) break;
          int nq = 0;
          for (int q = 0; q < kTileQ; ++q) nq += q0 + q < P.n_q ? 1 : 0;
          mbar_arrive_expect_tx(B.q_full, static_cast<uint32_t>(nq) * 2 * (kHpg * 128));
          for (int q = 0; q < nq; ++q) {
            const int row = (q0 + q) * (P.G * kHpg) + g * kHpg;      // q viewed as [n_q * Hq][128]
            uint8_t* dst = smem + Layout::kQOff + q * (kHpg * 128);
            tma_load_2d(dst, &tm_q, 0, row, B.q_full);
            tma_load_2d(dst + kHalf, &tm_q, 64, row, B.q_full);
          }
          ++q_use;
        }
        for (int j = 0; j < pl.n && ok; ++j, ++ring) {
          const int st = ring % kKRing;
          const int use = ring / kKRing;
          if (use > 0) ok = mbar_wait(&B.kempty[st], (use - 1) & 1);
          if (!ok) break;
          const int s = pl.seg_stream[pl.segs[j]];
          const int row = kPaged ? static_cast<int>(kv_block_row(P.pages, s, g, pl.blocks[j], P.G, P.capacity))
                                 : (s * P.G + g) * P.capacity + pl.blocks[j] * kBlock;
          uint8_t* dst = smem + Layout::kKOff + st * kTile;
          mbar_arrive_expect_tx(&B.kfull[st], kTile);
          tma_load_2d(dst, &tm_k, 0, row, &B.kfull[st]);
          tma_load_2d(dst + kHalf, &tm_k, 64, row, &B.kfull[st]);
        }
      }
      // no copy may still be landing when the CTA exits
      for (int j = max(0, ring - kKRing); j < ring; ++j) mbar_wait(&B.kfull[j % kKRing], (j / kKRing) & 1);
      if (q_use > 0) mbar_wait(B.q_full, (q_use - 1) & 1);
    }
  } else if (warp == 2) {
    // ------------------------------ V loader (lane 0) ------------------------------
    if (lane == 0) {
      int ring = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < n_tasks && ok; t += gridDim.x) {
        const Plan& pl = P.plans[t];
        int g, q0;
        tile_coords(P, t, g, q0);
        for (int j = 0; j < pl.n && ok; ++j, ++ring) {
          const int st = ring % kVRing;
          const int use = ring / kVRing;
          if (use > 0) ok = mbar_wait(&B.vempty[st], (use - 1) & 1);
          if (!ok) break;
          const int s = pl.seg_stream[pl.segs[j]];
          const int row = kPaged ? static_cast<int>(kv_block_row(P.pages, s, g, pl.blocks[j], P.G, P.capacity))
                                 : (s * P.G + g) * P.capacity + pl.blocks[j] * kBlock;
          uint8_t* dst = smem + Layout::kVOff + st * kTile;
          mbar_arrive_expect_tx(&B.vfull[st], kTile);
          tma_load_2d(dst, &tm_v, 0, row, &B.vfull[st]);
          tma_load_2d(dst + kHalf, &tm_v, 64, row, &B.vfull[st]);
        }
      }
      for (int j = max(0, ring - kVRing); j < ring; ++j) mbar_wait(&B.vfull[j % kVRing], (j / kVRing) & 1);
    }
  } else if (warp == 1) {
    // ------------------------- S issuer: S = Q . K_b^T (lane 0) -------------------
    // S and P . V come from two issuing threads: the tensor pipe drains when
    // one thread switches operand configuration (shared-memory / tensor-memory
    // A, K- / MN-major B), not when two threads' streams interleave.
    if (lane == 0) {
      const uint32_t q_base = smem_addr(smem + Layout::kQOff);
      const uint32_t k_base = smem_addr(smem + Layout::kKOff);
      int kr = 0, blk = 0, q_use = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < n_tasks && ok; t += gridDim.x) {
        const Plan& pl = P.plans[t];
        if (pl.n > 0) {
          ok = mbar_wait(B.q_full, q_use & 1);
          ++q_use;
          tc_fence_after();
          for (int j = 0; j < pl.n && ok; ++j) {
            const int b = blk + j;
            const int kst = kr % kKRing;
            const int sb = b % kSBufs;
            ok = mbar_wait(&B.kfull[kst], (kr / kKRing) & 1);
            // the buffer's previous block has finished its P . V
            if (ok && b >= kSBufs) ok = mbar_wait(&B.pv_done[sb], ((b / kSBufs) - 1) & 1);
            if (!ok) break;
            tc_fence_after();
            const uint32_t kb = k_base + kst * kTile;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint32_t off = (kk >> 2) * kHalf + (kk & 3) * 32;
              umma_f16_ss(tmem_base + kSCol + sb * 128, umma_desc_sw128(q_base + off), umma_desc_sw128(kb + off),
                          kIdescS, kk != 0);
            }
            umma_commit(&B.kempty[kst]);
            umma_commit(&B.s_full[sb]);
            if (j == pl.n - 1) umma_commit(B.q_empty);         // the tile's last use of Q
            ++kr;
          }
          blk += pl.n;
        }
      }
      umma_commit(&B.mma_done[0]);
      mbar_wait(&B.mma_done[0], 0);
    }
  } else if (warp == 3) {
    // ---------------------- P . V issuer: O (+)= P . V_b (lane 0) -----------------
    if (lane == 0) {
      const uint32_t v_base = smem_addr(smem + Layout::kVOff);
      int vr = 0, blk = 0, segs_done = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < n_tasks && ok; t += gridDim.x) {
        const Plan& pl = P.plans[t];
        for (int j = 0; j < pl.n && ok; ++j) {
          const int b = blk + j;
          const bool seg_first = j == 0 || pl.segs[j] != pl.segs[j - 1];
          const int sb = b % kSBufs;
          ok = mbar_wait(&B.p_full[sb], (b / kSBufs) & 1);
          if (ok && seg_first && segs_done > 0) ok = mbar_wait(B.o_empty, (segs_done - 1) & 1);
          const int st = vr % kVRing;
          if (ok) ok = mbar_wait(&B.vfull[st], (vr / kVRing) & 1);
          if (!ok) break;
          tc_fence_after();
          const uint32_t vb = v_base + st * kTile;
          const uint32_t pa = tmem_base + kSCol + sb * 128;      // P: 64 columns of bf16 pairs
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            umma_f16_ts(tmem_base + kOCol, pa + kk * 8, umma_desc_sw128_mn(vb + kk * 2048, kHalf), kIdescPV,
                        (seg_first && kk == 0) ? 0u : 1u);
          umma_commit(&B.vempty[st]);
          umma_commit(&B.pv_done[sb]);
          ++vr;
          if (seg_first) ++segs_done;
        }
        blk += pl.n;
      }
      umma_commit(&B.mma_done[1]);
      mbar_wait(&B.mma_done[1], 0);
    }
  } else if (warp >= 4) {
    // ---------------- softmax and output: one thread per (query, head) row --------
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;             // TMEM lane = MMA row
    const int q = r / kHpg;
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    int blk = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < n_tasks; t += gridDim.x) {
      const Plan& pl = P.plans[t];
      int g, q0;
      tile_coords(P, t, g, q0);
      const int qi = q0 + q;
      const int pq = pl.pos[q];
      bool wrote = false;
      float m_ref = -INFINITY, l = 0.f;
      for (int j = 0; j < pl.n && ok; ++j) {
        const int b = blk + j;
        const int seg = pl.segs[j];
        const bool seg_first = j == 0 || pl.segs[j - 1] != seg;
        const bool seg_last = j == pl.n - 1 || pl.segs[j + 1] != seg;
        if (seg_first) {
          m_ref = -INFINITY;
          l = 0.f;
        }
        const int sb = b % kSBufs;
        const uint32_t sbuf = tmem_base + lane_addr + kSCol + sb * 128;
        // mask: the row's query selected this block (else its P row is
        // exp2(-inf) = 0), and keys j <= its position (only its local block
        // is cut).  Read before the wait, so that the plan's latency hides
        // behind it.
        const bool mine = ((pl.masks[j] >> q) & 1) != 0 && pq >= 0;
        const int jmax = mine ? pq - pl.blocks[j] * kBlock : -1;       // last visible key in the block
        const bool active = __any_sync(0xffffffffu, mine);
        ok = mbar_wait(&B.s_full[sb], (b / kSBufs) & 1);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        float s[kBlock];
        if (active) {
          float v0[32], v1[32], v2[32], v3[32];
          tmem_ld32(sbuf, v0);
          tmem_ld32(sbuf + 32, v1);
          tmem_ld32(sbuf + 64, v2);
          tmem_ld32(sbuf + 96, v3);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            s[i] = v0[i];
            s[32 + i] = v1[i];
            s[64 + i] = v2[i];
            s[96 + i] = v3[i];
          }
        }
        float mb = -INFINITY;
        if (active && __any_sync(0xffffffffu, mine && jmax < kBlock - 1)) {
#pragma unroll
          for (int c = 0; c < kBlock; ++c) s[c] = c <= jmax ? s[c] : -INFINITY;
        }
        if (active) {
          // four independent chains of three-input maxima: 18 dependent steps
          // instead of 128
          float m4[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) m4[i] = fmax3(s[i], s[4 + i], s[8 + i]);
#pragma unroll
          for (int c = 12; c < kBlock - 4; c += 8)
#pragma unroll
            for (int i = 0; i < 4; ++i) m4[i] = fmax3(m4[i], s[c + i], s[c + 4 + i]);
#pragma unroll
          for (int i = 0; i < 4; ++i) m4[i] = fmaxf(m4[i], s[kBlock - 4 + i]);
          mb = fmaxf(fmax3(m4[0], m4[1], m4[2]), m4[3]);
          mb = mine ? mb * P.scale_log2 : -INFINITY;                     // max of the scaled scores
        }
        const bool raise = mb > m_ref + kRescale;
        const bool rescale = raise && !seg_first && m_ref != -INFINITY;
        if (__any_sync(0xffffffffu, rescale)) {
          // O of the rows that raise their max is rescaled once the previous
          // block's P . V (in the other buffer) has finished
          const int pb = b - 1;
          ok = mbar_wait(&B.pv_done[pb % kSBufs], (pb / kSBufs) & 1);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          tc_fence_after();
          const float f = rescale ? ex2_approx(m_ref - mb) : 1.f;
          l *= f;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            float v[32];
            tmem_ld32(tmem_base + lane_addr + kOCol + c * 32, v);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] *= f;
            tmem_st32(tmem_base + lane_addr + kOCol + c * 32, v);
          }
        }
        if (raise) m_ref = mb;
        const float neg_m = mine ? -m_ref : -INFINITY;
        // P = exp2(s - m_ref) as bf16 pairs over the first 64 columns of the
        // buffer; the row sum adds the rounded P values the P . V product
        // uses, so the normalisation matches the weights applied
        if (active) {
          const float2 sc2 = make_float2(P.scale_log2, P.scale_log2);
          const float2 nm2 = make_float2(neg_m, neg_m);
          float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            float pk[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const float2 x = ffma2(make_float2(s[h * 64 + 2 * i], s[h * 64 + 2 * i + 1]), sc2, nm2);
              const uint32_t pp = cvt_bf16x2(ex2_approx(x.x), ex2_approx(x.y));
              acc[i & 3] = add_bf16x2_f32(pp, acc[i & 3]);
              pk[i] = __uint_as_float(pp);
            }
            tmem_st32(sbuf + h * 32, pk);
          }
          l += (acc[0] + acc[1]) + (acc[2] + acc[3]);
        } else {
          float z[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) z[i] = 0.f;
          tmem_st32(sbuf, z);
          tmem_st32(sbuf + 32, z);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&B.p_full[sb]);
        if (seg_last) {
          // O of the segment is complete once this block's P . V has finished
          ok = mbar_wait(&B.pv_done[sb], (b / kSBufs) & 1);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          tc_fence_after();
          const bool row_here = ((pl.seg_rows[seg] >> q) & 1) != 0 && pq >= 0;
          const float inv = l > 0.f ? 1.f / l : 0.f;
          __nv_bfloat16* dst = P.out + (static_cast<size_t>(qi) * (P.G * kHpg) + g * kHpg + (r % kHpg)) * kD;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            float v[32];
            tmem_ld32(tmem_base + lane_addr + kOCol + c * 32, v);
            tmem_ld_wait();
            if (row_here) {
#pragma unroll
              for (int i = 0; i < 32; i += 8) {
                *reinterpret_cast<uint4*>(dst + c * 32 + i) =
                    make_uint4(pack_bf16(v[i] * inv, v[i + 1] * inv), pack_bf16(v[i + 2] * inv, v[i + 3] * inv),
                               pack_bf16(v[i + 4] * inv, v[i + 5] * inv), pack_bf16(v[i + 6] * inv, v[i + 7] * inv));
              }
            }
          }
          if (row_here) wrote = true;
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(B.o_empty);
        }
      }
      if (!ok) break;
      blk += pl.n;
      // queries with nothing to attend (invalid, or no visible selected block): zeros
      if (!wrote && qi < P.n_q) {
        __nv_bfloat16* dst = P.out + (static_cast<size_t>(qi) * (P.G * kHpg) + g * kHpg + (r % kHpg)) * kD;
#pragma unroll
        for (int i = 0; i < kD; i += 8) *reinterpret_cast<uint4*>(dst + i) = make_uint4(0u, 0u, 0u, 0u);
      }
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace uattn
}  // namespace msa
