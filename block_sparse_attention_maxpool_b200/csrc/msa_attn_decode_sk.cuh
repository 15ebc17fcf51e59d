// Block-sparse GQA attention for decode batches: persistent, stream-K style.
//
// MSA pull request "Add MiniMax-M3 (MSA) support", section "Overview": each
// query attends to the rows of its selected blocks only (16 x 128 = 2048
// keys), shared by the 16 heads of its GQA group; the token-level causal mask
// applies inside the local block.
//
// A decode step has few (query, group) pairs, each reading 16 blocks of K and
// V (1 MB).  The work units are (pair, selected block); every CTA of a
// persistent grid (at most one per SM) takes one contiguous, equal share of
// the units, so all SMs stream K/V for the whole kernel with no wave tail.
// One producer thread resolves each unit (query position, selected block,
// cache row), writes what the consumers need into a small per-stage record
// and TMA-loads the unit's K and V tiles (four 16 KB boxes, 128-byte
// swizzle) into a three-stage ring, plus the pair's Q (16 heads x 128 dims)
// when the unit is the first of its pair in this CTA; the consumers so make
// no global-memory round trip between units.  Eight consumer warps each own
// 16 key rows of the block and compute S = Q K^T (16 heads x 16 rows) and
// O += P V with bf16 m16n8k16 MMAs, fp32 accumulation and a streaming base-2
// softmax.  Consecutive units of one pair accumulate in registers; when the
// pair changes the eight warps merge through shared memory.  A pair whose
// units all lie in one CTA's share is written out directly; a pair cut by a
// share boundary is merged inside the kernel by the CTA holding its first
// unit, which reaches it last (at the end of its share), from the partials
// (max, sum, unnormalised O) the later CTAs published; no merge kernel
// follows.
//
// Fused selection (Params::bs set): before the ring starts, the CTA's
// consumer warps rank the block scores of the (at most kSelPairs) pairs its
// units touch, one warp per pair with the top-16 routine of the selection
// kernel, keys staged in the stage ring (idle until the first load); the
// producer then reads the selection from shared memory, and the CTA holding
// a pair's first unit writes that pair's selection and count for the caller.
// The result is the selection kernel's, bit for bit, without its launch.
//
// Token-level variant ("deepseek2 : GLM-DSA sparse attention (lightning
// indexer)": top-k tokens per query, the same set for every group): a unit
// is a chunk of 128 consecutive entries of the query's ascending token list
// (2048 entries, 16 chunks, -1 padded).  The rows are scattered, so two
// producer warps gather them (one row per lane) with 16-byte cp.async copies
// straight into the same 128-byte-swizzled tile layout the TMA path
// produces, each lane arriving on the stage's barrier when its copies land;
// rows of padding or of an unmapped page are copied from a zero row and
// masked through a 128-bit row mask in the stage record.  Random 256-byte
// rows bound this path near 2 TB/s on B200 (a TMA tile::gather4 form
// measured slower).
#pragma once

#include "msa_common.cuh"
#include "msa_select.cuh"

namespace msa {
namespace dattn {

constexpr int kD = 128;
constexpr int kBlock = 128;
constexpr int kHpg = 16;
constexpr int kTopK = 16;
constexpr int kWarps = 8;                           // consumer warps
constexpr int kGatherWarps = 2;                     // producer warps of the token-level variant
constexpr int kThreads = (kWarps + kGatherWarps) * 32;   // block path: one producer thread, one idle warp
constexpr int kRowsPerWarp = kBlock / kWarps;       // 16
constexpr uint32_t kTileBytes = kBlock * 64 * 2;    // [128 rows][64 dims] bf16 = 16 KB
constexpr uint32_t kStageBytes = 4 * kTileBytes;    // K lo, K hi, V lo, V hi
constexpr uint32_t kQBytes = kHpg * kD * 2;         // Q of one pair: two [16 heads][64 dims] boxes, 4 KB
constexpr int kStages = 3;
constexpr int kMergeCols = 32;                      // dims of O merged per round (four rounds)
constexpr int kMStride = kMergeCols + 4;            // padded fp32 row of the merge buffer
constexpr int kMaxCtas = 256;                       // grid cap (bounds the workspace)
constexpr int kPartial = kHpg * (kD + 2);           // floats of one partial: O[16][128], m[16], l[16]
constexpr int kSelPairs = 8;                        // fused selection: pairs one CTA may touch

// One CTA slot of the workspace's merge bookkeeping (kMaxCtas slots at the
// start of the workspace, kept from call to call).  A pair cut by share
// boundaries is merged by the CTA holding its first unit (its "merger"),
// which reaches that pair last, at the end of its share; every later CTA
// holding some of its units publishes a partial and sets `flag` to
// kFlagTag | merger << 32 | (merger's epoch + 1).  The merger waits for
// exactly that value, merges, and then raises its own epoch, so a flag left
// from an earlier call (or any other contents of a reused buffer) never
// matches, and the slots need no zeroing.
struct SyncSlot {
  unsigned long long flag;
  unsigned int epoch;
  unsigned int pad;
};
constexpr unsigned long long kFlagTag = 0x4d53ull << 48;
constexpr size_t kSyncBytes = kMaxCtas * sizeof(SyncSlot);

// What the producer tells the consumers about the unit in a stage.
struct UnitInfo {
  int32_t flags;      // kUnitData: K/V rows landed; kUnitQ: the pair's Q landed
  int32_t p;          // query position
  int32_t slot0;      // first slot of the block in its stream (block path)
  int32_t pad;
  uint32_t mask[4];   // token path: bit r set = row r of the unit is attended
};
constexpr int32_t kUnitData = 1;
constexpr int32_t kUnitQ = 2;

struct Layout {
  static constexpr uint32_t kStageOff = 0;
  static constexpr uint32_t kQOff = kStages * kStageBytes;
  static constexpr uint32_t kMergeOff = kQOff + kStages * kQBytes;
  static constexpr uint32_t kMlOff = kMergeOff + kWarps * kHpg * kMStride * 4;
  static constexpr uint32_t kInfoOff = kMlOff + kWarps * kHpg * 2 * 4;
  static constexpr uint32_t kSelOff = kInfoOff + kStages * sizeof(UnitInfo);
  static constexpr uint32_t kMiscOff = kSelOff + kSelPairs * (kTopK + 1) * 4 + 16;   // the CTA's epoch
  static constexpr uint32_t kBarOff = kMiscOff + 16;
  static constexpr uint32_t kEnd = kBarOff + 64;
  static constexpr size_t kBytes = kEnd + 1024;
};
static_assert(Layout::kQOff % 1024 == 0 && kQBytes % 1024 == 0, "128-byte-swizzled TMA boxes start on 1 KB");
static_assert(Layout::kBarOff % 8 == 0 && Layout::kInfoOff % 16 == 0, "barrier and record alignment");
static_assert(kWarps * sel::KeySmem<32>::kBytesPerWarp <= Layout::kQOff - Layout::kStageOff,
              "fused selection: every consumer warp's keys fit the stage ring");
static_assert(Layout::kBytes + 256 <= 227 * 1024, "shared memory of one CTA (and of the one-kernel step)");

struct Params {
  const __nv_bfloat16* q;     // [n_q][Hq][D]
  const int32_t* sel;         // [n_q][G][16]
  const int32_t* q_stream;
  const int32_t* q_pos;
  __nv_bfloat16* out;         // [n_q][Hq][D]
  float* ws;                  // [n_cta][kPartial]: the partial of each CTA's first pair when it began earlier
  SyncSlot* sync;             // [kMaxCtas], kept between calls
  int n_q, G, n_streams, capacity, n_cta;
  long long n_units;          // n_q * G * 16
  float scale_log2;
  KvPages pages;              // block table of paged K/V caches (table null: contiguous)
  const int32_t* tok_sel;     // token-level variant: [n_q][16 * 128] ascending token ids (else null)
  const __nv_bfloat16* k_cache;   // token-level variant: the K and V caches (or pools) the gathers read
  const __nv_bfloat16* v_cache;
  const float* bs;            // fused selection: block scores [n_q][G][nblk] (else null)
  int nblk;
  int32_t* sel_out;           // fused selection: the selection and its counts, written for the caller
  int32_t* n_sel_out;         // (nullable)
};

// 256 zero bytes: the source of the K and V rows of masked token slots.
__device__ __align__(16) uint8_t g_zero_row[256];

// Token-level unit u: query position, stream, group and the unit's 128 token
// slots; false when the unit has nothing to attend.
__device__ __forceinline__ bool tok_unit(const Params& P, long long u, int& s, int& g, int& p,
                                         const int32_t*& toks, bool report) {
  const long long pair = u / kTopK;
  const int j = static_cast<int>(u - pair * kTopK);
  const int qi = static_cast<int>(pair / P.G);
  g = static_cast<int>(pair - static_cast<long long>(qi) * P.G);
  s = P.q_stream[qi];
  p = P.q_pos[qi];
  if (s < 0 || s >= P.n_streams || p < 0 || p >= P.capacity) {
    if (report && j == 0 && g == 0) raise_error(MSA_DEVERR_QUERY_RANGE);
    return false;
  }
  toks = P.tok_sel + static_cast<size_t>(qi) * (kTopK * kBlock) + j * kBlock;
  return __ldg(toks) >= 0;
}

// Cache row of a selected token, or -1 when the slot is padding, names a
// token the query cannot see, or lies in an unmapped page.
__device__ __forceinline__ long long tok_row(const Params& P, int s, int g, int p, int tok) {
  if (tok < 0 || tok > p) return -1;
  const long long blk = kv_block_row(P.pages, s, g, tok >> 7, P.G, P.capacity);
  return blk < 0 ? -1 : blk + (tok & 127);
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}

// The mbarrier receives one arrival when all of this thread's earlier
// cp.async copies have landed (counted in the barrier's expected arrivals).
__device__ __forceinline__ void cp_async_arrive(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__host__ __device__ inline long long unit_begin(long long U, int C, int c) { return U * c / C; }

// The CTA whose share holds unit u.
__device__ inline int cta_of(long long U, int C, long long u) {
  int c = static_cast<int>(u * C / U);
  while (c + 1 < C && unit_begin(U, C, c + 1) <= u) ++c;
  while (c > 0 && unit_begin(U, C, c) > u) --c;
  return c;
}

// Cache row of unit u's block, or -1 when the unit has nothing to attend
// (padding, an invalid selection, an invalid query or a block with no valid
// page).  p: query position; slot0: first slot of the block in its stream.
// sel_s: the CTA's fused selection (rows of pairs pf, pf + 1, ...), else null
// and the selection is read from P.sel.
__device__ __forceinline__ int unit_row(const Params& P, long long u, int& p, int& slot0, bool report,
                                        const int32_t* sel_s, long long pf) {
  const long long pair = u / kTopK;
  const int j = static_cast<int>(u - pair * kTopK);
  const int qi = static_cast<int>(pair / P.G);
  const int g = static_cast<int>(pair - static_cast<long long>(qi) * P.G);
  const int s = P.q_stream[qi];
  p = P.q_pos[qi];
  if (s < 0 || s >= P.n_streams || p < 0 || p >= P.capacity) {
    if (report && j == 0 && g == 0) raise_error(MSA_DEVERR_QUERY_RANGE);
    return -1;
  }
  int b;
  if (sel_s != nullptr) {
    if (pair - pf >= kSelPairs) return -1;            // the host never launches such a share
    b = sel_s[(pair - pf) * kTopK + j];
  } else {
    b = __ldcg(P.sel + pair * kTopK + j);             // L2 only: the selection may come from the previous kernel
  }
  if (b < 0) return -1;
  if (b > p / kBlock) {
    if (report) raise_error(MSA_DEVERR_SEL_RANGE);
    return -1;
  }
  const long long row = kv_block_row(P.pages, s, g, b, P.G, P.capacity);
  if (row < 0) {
    if (report) raise_error(MSA_DEVERR_PAGE_RANGE);
    return -1;
  }
  slot0 = b * kBlock;
  return static_cast<int>(row);   // the host checks that every row fits 31 bits
}

__device__ __forceinline__ unsigned long long ld_acquire_u64(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_release_u64(unsigned long long* p, unsigned long long v) {
  asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

// Merge the eight warps' states of one pair and write the output rows.  O
// goes through shared memory in four rounds of 32 dims (a quarter-size
// buffer, which leaves room for a third stage of the ring); thread (head,
// 2 dims) sums the eight warps' slices, scaled to the common maximum.  A
// pair this CTA holds only the tail of (it began in an earlier CTA) is
// published as this CTA's partial instead (`pub`: the flag value, thread
// 0).  A pair that begins here and ends in later CTAs is the CTA's last, so
// the ring is idle: its merged state goes to the stage area, and once the
// later CTAs' flags read this CTA's next epoch, thread (head, 8 dims) folds
// their partials in, all loads in flight at once, and writes the rows.
__device__ __forceinline__ void flush_pair(const Params& P, uint8_t* smem, long long pair, long long u0,
                                           long long u1, int cta, float (&o)[16][4], float (&m_run)[2],
                                           float (&l_run)[2], int warp, int lane, unsigned long long pub) {
  const int gr = lane >> 2, tq = lane & 3;
  const int tid = warp * 32 + lane;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    l_run[h] += __shfl_xor_sync(0xffffffffu, l_run[h], 1);
    l_run[h] += __shfl_xor_sync(0xffffffffu, l_run[h], 2);
  }
  float* so = reinterpret_cast<float*>(smem + Layout::kMergeOff);   // [8][16][kMStride]
  float* sml = reinterpret_cast<float*>(smem + Layout::kMlOff);     // [8][16][2]
  float* mine = reinterpret_cast<float*>(smem + Layout::kStageOff); // merger: [16][128] own merged O
  const int head = tid >> 4;            // 16 heads x 16 threads
  const int dd = (tid & 15) * 2;        // 2 dims of the round's 32 per thread
  const bool tail = pair * kTopK < u0;                               // began in an earlier CTA
  const bool merger = !tail && pair * kTopK + kTopK > u1;            // begins here, ends later
  float* part = P.ws + static_cast<size_t>(cta) * kPartial;
  float sc[kWarps];
  float M = -INFINITY, L = 0.f, inv = 0.f;
#pragma unroll
  for (int r = 0; r < kD / kMergeCols; ++r) {
    named_barrier_sync(1, kWarps * 32);                               // the previous round fully read
    {
      float* ow = so + warp * kHpg * kMStride;
#pragma unroll
      for (int nn = 0; nn < kMergeCols / 8; ++nn) {
        const int n = r * (kMergeCols / 8) + nn;
        const int col = nn * 8 + tq * 2;
        *reinterpret_cast<float2*>(ow + gr * kMStride + col) = make_float2(o[n][0], o[n][1]);
        *reinterpret_cast<float2*>(ow + (gr + 8) * kMStride + col) = make_float2(o[n][2], o[n][3]);
      }
      if (r == 0 && tq == 0) {
        sml[(warp * kHpg + gr) * 2 + 0] = m_run[0];
        sml[(warp * kHpg + gr) * 2 + 1] = l_run[0];
        sml[(warp * kHpg + gr + 8) * 2 + 0] = m_run[1];
        sml[(warp * kHpg + gr + 8) * 2 + 1] = l_run[1];
      }
    }
    named_barrier_sync(1, kWarps * 32);
    if (r == 0) {
#pragma unroll
      for (int w = 0; w < kWarps; ++w) M = fmaxf(M, sml[(w * kHpg + head) * 2]);
      const float Mu = M == -INFINITY ? 0.f : M;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        sc[w] = exp2f(sml[(w * kHpg + head) * 2] - Mu);
        L += sml[(w * kHpg + head) * 2 + 1] * sc[w];
      }
      inv = L > 0.f ? 1.f / L : 0.f;
    }
    float a0 = 0.f, a1 = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const float2 v = *reinterpret_cast<const float2*>(so + (w * kHpg + head) * kMStride + dd);
      a0 += v.x * sc[w];
      a1 += v.y * sc[w];
    }
    const int d = r * kMergeCols + dd;
    if (tail) {
      *reinterpret_cast<float2*>(part + head * kD + d) = make_float2(a0, a1);
    } else if (merger) {
      *reinterpret_cast<float2*>(mine + head * kD + d) = make_float2(a0, a1);
    } else {
      __nv_bfloat16* dst = P.out + (static_cast<size_t>(pair) * kHpg + head) * kD + d;
      *reinterpret_cast<uint32_t*>(dst) = pack_bf16(a0 * inv, a1 * inv);
    }
  }
  if (tail) {
    if ((tid & 15) == 0) {
      part[kHpg * kD + head] = M;
      part[kHpg * kD + kHpg + head] = L;
    }
    __syncwarp();
    named_barrier_sync(1, kWarps * 32);    // every thread's share of the partial written
    if (tid == 0) st_release_u64(&P.sync[cta].flag, pub);   // releases what the barrier ordered before it
    return;
  }
  if (!merger) return;
  // the later CTAs holding some of this pair publish their partials early
  // in their shares; by now they are normally there
  const int n_later = cta_of(P.n_units, P.n_cta, pair * kTopK + kTopK - 1) - cta;
  const unsigned int epoch = *reinterpret_cast<const unsigned int*>(smem + Layout::kMiscOff);
  if (tid < n_later) {
    const unsigned long long want = kFlagTag | (static_cast<unsigned long long>(cta) << 32) | (epoch + 1u);
    const unsigned long long* f = &P.sync[cta + 1 + tid].flag;
    if (ld_acquire_u64(f) != want) {
      const long long t0 = clock64();
      while (ld_acquire_u64(f) != want) {
        if (clock64() - t0 > kWaitCycles) {
          raise_error(MSA_DEVERR_TIMEOUT);
          break;
        }
      }
    }
  }
  __syncwarp();
  named_barrier_sync(1, kWarps * 32);      // the flags seen, the own state in `mine`
  const int d8 = (tid & 15) * 8;           // thread (head, 8 dims)
  // fold the later partials in, eight at a time with all their loads in
  // flight, rescaling the running state to each batch's maximum
  float acc[8];
  {
    const float4 x = *reinterpret_cast<const float4*>(mine + head * kD + d8);
    const float4 y = *reinterpret_cast<const float4*>(mine + head * kD + d8 + 4);
    acc[0] = x.x; acc[1] = x.y; acc[2] = x.z; acc[3] = x.w;
    acc[4] = y.x; acc[5] = y.y; acc[6] = y.z; acc[7] = y.w;
  }
  float Mrun = M, Lrun = L;
  for (int base = 0; base < n_later; base += 8) {
    float mj[8], lj[8];
    float4 xj[8], yj[8];
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      mj[t] = -INFINITY;
      lj[t] = 0.f;
      xj[t] = yj[t] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (base + t < n_later) {
        const float* pj = P.ws + static_cast<size_t>(cta + 1 + base + t) * kPartial;
        mj[t] = __ldcg(pj + kHpg * kD + head);
        lj[t] = __ldcg(pj + kHpg * kD + kHpg + head);
        xj[t] = __ldcg(reinterpret_cast<const float4*>(pj + head * kD + d8));
        yj[t] = __ldcg(reinterpret_cast<const float4*>(pj + head * kD + d8 + 4));
      }
    }
    float Mnew = Mrun;
#pragma unroll
    for (int t = 0; t < 8; ++t) Mnew = fmaxf(Mnew, mj[t]);
    const float Mu = Mnew == -INFINITY ? 0.f : Mnew;
    const float sr = exp2f(Mrun - Mu);
    Lrun *= sr;
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] *= sr;
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      const float sj = exp2f(mj[t] - Mu);
      Lrun += lj[t] * sj;
      acc[0] += xj[t].x * sj; acc[1] += xj[t].y * sj; acc[2] += xj[t].z * sj; acc[3] += xj[t].w * sj;
      acc[4] += yj[t].x * sj; acc[5] += yj[t].y * sj; acc[6] += yj[t].z * sj; acc[7] += yj[t].w * sj;
    }
    Mrun = Mnew;
  }
  const float iall = Lrun > 0.f ? 1.f / Lrun : 0.f;
  uint32_t pk[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) pk[e] = pack_bf16(acc[2 * e] * iall, acc[2 * e + 1] * iall);
  *reinterpret_cast<uint4*>(P.out + (static_cast<size_t>(pair) * kHpg + head) * kD + d8) =
      make_uint4(pk[0], pk[1], pk[2], pk[3]);
  named_barrier_sync(1, kWarps * 32);      // every later partial read
  if (tid == 0) P.sync[cta].epoch = epoch + 1u;   // read by the next call's CTAs, after this kernel ends
}

// The top-16 of the pairs this CTA's units touch (fused selection), into
// sel_s: consumer warp w ranks pairs pf + w, pf + w + kWarps, ... with its
// keys in its slice of the stage ring; the CTA holding a pair's first unit
// writes the pair's selection and count to the caller's buffers.
__device__ __forceinline__ void select_share(const Params& P, uint8_t* smem, int32_t* sel_s, long long u0,
                                             long long u1, int warp, int lane) {
  const long long pf = u0 / kTopK;
  const int np = u1 > u0 ? static_cast<int>((u1 - 1) / kTopK - pf + 1) : 0;
  int32_t* cnt_s = sel_s + kSelPairs * kTopK;
  uint64_t* wsm = reinterpret_cast<uint64_t*>(smem + Layout::kStageOff) +
                  warp * (sel::KeySmem<32>::kBytesPerWarp / sizeof(uint64_t));
  for (int i = warp; i < np && i < kSelPairs; i += kWarps) {
    const long long pair = pf + i;
    int32_t* row = sel_s + i * kTopK;
    sel::select_pair_any(P.bs, P.q_pos, P.G, P.nblk, P.capacity, row, cnt_s + i, static_cast<int>(pair), lane,
                         wsm);
    __syncwarp();
    if (pair * kTopK >= u0) {
      if (lane < kTopK) P.sel_out[pair * kTopK + lane] = row[lane];
      if (lane == 0 && P.n_sel_out != nullptr) P.n_sel_out[pair] = cnt_s[i];
    }
    __syncwarp();
  }
  // the keys were stored to the stage ring, which TMA writes next
  fence_proxy_async_smem();
}

// The kernel body for CTA `cta` of the P.n_cta sharing the units.  tm_k, tm_v:
// tensor maps of the K and V caches (block path); tm_q: of Q, [n_q * Hq][128]
// with [16][64] boxes; smem: Layout::kBytes, 1024-byte aligned; the CTA has
// kThreads threads.  kSel: rank the block scores first (P.bs).
template <bool kTok, bool kSel>
__device__ __forceinline__ void sparse_attn_decode_sk_body(const CUtensorMap* tm_k, const CUtensorMap* tm_v,
                                                           const CUtensorMap* tm_q, const Params& P, uint8_t* smem,
                                                           int cta) {
  static_assert(!(kTok && kSel), "the token-level variant takes its selection from the caller");
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + Layout::kBarOff);
  uint64_t* empty = full + kStages;
  UnitInfo* info = reinterpret_cast<UnitInfo*>(smem + Layout::kInfoOff);
  int32_t* sel_s = reinterpret_cast<int32_t*>(smem + Layout::kSelOff);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const long long U = P.n_units;
  const long long u0 = unit_begin(U, P.n_cta, cta);
  const long long u1 = unit_begin(U, P.n_cta, cta + 1);

  if (threadIdx.x == kWarps * 32) {
    // the producer thread sets up the ring while the consumer warps rank
    for (int st = 0; st < kStages; ++st) {
      // token gathers: one arrival per producer lane (its copies landed) and
      // one per producer warp (its record written); TMA: the producer's one
      mbar_init(&full[st], kTok ? (32 + 1) * kGatherWarps : 1);
      mbar_init(&empty[st], kWarps);
    }
    mbar_fence_init();
    if (u1 > u0) {                                 // the first unit's query, into L1
      const int qi = static_cast<int>(u0 / kTopK / P.G);
      prefetch_l1(P.q_stream + qi);
      prefetch_l1(P.q_pos + qi);
    }
  }
  // merges of cut pairs: this CTA's epoch (as a merger), and the flag value
  // it publishes with its first pair's partial when that pair began earlier
  unsigned long long pub = 0ull;
  if (threadIdx.x == 0) {
    *reinterpret_cast<unsigned int*>(smem + Layout::kMiscOff) = __ldcg(&P.sync[cta].epoch);
    const long long first = u0 / kTopK * kTopK;
    if (u1 > u0 && first < u0) {
      const int m = cta_of(U, P.n_cta, first);
      pub = kFlagTag | (static_cast<unsigned long long>(m) << 32) | (__ldcg(&P.sync[m].epoch) + 1u);
    }
  }
  if constexpr (kSel) {
    if (warp < kWarps) select_share(P, smem, sel_s, u0, u1, warp, lane);
  }
  __syncthreads();

  if (kTok && warp >= kWarps) {
    // ----------------------- producer: token gathers (whole warp) -----------------------
    const __nv_bfloat16* kc = reinterpret_cast<const __nv_bfloat16*>(P.k_cache);
    const __nv_bfloat16* vc = reinterpret_cast<const __nv_bfloat16*>(P.v_cache);
    const int pw = warp - kWarps;
    int k = 0;
    bool ok = true;
    for (long long u = u0; u < u1; ++u, ++k) {
      const int st = k % kStages;
      const int use = k / kStages;
      if (use > 0) ok = mbar_wait(&empty[st], (use - 1) & 1);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      int s = 0, g = 0, p = 0;
      const int32_t* toks = nullptr;
      const bool any = tok_unit(P, u, s, g, p, toks, pw == 0 && lane == 0);
      const bool qstart = u == u0 || u % kTopK == 0;
      const uint32_t dst = smem_addr(smem + Layout::kStageOff + st * kStageBytes);
      uint32_t m[2] = {0u, 0u};
      if (any) {
        // one row per lane (two producer warps: 64 rows each), all 16 chunks
        // of K and V; measured faster than spreading a row over 16 lanes
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const int r = pw * 64 + lane + 32 * i;
          const int tok = __ldg(toks + r);
          const long long row = tok_row(P, s, g, p, tok);
          if (row < 0 && tok >= 0) raise_error(tok > p ? MSA_DEVERR_SEL_RANGE : MSA_DEVERR_PAGE_RANGE);
          m[i] = __ballot_sync(0xffffffffu, row >= 0);
          const uint8_t* ksrc = row < 0 ? g_zero_row : reinterpret_cast<const uint8_t*>(kc + row * kD);
          const uint8_t* vsrc = row < 0 ? g_zero_row : reinterpret_cast<const uint8_t*>(vc + row * kD);
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const uint32_t off = (c >> 3) * kTileBytes + swz128(r, c & 7);
            cp_async16(dst + off, ksrc + 16 * c);
            cp_async16(dst + 2 * kTileBytes + off, vsrc + 16 * c);
          }
        }
      }
      if (lane == 0) {
        UnitInfo& in = info[st];
        in.mask[2 * pw] = m[0];
        in.mask[2 * pw + 1] = m[1];
        if (pw == 0) {
          in.flags = (any ? kUnitData : 0) | (qstart ? kUnitQ : 0);
          in.p = p;
          in.slot0 = 0;
          if (qstart) {
            // the record's arrival also announces the pair's Q
            const int qrow = static_cast<int>(u / kTopK) * kHpg;
            uint8_t* qdst = smem + Layout::kQOff + st * kQBytes;
            mbar_arrive_expect_tx(&full[st], kQBytes);
            tma_load_2d(qdst, tm_q, 0, qrow, &full[st]);
            tma_load_2d(qdst + kQBytes / 2, tm_q, 64, qrow, &full[st]);
          } else {
            mbar_arrive(&full[st]);
          }
        } else {
          mbar_arrive(&full[st]);
        }
      }
      cp_async_arrive(&full[st]);
    }
    // no copy may still be landing when the CTA exits
    for (int j = max(0, k - kStages); j < k; ++j) mbar_wait(&full[j % kStages], (j / kStages) & 1);
    return;
  }
  if (!kTok && warp >= kWarps) {
    // -------------------------------- producer --------------------------------
    if (warp != kWarps || lane != 0) return;
    const long long pf = u0 / kTopK;
    int k = 0;
    bool ok = true;
    for (long long u = u0; u < u1; ++u, ++k) {
      const int st = k % kStages;
      const int use = k / kStages;
      if (use > 0) ok = mbar_wait(&empty[st], (use - 1) & 1);
      if (!ok) break;
      int p = 0, slot0 = 0;
      const int row = unit_row(P, u, p, slot0, true, kSel ? sel_s : nullptr, pf);
      const bool qstart = u == u0 || u % kTopK == 0;
      UnitInfo& in = info[st];
      in.flags = (row >= 0 ? kUnitData : 0) | (qstart ? kUnitQ : 0);
      in.p = p;
      in.slot0 = slot0;
      mbar_arrive_expect_tx(&full[st], (row >= 0 ? kStageBytes : 0u) + (qstart ? kQBytes : 0u));
      if (qstart) {
        const int qrow = static_cast<int>(u / kTopK) * kHpg;
        uint8_t* qdst = smem + Layout::kQOff + st * kQBytes;
        tma_load_2d(qdst, tm_q, 0, qrow, &full[st]);
        tma_load_2d(qdst + kQBytes / 2, tm_q, 64, qrow, &full[st]);
      }
      if (row >= 0) {
        uint8_t* dst = smem + Layout::kStageOff + st * kStageBytes;
        tma_load_2d(dst, tm_k, 0, row, &full[st]);
        tma_load_2d(dst + kTileBytes, tm_k, 64, row, &full[st]);
        tma_load_2d(dst + 2 * kTileBytes, tm_v, 0, row, &full[st]);
        tma_load_2d(dst + 3 * kTileBytes, tm_v, 64, row, &full[st]);
      }
    }
    // no copy may still be landing when the CTA exits
    for (int j = max(0, k - kStages); j < k; ++j) mbar_wait(&full[j % kStages], (j / kStages) & 1);
    return;
  }

  // -------------------------------- consumers --------------------------------
  const int tq = lane & 3;    // thread in quad
  const int wr = warp * kRowsPerWarp;
  uint32_t qa[8][4];
  float o[16][4];
  float m_run[2], l_run[2];
  long long cur = -1;
  int k = 0;
  bool ok = true;
  for (long long u = u0; u < u1; ++u, ++k) {
    const int st = k % kStages;
    if (ok) ok = mbar_wait(&full[st], (k / kStages) & 1);
    ok = __all_sync(0xffffffffu, ok);     // warp-uniform: the MMAs below take the whole warp
    const long long pair = u / kTopK;
    if (pair != cur) {
      if (cur >= 0) flush_pair(P, smem, cur, u0, u1, cta, o, m_run, l_run, warp, lane, pub);
      cur = pair;
#pragma unroll
      for (int n = 0; n < 16; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
      m_run[0] = m_run[1] = -INFINITY;
      l_run[0] = l_run[1] = 0.f;
      // Q of the pair's 16 heads as the A operand, from the Q boxes that
      // landed with this unit
      const uint32_t qbase = smem_addr(smem + Layout::kQOff + st * kQBytes);
      const int mi = lane >> 3;
      const int qr = (mi & 1) * 8 + (lane & 7);
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const int kc = ks * 2 + (mi >> 1);    // 16-byte chunk of dims 8kc .. 8kc + 7
        ldmatrix_x4(qa[ks], qbase + (kc >> 3) * (kQBytes / 2) + swz128(qr, kc & 7));
      }
    }
    const int flags = info[st].flags;
    if (ok && (flags & kUnitData)) {
      const int p = info[st].p;
      const int slot0 = info[st].slot0;
      const uint32_t kbase = smem_addr(smem + Layout::kStageOff + st * kStageBytes);
      const uint32_t vbase = kbase + 2 * kTileBytes;
      // S = Q K^T: two n-tiles of 8 key rows
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
      // causal mask inside the block (token path: the unit's row mask),
      // base-2 scaling, online softmax
      uint32_t rmask = 0u;
      if constexpr (kTok) rmask = info[st].mask[warp >> 1] >> ((warp & 1) * 16);   // this warp's 16 rows
      float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int rr = nt * 8 + tq * 2 + (e & 1);    // row within this warp's 16
          bool valid;
          if constexpr (kTok) {
            valid = (rmask >> rr) & 1u;
          } else {
            valid = slot0 + wr + rr <= p;
          }
          const float x = valid ? sacc[nt][e] * P.scale_log2 : -INFINITY;
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
        alpha[h] = exp2f(m_run[h] - m_use[h]);
        m_run[h] = m_new;
      }
      // P rounded to bf16 as the P . V product takes it, and the row sum of
      // those rounded values, so the normalisation matches the weights used
      float rs[2] = {0.f, 0.f};
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float pe = __bfloat162float(__float2bfloat16_rn(exp2f(sacc[nt][e] - m_use[e >> 1])));
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
      // O += P V: P (16 heads x 16 rows) is the A operand of one k-step
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
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[st]);
  }
  if (cur >= 0) flush_pair(P, smem, cur, u0, u1, cta, o, m_run, l_run, warp, lane, pub);
}

template <bool kTok, bool kSel>
__global__ void __launch_bounds__(kThreads, 1)
    sparse_attn_decode_sk_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                                 const __grid_constant__ CUtensorMap tm_q, const Params P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  if (threadIdx.x == kWarps * 32 && !kTok) {       // descriptors fetched before the dependency wait
    prefetch_tensormap(&tm_k);
    prefetch_tensormap(&tm_v);
    prefetch_tensormap(&tm_q);
  }
  pdl_trigger();
  pdl_wait();
  sparse_attn_decode_sk_body<kTok, kSel>(&tm_k, &tm_v, &tm_q, P, smem, blockIdx.x);
}

}  // namespace dattn
}  // namespace msa
