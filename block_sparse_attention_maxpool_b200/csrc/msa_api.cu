// C ABI of the MSA hot path (declarations and contracts in include/msa.h).
// Host-side argument checks, launch configuration and TMA descriptors; the
// kernels live in the msa_*.cuh headers included below (one translation
// unit, so the per-device error word needs no relocatable device code).
#include <algorithm>
#include <atomic>
#include <type_traits>
#include <cmath>
#include <cstdint>
#include <mutex>
#include <utility>

#include "msa.h"
#include "msa_append.cuh"
#include "msa_attn_decode_sk.cuh"
#include "msa_attn_prefill_union.cuh"
#include "msa_common.cuh"
#include "msa_decode_fused.cuh"
#include "msa_dsa_scores.cuh"
#include "msa_dsa_select.cuh"
#include "msa_scores_gemv.cuh"
#include "msa_scores_tc.cuh"
#include "msa_select.cuh"

namespace {

constexpr int kVersion = 100;  // 0.1.0

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_shape(const msa_shape* sh) {
  if (sh == nullptr) return MSA_ERR_NULL;
  if (sh->n_streams <= 0 || sh->capacity <= 0 || sh->block != 128 || sh->capacity % 128 != 0 ||
      sh->head_dim != 128 || sh->idx_dim != 128 || sh->top_k != 16 || sh->n_kv_heads < 1 ||
      sh->n_kv_heads > 16 || sh->n_q_heads != 16 * sh->n_kv_heads)
    return MSA_ERR_SHAPE;
  // every cache row index must fit a signed 32-bit TMA coordinate
  if (static_cast<int64_t>(sh->n_streams) * sh->n_kv_heads * sh->capacity >= (int64_t{1} << 31))
    return MSA_ERR_SHAPE;
  return MSA_OK;
}

int cuda_status(cudaError_t e) { return e == cudaSuccess ? MSA_OK : MSA_ERR_CUDA; }

// Device view of a page table (null: contiguous caches) and the number of
// rows of the cache (or page pool) viewed as 2-D [rows][128].  Every row
// index must fit a signed 32-bit TMA coordinate.
int pages_of(const msa_shape* sh, const msa_pages* pg, msa::KvPages* out, int64_t* rows) {
  out->table = nullptr;
  out->n_pages = 0;
  *rows = static_cast<int64_t>(sh->n_streams) * sh->n_kv_heads * sh->capacity;
  if (pg == nullptr) return MSA_OK;
  if (pg->block_table == nullptr) return MSA_ERR_NULL;
  if ((reinterpret_cast<uintptr_t>(pg->block_table) & 3u) != 0) return MSA_ERR_ALIGN;
  if (pg->n_pages <= 0) return MSA_ERR_RANGE;
  *rows = static_cast<int64_t>(pg->n_pages) * sh->n_kv_heads * 128;
  if (*rows >= (int64_t{1} << 31)) return MSA_ERR_SHAPE;
  out->table = pg->block_table;
  out->n_pages = pg->n_pages;
  return MSA_OK;
}

// Every kernel is launched with programmatic stream serialization: its grid
// may begin launching while the previous kernel in the stream finishes (so
// launch latency and the prologue overlap it); the kernel waits in
// pdl_wait() before it touches global memory, so results are the same as
// with plain stream order.
template <typename... Params, typename... Args>
cudaError_t launch(void (*kernel)(Params...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                   Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

int current_device_sms(int* sms) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MSA_ERR_CUDA;
  if (cudaDeviceGetAttribute(sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return MSA_ERR_CUDA;
  return MSA_OK;
}

// Opt a kernel into more than 48 KB of dynamic shared memory, once per device.
template <typename Kernel>
int ensure_smem(Kernel kernel, size_t bytes, std::atomic<uint64_t>& done_mask) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MSA_ERR_CUDA;
  const uint64_t bit = uint64_t{1} << (dev & 63);
  if (done_mask.load(std::memory_order_acquire) & bit) return MSA_OK;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes)) !=
      cudaSuccess)
    return MSA_ERR_CUDA;
  done_mask.fetch_or(bit, std::memory_order_acq_rel);
  return MSA_OK;
}

// ---- TMA descriptors ----------------------------------------------------------
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                   CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                   CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled() {
  static EncodeTiledFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return static_cast<EncodeTiledFn>(nullptr);
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

// A [rows][128] tensor of 16-bit elements viewed as 2-D; boxes of 128 rows x
// 64 columns (128 bytes, the widest box the 128-byte swizzle allows).
int make_map_16bit(CUtensorMap* m, CUtensorMapDataType dtype, const void* base, int64_t rows,
                   uint32_t box_rows = 128) {
  EncodeTiledFn enc = encode_tiled();
  if (enc == nullptr) return MSA_ERR_CUDA;
  const cuuint64_t dims[2] = {128, static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {128 * 2};
  const cuuint32_t box[2] = {64, box_rows};
  const cuuint32_t estride[2] = {1, 1};
  const CUresult r = enc(m, dtype, 2, const_cast<void*>(base), dims, strides, box, estride,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? MSA_OK : MSA_ERR_CUDA;
}

int make_kv_map(CUtensorMap* m, const void* base, int64_t rows) {
  return make_map_16bit(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, base, rows);
}

// Block scores take the tensor-core tile path for prefill-shaped batches:
// at least 256 queries and on average at least 64 per stream (so tiles of
// 128 consecutive queries mostly share a stream).  A function of the shape
// and the count only, so the workspace query and the call agree.
bool scores_use_tiles(const msa_shape* sh, int32_t n_q) {
  return n_q >= 256 && static_cast<int64_t>(n_q) >= int64_t{64} * sh->n_streams;
}

size_t scores_workspace(const msa_shape* sh, int32_t n_q) {
  if (!scores_use_tiles(sh, n_q)) return 0;
  return msa::tc::workspace_layout(n_q, sh->n_kv_heads, sh->n_streams, sh->capacity).total;
}

// Decode attention workspace: the merge bookkeeping of kMaxCtas CTA slots
// (kept from call to call), then one partial result per CTA of the
// persistent grid (at most kMaxCtas CTAs, at most one per unit).  Depends
// only on the pair count, so the workspace query and the launch always agree.

// Prefill attention: the plan of every 8-query tile.
int64_t union_tasks(const msa_shape* sh, int32_t n_q) {
  return static_cast<int64_t>(sh->n_kv_heads) * ((n_q + msa::uattn::kTileQ - 1) / msa::uattn::kTileQ);
}

size_t attn_workspace(const msa_shape* sh, int32_t n_q, int mode) {
  if (n_q == 0) return 0;
  if (mode == MSA_MODE_PREFILL) return static_cast<size_t>(union_tasks(sh, n_q)) * sizeof(msa::uattn::Plan);
  const int64_t units = static_cast<int64_t>(n_q) * sh->n_kv_heads * msa::dattn::kTopK;
  const int64_t ctas = std::min<int64_t>(units, msa::dattn::kMaxCtas);
  return msa::dattn::kSyncBytes + static_cast<size_t>(ctas) * msa::dattn::kPartial * sizeof(float);
}

// CTAs of the decode attention grid.  The even split (one CTA per SM, equal
// shares) cuts pairs at arbitrary units, and a pair's merger then waits for
// CTAs that hold a different amount of that pair.  When the pairs fit, k
// CTAs per pair (k dividing 16, as many as the SMs allow) gives shares that
// line up with pair boundaries: the CTAs of a pair finish together, and
// with k = 1 nothing is merged.  Measured on 148 SMs: 128 pairs, 128 CTAs
// instead of 148: 4 us less per step; 32 pairs, 128 instead of 148: 2 us.
// It is taken unless its shares are more than two units longer.
int decode_attn_ctas(int64_t n_pairs, int sms) {
  const int64_t units = n_pairs * msa::dattn::kTopK;
  const int64_t cap = std::min<int64_t>(sms, msa::dattn::kMaxCtas);
  const int64_t even = std::min<int64_t>(cap, units);
  const int64_t even_units = (units + even - 1) / even;
  for (int k = msa::dattn::kTopK; k >= 1; k /= 2) {
    if (n_pairs * k <= cap) return static_cast<int>(msa::dattn::kTopK / k <= even_units + 2 ? n_pairs * k : even);
  }
  return static_cast<int>(even);
}

// Most pairs one CTA's share of the decode units touches.
int64_t max_pairs_per_cta(int64_t units, int n_cta) {
  int64_t most = 0;
  for (int c = 0; c < n_cta; ++c) {
    const int64_t u0 = msa::dattn::unit_begin(units, n_cta, c), u1 = msa::dattn::unit_begin(units, n_cta, c + 1);
    if (u1 > u0) most = std::max(most, (u1 - 1) / msa::dattn::kTopK - u0 / msa::dattn::kTopK + 1);
  }
  return most;
}

// Decode and prefill attention over a selection.  Decode with block_scores
// set: the top-16 is taken inside the attention kernel (or, when a CTA's
// share would touch more than kSelPairs pairs, by the selection kernel
// first) and written to sel_out / n_sel_out; `sel` is then sel_out.
int sparse_attn(const msa_shape* sh, const msa_bf16* q, const msa_bf16* k_cache, const msa_bf16* v_cache,
                const int32_t* sel, const int32_t* q_stream, const int32_t* q_pos, int32_t n_q,
                float softmax_scale, msa_bf16* out, void* workspace, size_t workspace_bytes, void* stream,
                int mode, const msa_pages* pages, const int32_t* tok_sel = nullptr,
                const float* block_scores = nullptr, int32_t* sel_out = nullptr, int32_t* n_sel_out = nullptr) {
  int st = check_shape(sh);
  if (st != MSA_OK) return st;
  if (n_q < 0) return MSA_ERR_RANGE;
  if (n_q == 0) return MSA_OK;
  if (!q || !k_cache || !v_cache || !sel || !q_stream || !q_pos || !out) return MSA_ERR_NULL;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(sel) || !aligned16(out))
    return MSA_ERR_ALIGN;
  if (!std::isfinite(softmax_scale)) return MSA_ERR_RANGE;
  const int G = sh->n_kv_heads;
  const int64_t n_pairs = static_cast<int64_t>(n_q) * G;
  if (n_pairs * msa::dattn::kTopK >= (int64_t{1} << 40)) return MSA_ERR_RANGE;
  msa::KvPages pg;
  int64_t rows = 0;
  if ((st = pages_of(sh, pages, &pg, &rows)) != MSA_OK) return st;
  const size_t need = attn_workspace(sh, n_q, mode);
  if (need > 0) {
    if (workspace == nullptr || workspace_bytes < need) return MSA_ERR_WORKSPACE;
    if (!aligned16(workspace)) return MSA_ERR_ALIGN;
  }
  CUtensorMap tm_k, tm_v;
  if ((st = make_kv_map(&tm_k, k_cache, rows)) != MSA_OK) return st;
  if ((st = make_kv_map(&tm_v, v_cache, rows)) != MSA_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int sms = 0;
  if ((st = current_device_sms(&sms)) != MSA_OK) return st;
  if (mode == MSA_MODE_PREFILL) {
    // tensor-core kernels, one persistent CTA per SM: tiles of 8 queries over the
    // union of their selected blocks; a first kernel plans every tile into the
    // workspace, the attention kernel reads the plans after its dependent-launch wait
    CUtensorMap tm_q;
    if ((st = make_map_16bit(&tm_q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, q,
                             static_cast<int64_t>(n_q) * sh->n_q_heads, 16)) != MSA_OK)
      return st;
    const auto ukernel = pg.table != nullptr ? msa::uattn::sparse_attn_prefill_union_kernel<true>
                                             : msa::uattn::sparse_attn_prefill_union_kernel<false>;
    static std::atomic<uint64_t> u_smem_done[2] = {0, 0};
    if ((st = ensure_smem(ukernel, msa::uattn::Layout::kBytes, u_smem_done[pg.table != nullptr])) != MSA_OK)
      return st;
    msa::uattn::Params U;
    U.sel = sel;
    U.q_stream = q_stream;
    U.q_pos = q_pos;
    U.out = reinterpret_cast<__nv_bfloat16*>(out);
    U.n_q = n_q;
    U.G = G;
    U.n_streams = sh->n_streams;
    U.capacity = sh->capacity;
    U.n_tiles = (n_q + msa::uattn::kTileQ - 1) / msa::uattn::kTileQ;
    U.scale_log2 = softmax_scale * 1.4426950408889634f;
    U.pages = pg;
    U.plans = static_cast<msa::uattn::Plan*>(workspace);
    const int64_t tasks = static_cast<int64_t>(G) * U.n_tiles;
    const int64_t ugrid = std::min<int64_t>(sms, tasks);
    const auto pkernel_plan = pg.table != nullptr ? msa::uattn::plan_tiles_kernel<true>
                                                  : msa::uattn::plan_tiles_kernel<false>;
    launch(pkernel_plan, dim3(static_cast<unsigned>((tasks + 7) / 8)), dim3(256), 0, s, U);
    launch(ukernel, dim3(static_cast<unsigned>(ugrid)), dim3(msa::uattn::kThreads), msa::uattn::Layout::kBytes, s, tm_q,
           tm_k, tm_v, U);
    return cuda_status(cudaGetLastError());
  }
  // decode: persistent stream-K grid over (pair, selected block) units, or
  // (pair, chunk of 128 kept tokens) units for the token-level variant
  if (n_pairs * msa::dattn::kHpg >= (int64_t{1} << 31)) return MSA_ERR_RANGE;   // Q rows: TMA coordinates
  CUtensorMap tm_q;
  if ((st = make_map_16bit(&tm_q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, q, n_pairs * msa::dattn::kHpg,
                           msa::dattn::kHpg)) != MSA_OK)
    return st;
  const int64_t n_units = n_pairs * msa::dattn::kTopK;
  const int n_cta = decode_attn_ctas(n_pairs, sms);
  bool fuse_sel = false;
  if (block_scores != nullptr) {
    fuse_sel = max_pairs_per_cta(n_units, n_cta) <= msa::dattn::kSelPairs;
    if (!fuse_sel && (st = msa_select_topk(sh, block_scores, q_pos, n_q, sel_out, n_sel_out, stream)) != MSA_OK)
      return st;
  }
  const int variant = tok_sel != nullptr ? 1 : (fuse_sel ? 2 : 0);
  const auto kernel = variant == 1 ? msa::dattn::sparse_attn_decode_sk_kernel<true, false>
                                   : (variant == 2 ? msa::dattn::sparse_attn_decode_sk_kernel<false, true>
                                                   : msa::dattn::sparse_attn_decode_sk_kernel<false, false>);
  static std::atomic<uint64_t> smem_done[3] = {0, 0, 0};
  if ((st = ensure_smem(kernel, msa::dattn::Layout::kBytes, smem_done[variant])) != MSA_OK) return st;
  msa::dattn::Params P;
  P.q = reinterpret_cast<const __nv_bfloat16*>(q);
  P.sel = sel;
  P.q_stream = q_stream;
  P.q_pos = q_pos;
  P.out = reinterpret_cast<__nv_bfloat16*>(out);
  P.sync = static_cast<msa::dattn::SyncSlot*>(workspace);
  P.ws = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + msa::dattn::kSyncBytes);
  P.n_q = n_q;
  P.G = G;
  P.n_streams = sh->n_streams;
  P.capacity = sh->capacity;
  P.n_units = n_units;
  P.n_cta = n_cta;
  P.scale_log2 = softmax_scale * 1.4426950408889634f;
  P.pages = pg;
  P.tok_sel = tok_sel;
  P.k_cache = reinterpret_cast<const __nv_bfloat16*>(k_cache);
  P.v_cache = reinterpret_cast<const __nv_bfloat16*>(v_cache);
  P.bs = fuse_sel ? block_scores : nullptr;
  P.nblk = sh->capacity / msa::dattn::kBlock;
  P.sel_out = fuse_sel ? sel_out : nullptr;
  P.n_sel_out = fuse_sel ? n_sel_out : nullptr;
  launch(kernel, dim3(static_cast<unsigned>(P.n_cta)), dim3(msa::dattn::kThreads), msa::dattn::Layout::kBytes, s,
         tm_k, tm_v, tm_q, P);
  return cuda_status(cudaGetLastError());
}

int append_rows(const msa_shape* sh, void* cache0, const void* src0, void* cache1, const void* src1,
                const int32_t* tok_stream, const int32_t* tok_pos, int32_t n_tok, int row_bytes,
                void* stream, const msa_pages* pages) {
  int st = check_shape(sh);
  if (st != MSA_OK) return st;
  if (n_tok < 0) return MSA_ERR_RANGE;
  if (n_tok == 0) return MSA_OK;
  if (!cache0 || !src0 || !tok_stream || !tok_pos) return MSA_ERR_NULL;
  if (!aligned16(cache0) || !aligned16(src0) || (cache1 && !aligned16(cache1)) || (src1 && !aligned16(src1)))
    return MSA_ERR_ALIGN;
  msa::KvPages pg;
  int64_t rows = 0;
  if ((st = pages_of(sh, pages, &pg, &rows)) != MSA_OK) return st;
  const int64_t warps = static_cast<int64_t>(n_tok) * sh->n_kv_heads;
  if (warps * 32 >= (int64_t{1} << 31)) return MSA_ERR_RANGE;
  const unsigned grid = static_cast<unsigned>((warps * 32 + 255) / 256);
  launch(msa::append_rows_kernel, dim3(grid), dim3(256), 0, static_cast<cudaStream_t>(stream), 
      static_cast<uint8_t*>(cache0), static_cast<const uint8_t*>(src0), static_cast<uint8_t*>(cache1),
      static_cast<const uint8_t*>(src1), tok_stream, tok_pos, n_tok, sh->n_streams, sh->n_kv_heads,
      sh->capacity, row_bytes, pg);
  return cuda_status(cudaGetLastError());
}

// The appends of one step (F32 indexer keys, K, V) in one launch.
int step_append(const msa_shape* sh, float* idx_k_cache, msa_bf16* k_cache, msa_bf16* v_cache,
                const float* idx_k_new, const msa_bf16* k_new, const msa_bf16* v_new, const int32_t* tok_stream,
                const int32_t* tok_pos, int32_t n_tok, void* stream, const msa_pages* pages) {
  int st = check_shape(sh);
  if (st != MSA_OK) return st;
  if (n_tok < 0) return MSA_ERR_RANGE;
  if (n_tok == 0) return MSA_OK;
  if (!idx_k_cache || !k_cache || !v_cache || !idx_k_new || !k_new || !v_new || !tok_stream || !tok_pos)
    return MSA_ERR_NULL;
  if (!aligned16(idx_k_cache) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(idx_k_new) ||
      !aligned16(k_new) || !aligned16(v_new))
    return MSA_ERR_ALIGN;
  msa::KvPages pg;
  int64_t rows = 0;
  if ((st = pages_of(sh, pages, &pg, &rows)) != MSA_OK) return st;
  const int64_t warps = static_cast<int64_t>(n_tok) * sh->n_kv_heads;
  if (warps * 32 >= (int64_t{1} << 31)) return MSA_ERR_RANGE;
  const unsigned grid = static_cast<unsigned>((warps * 32 + 255) / 256);
  launch(msa::append_step_kernel, dim3(grid), dim3(256), 0, static_cast<cudaStream_t>(stream), idx_k_cache,
         idx_k_new, reinterpret_cast<uint8_t*>(k_cache), reinterpret_cast<const uint8_t*>(k_new),
         reinterpret_cast<uint8_t*>(v_cache), reinterpret_cast<const uint8_t*>(v_new), tok_stream, tok_pos, n_tok,
         sh->n_streams, sh->n_kv_heads, sh->capacity, pg);
  return cuda_status(cudaGetLastError());
}

template <typename KeyT>
int block_scores_impl(const msa_shape* shape, const float* idx_q, const KeyT* idx_k_cache,
                      const int32_t* q_stream, const int32_t* q_pos, int32_t n_q, float* block_scores,
                      void* workspace, size_t workspace_bytes, void* stream, const msa_pages* pages) {
  constexpr bool kF16 = std::is_same<KeyT, __half>::value;
  using Cfg = msa::gemv::Config<KeyT>;
  int st = check_shape(shape);
  if (st != MSA_OK) return st;
  if (n_q < 0) return MSA_ERR_RANGE;
  if (n_q == 0) return MSA_OK;
  if (!idx_q || !idx_k_cache || !q_stream || !q_pos || !block_scores) return MSA_ERR_NULL;
  if (!aligned16(idx_q) || !aligned16(idx_k_cache) || !aligned16(block_scores)) return MSA_ERR_ALIGN;
  msa::KvPages pg;
  int64_t key_rows_all = 0;
  if ((st = pages_of(shape, pages, &pg, &key_rows_all)) != MSA_OK) return st;
  const bool tiles = scores_use_tiles(shape, n_q);
  const size_t need = scores_workspace(shape, n_q);
  if (need > 0) {
    if (workspace == nullptr || workspace_bytes < need) return MSA_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return MSA_ERR_ALIGN;
  }
  int sms = 0;
  if ((st = current_device_sms(&sms)) != MSA_OK) return st;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  const int G = shape->n_kv_heads;
  const int S = shape->n_streams;
  const int cap = shape->capacity;

  using namespace msa::gemv;
  Params<KeyT> P;
  P.idx_q = idx_q;
  P.idx_k = idx_k_cache;
  P.q_stream = q_stream;
  P.q_pos = q_pos;
  P.bs = block_scores;
  P.n_q = n_q;
  P.G = G;
  P.n_streams = S;
  P.capacity = cap;
  P.nblk = cap / 128;
  P.n_tasks = static_cast<long long>(n_q) * G * P.nblk;
  P.q_list = nullptr;
  P.q_count = nullptr;
  P.pages = pg;
  const size_t smem = sizeof(Smem<KeyT, Cfg::kStages, Cfg::kWarps>);
  const auto kernel = block_scores_gemv_kernel<KeyT, Cfg::kStages, Cfg::kWarps, Cfg::kCtasPerSm>;
  constexpr int kThreads = (Cfg::kWarps + 1) * 32;
  static std::atomic<uint64_t> smem_done{0};
  if ((st = ensure_smem(kernel, smem, smem_done)) != MSA_OK) return st;

  if (tiles) {
    namespace T = msa::tc;
    const T::Workspace L = T::workspace_layout(n_q, G, S, cap);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    T::Params Q;
    Q.idx_q = idx_q;
    Q.idx_k = kF16 ? nullptr : reinterpret_cast<const float*>(idx_k_cache);
    Q.idx_k16 = kF16 ? reinterpret_cast<const __half*>(idx_k_cache) : nullptr;
    Q.q_stream = q_stream;
    Q.q_pos = q_pos;
    Q.bs = block_scores;
    Q.n_q = n_q;
    Q.G = G;
    Q.n_streams = S;
    Q.capacity = cap;
    Q.nblk = cap / 128;
    Q.n_tiles = L.n_tiles;
    Q.n_q_pad = L.n_q_pad;
    Q.n_chunks = (Q.nblk + T::kChunk - 1) / T::kChunk;
    Q.counters = reinterpret_cast<int*>(ws + L.counters);
    Q.tile_stream = reinterpret_cast<int*>(ws + L.tile_stream);
    Q.tile_nb = reinterpret_cast<int*>(ws + L.tile_nb);
    Q.leftover = reinterpret_cast<int*>(ws + L.leftover);
    Q.qscale = reinterpret_cast<float*>(ws + L.qscale);
    Q.qhi = reinterpret_cast<__half*>(ws + L.qhi);
    Q.qlo = reinterpret_cast<__half*>(ws + L.qlo);
    Q.kscale = reinterpret_cast<float*>(ws + L.kscale);
    Q.khi = reinterpret_cast<__half*>(ws + L.khi);
    Q.klo = reinterpret_cast<__half*>(ws + L.klo);
    Q.qlo_nz = reinterpret_cast<int*>(ws + L.qlo_nz);
    Q.klo_mask = reinterpret_cast<uint32_t*>(ws + L.klo_mask);
    Q.n_flags = G * L.n_tiles + S * G * Q.n_chunks;
    Q.pages = pg;
    const int64_t key_rows = static_cast<int64_t>(S) * G * cap;
    const int64_t q_rows = static_cast<int64_t>(G) * L.n_q_pad;
    CUtensorMap m_qhi, m_qlo, m_khi, m_klo;
    if ((st = make_map_16bit(&m_qhi, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, Q.qhi, q_rows)) != MSA_OK) return st;
    if ((st = make_map_16bit(&m_qlo, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, Q.qlo, q_rows)) != MSA_OK) return st;
    if ((st = make_map_16bit(&m_khi, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, Q.khi, key_rows)) != MSA_OK) return st;
    if ((st = make_map_16bit(&m_klo, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, Q.klo, key_rows)) != MSA_OK) return st;
    static std::atomic<uint64_t> tc_smem_done{0};
    if ((st = ensure_smem(T::block_scores_tc_kernel, T::SmemLayout::kBytes, tc_smem_done)) != MSA_OK) return st;

    launch(T::tc_init_kernel, dim3(1), dim3(1024), 0, cs, Q.counters, 1 + S, Q);
    launch(T::tc_tile_info_kernel, dim3((L.n_tiles * 32 + 255) / 256), dim3(256), 0, cs, Q);
    launch(T::tc_split_queries_kernel, dim3(static_cast<unsigned>((q_rows * 32 + 255) / 256)), dim3(256), 0, cs, Q);
    launch(T::tc_split_keys_kernel, dim3(static_cast<unsigned>((key_rows * 32 + 255) / 256)), dim3(256), 0, cs, Q);
    const int n_tasks = G * Q.n_chunks * Q.n_tiles;
    launch(T::block_scores_tc_kernel, dim3(static_cast<unsigned>(std::min(sms, n_tasks))), dim3(T::kThreads), T::SmemLayout::kBytes, cs, m_qhi, m_qlo, m_khi, m_klo, Q);
    if (cudaGetLastError() != cudaSuccess) return MSA_ERR_CUDA;
    // queries of mixed-stream tiles: streaming kernel over the leftover list
    P.q_list = Q.leftover;
    P.q_count = Q.counters;
    launch(kernel, dim3(static_cast<unsigned>(Cfg::kCtasPerSm * sms)), dim3(kThreads), smem, cs, P);
    return cuda_status(cudaGetLastError());
  }

  const long long grid = std::min<long long>(static_cast<long long>(Cfg::kCtasPerSm) * sms, P.n_tasks);
  launch(kernel, dim3(static_cast<unsigned>(grid)), dim3(kThreads), smem, cs, P);
  return cuda_status(cudaGetLastError());
}

int append_idx_f16(const msa_shape* shape, msa_f16* idx_k_cache, const float* idx_k_new,
                   const int32_t* tok_stream, const int32_t* tok_pos, int32_t n_tok, void* stream,
                   const msa_pages* pages) {
  int st = check_shape(shape);
  if (st != MSA_OK) return st;
  if (n_tok < 0) return MSA_ERR_RANGE;
  if (n_tok == 0) return MSA_OK;
  if (!idx_k_cache || !idx_k_new || !tok_stream || !tok_pos) return MSA_ERR_NULL;
  if (!aligned16(idx_k_cache) || !aligned16(idx_k_new)) return MSA_ERR_ALIGN;
  msa::KvPages pg;
  int64_t rows = 0;
  if ((st = pages_of(shape, pages, &pg, &rows)) != MSA_OK) return st;
  const int64_t warps = static_cast<int64_t>(n_tok) * shape->n_kv_heads;
  if (warps * 32 >= (int64_t{1} << 31)) return MSA_ERR_RANGE;
  const unsigned grid = static_cast<unsigned>((warps * 32 + 255) / 256);
  launch(msa::append_idx_f16_kernel, dim3(grid), dim3(256), 0, static_cast<cudaStream_t>(stream), 
      reinterpret_cast<__half*>(idx_k_cache), idx_k_new, tok_stream, tok_pos, n_tok, shape->n_streams,
      shape->n_kv_heads, shape->capacity, pg);
  return cuda_status(cudaGetLastError());
}

// ---- token-level variant ---------------------------------------------------
int check_dsa_shape(const msa_dsa_shape* sh) {
  if (sh == nullptr) return MSA_ERR_NULL;
  if (sh->n_streams <= 0 || sh->capacity <= 0 || sh->capacity % 128 != 0 || sh->index_dim != 128 ||
      sh->n_index_heads != msa::dsa::kHeads || sh->top_k < 1 || sh->top_k > msa::dsa::kMaxTopK)
    return MSA_ERR_SHAPE;
  if (static_cast<int64_t>(sh->n_streams) * sh->capacity >= (int64_t{1} << 31)) return MSA_ERR_SHAPE;
  return MSA_OK;
}

// The indexer-key cache as an MSA cache of one group: the same page-table
// checks and row counts.
msa_shape dsa_as_msa(const msa_dsa_shape* sh) {
  msa_shape m{};
  m.n_streams = sh->n_streams;
  m.capacity = sh->capacity;
  m.n_q_heads = 16;
  m.n_kv_heads = 1;
  m.head_dim = 128;
  m.idx_dim = 128;
  m.block = 128;
  m.top_k = 16;
  return m;
}

}  // namespace

extern "C" {

int msa_indexer_append(const msa_shape* shape, float* idx_k_cache, const float* idx_k_new,
                       const int32_t* tok_stream, const int32_t* tok_pos, int32_t n_tok, void* stream) {
  return append_rows(shape, idx_k_cache, idx_k_new, nullptr, nullptr, tok_stream, tok_pos, n_tok,
                     128 * static_cast<int>(sizeof(float)), stream, nullptr);
}

int msa_kv_append(const msa_shape* shape, msa_bf16* k_cache, msa_bf16* v_cache, const msa_bf16* k_new,
                  const msa_bf16* v_new, const int32_t* tok_stream, const int32_t* tok_pos, int32_t n_tok,
                  void* stream) {
  if (n_tok > 0 && (!v_cache || !v_new)) return MSA_ERR_NULL;
  return append_rows(shape, k_cache, k_new, v_cache, v_new, tok_stream, tok_pos, n_tok,
                     128 * static_cast<int>(sizeof(msa_bf16)), stream, nullptr);
}

int msa_step_append(const msa_shape* shape, float* idx_k_cache, msa_bf16* k_cache, msa_bf16* v_cache,
                    const float* idx_k_new, const msa_bf16* k_new, const msa_bf16* v_new, const int32_t* tok_stream,
                    const int32_t* tok_pos, int32_t n_tok, void* stream) {
  return step_append(shape, idx_k_cache, k_cache, v_cache, idx_k_new, k_new, v_new, tok_stream, tok_pos, n_tok,
                     stream, nullptr);
}

int msa_step_append_paged(const msa_shape* shape, const msa_pages* pages, float* idx_k_pool, msa_bf16* k_pool,
                          msa_bf16* v_pool, const float* idx_k_new, const msa_bf16* k_new, const msa_bf16* v_new,
                          const int32_t* tok_stream, const int32_t* tok_pos, int32_t n_tok, void* stream) {
  if (pages == nullptr) return MSA_ERR_NULL;
  return step_append(shape, idx_k_pool, k_pool, v_pool, idx_k_new, k_new, v_new, tok_stream, tok_pos, n_tok, stream,
                     pages);
}

int msa_block_scores(const msa_shape* shape, const float* idx_q, const float* idx_k_cache,
                     const int32_t* q_stream, const int32_t* q_pos, int32_t n_q, float* block_scores,
                     void* workspace, size_t workspace_bytes, void* stream) {
  return block_scores_impl<float>(shape, idx_q, idx_k_cache, q_stream, q_pos, n_q, block_scores, workspace,
                                  workspace_bytes, stream, nullptr);
}

int msa_block_scores_f16(const msa_shape* shape, const float* idx_q, const msa_f16* idx_k_cache,
                         const int32_t* q_stream, const int32_t* q_pos, int32_t n_q, float* block_scores,
                         void* workspace, size_t workspace_bytes, void* stream) {
  return block_scores_impl<__half>(shape, idx_q, reinterpret_cast<const __half*>(idx_k_cache), q_stream, q_pos,
                                   n_q, block_scores, workspace, workspace_bytes, stream, nullptr);
}

int msa_indexer_append_f16(const msa_shape* shape, msa_f16* idx_k_cache, const float* idx_k_new,
                           const int32_t* tok_stream, const int32_t* tok_pos, int32_t n_tok, void* stream) {
  return append_idx_f16(shape, idx_k_cache, idx_k_new, tok_stream, tok_pos, n_tok, stream, nullptr);
}

int msa_select_topk(const msa_shape* shape, const float* block_scores, const int32_t* q_pos, int32_t n_q,
                    int32_t* sel, int32_t* n_sel, void* stream) {
  int st = check_shape(shape);
  if (st != MSA_OK) return st;
  if (n_q < 0) return MSA_ERR_RANGE;
  if (n_q == 0) return MSA_OK;
  if (!block_scores || !q_pos || !sel) return MSA_ERR_NULL;
  if (!aligned16(block_scores) || !aligned16(sel)) return MSA_ERR_ALIGN;
  const int G = shape->n_kv_heads;
  const int nblk = shape->capacity / 128;
  const int64_t warps = static_cast<int64_t>(n_q) * G;
  if (warps * 32 >= (int64_t{1} << 31)) return MSA_ERR_RANGE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  using msa::sel::SelectLaunch;
  auto grid_of = [&](int threads) { return dim3(static_cast<unsigned>((warps * 32 + threads - 1) / threads)); };
  if (nblk <= 32 * 8) {
    launch(msa::sel::select_topk_kernel<8>, grid_of(SelectLaunch<8>::kThreads), dim3(SelectLaunch<8>::kThreads),
           SelectLaunch<8>::kSmem, s, block_scores, q_pos, n_q, G, nblk, shape->capacity, sel, n_sel);
  } else if (nblk <= 32 * 32) {
    launch(msa::sel::select_topk_kernel<32>, grid_of(SelectLaunch<32>::kThreads), dim3(SelectLaunch<32>::kThreads),
           SelectLaunch<32>::kSmem, s, block_scores, q_pos, n_q, G, nblk, shape->capacity, sel, n_sel);
  } else {
    launch(msa::sel::select_topk_kernel<0>, grid_of(SelectLaunch<0>::kThreads), dim3(SelectLaunch<0>::kThreads),
           SelectLaunch<0>::kSmem, s, block_scores, q_pos, n_q, G, nblk, shape->capacity, sel, n_sel);
  }
  return cuda_status(cudaGetLastError());
}

int msa_select_attn_decode(const msa_shape* shape, const float* block_scores, const msa_bf16* q,
                           const msa_bf16* k_cache, const msa_bf16* v_cache, const int32_t* q_stream,
                           const int32_t* q_pos, int32_t n_q, float softmax_scale, int32_t* sel, int32_t* n_sel,
                           msa_bf16* out, void* workspace, size_t workspace_bytes, void* stream) {
  if (n_q > 0 && (block_scores == nullptr || sel == nullptr)) return MSA_ERR_NULL;
  if (n_q > 0 && !aligned16(block_scores)) return MSA_ERR_ALIGN;
  return sparse_attn(shape, q, k_cache, v_cache, sel, q_stream, q_pos, n_q, softmax_scale, out, workspace,
                     workspace_bytes, stream, MSA_MODE_DECODE, nullptr, nullptr, block_scores, sel, n_sel);
}

int msa_sparse_attn_decode(const msa_shape* shape, const msa_bf16* q, const msa_bf16* k_cache,
                           const msa_bf16* v_cache, const int32_t* sel, const int32_t* q_stream,
                           const int32_t* q_pos, int32_t n_q, float softmax_scale, msa_bf16* out,
                           void* workspace, size_t workspace_bytes, void* stream) {
  return sparse_attn(shape, q, k_cache, v_cache, sel, q_stream, q_pos, n_q, softmax_scale, out, workspace,
                     workspace_bytes, stream, MSA_MODE_DECODE, nullptr);
}

int msa_sparse_attn_prefill(const msa_shape* shape, const msa_bf16* q, const msa_bf16* k_cache,
                            const msa_bf16* v_cache, const int32_t* sel, const int32_t* q_stream,
                            const int32_t* q_pos, int32_t n_q, float softmax_scale, msa_bf16* out,
                            void* workspace, size_t workspace_bytes, void* stream) {
  return sparse_attn(shape, q, k_cache, v_cache, sel, q_stream, q_pos, n_q, softmax_scale, out, workspace,
                     workspace_bytes, stream, MSA_MODE_PREFILL, nullptr);
}

// ---- attention without a caller workspace ----------------------------------
// File-scope scratch for msa_sparse_attn_decode_noalloc.  In host code the
// name is only a stand-in for the symbol: its device address is looked up
// once per device with cudaGetSymbolAddress and passed to the kernels.
static __device__ __align__(256) unsigned char g_noalloc_scratch[MSA_NOALLOC_SCRATCH_BYTES];

}  // extern "C"

namespace {
// The buffer's device address, per device, with the context it was looked up
// in: a new context on the device (after cudaDeviceReset, or once the
// primary context was released and re-created) holds a new copy of the
// buffer, so the address is looked up again whenever the current context
// differs from the recorded one.
struct NoallocSlot {
  CUcontext ctx;
  void* ptr;
};
std::mutex g_noalloc_mutex;
NoallocSlot g_noalloc[64] = {};

using CtxGetCurrentFn = CUresult (*)(CUcontext*);

CtxGetCurrentFn ctx_get_current() {
  static CtxGetCurrentFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return static_cast<CtxGetCurrentFn>(nullptr);
    return reinterpret_cast<CtxGetCurrentFn>(p);
  }();
  return fn;
}

int noalloc_scratch(void** ptr) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return MSA_ERR_CUDA;
  CtxGetCurrentFn get_ctx = ctx_get_current();
  if (get_ctx == nullptr) return MSA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  CUcontext ctx = nullptr;
  if (get_ctx(&ctx) != CUDA_SUCCESS) return MSA_ERR_CUDA;
  NoallocSlot& slot = g_noalloc[dev];
  if (slot.ptr == nullptr || ctx == nullptr || slot.ctx != ctx) {
    void* p = nullptr;
    // with that device current (it is): also makes the device's primary
    // context current if no context was yet
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return MSA_ERR_CUDA;
    if (get_ctx(&ctx) != CUDA_SUCCESS || ctx == nullptr) return MSA_ERR_CUDA;
    slot.ctx = ctx;
    slot.ptr = p;
  }
  *ptr = slot.ptr;
  return MSA_OK;
}
}  // namespace

extern "C" {

int msa_sparse_attn_decode_noalloc(const msa_shape* shape, const msa_bf16* q, const msa_bf16* k_cache,
                                   const msa_bf16* v_cache, const int32_t* sel, const int32_t* q_stream,
                                   const int32_t* q_pos, int32_t n_q, float softmax_scale, msa_bf16* out,
                                   void* stream) {
  const int st = check_shape(shape);
  if (st != MSA_OK) return st;
  if (n_q < 0) return MSA_ERR_RANGE;
  if (n_q == 0) return MSA_OK;
  // argument errors are reported before the one-time device set-up below
  if (!q || !k_cache || !v_cache || !sel || !q_stream || !q_pos || !out) return MSA_ERR_NULL;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(sel) || !aligned16(out))
    return MSA_ERR_ALIGN;
  if (!std::isfinite(softmax_scale)) return MSA_ERR_RANGE;
  const size_t need = attn_workspace(shape, n_q, MSA_MODE_DECODE);
  if (need > MSA_NOALLOC_SCRATCH_BYTES) return MSA_ERR_WORKSPACE;
  void* scratch = nullptr;
  if (need > 0) {
    const int s2 = noalloc_scratch(&scratch);
    if (s2 != MSA_OK) return s2;
  }
  return sparse_attn(shape, q, k_cache, v_cache, sel, q_stream, q_pos, n_q, softmax_scale, out, scratch,
                     MSA_NOALLOC_SCRATCH_BYTES, stream, MSA_MODE_DECODE, nullptr);
}

// ---- paged caches ----------------------------------------------------------
int msa_indexer_append_paged(const msa_shape* shape, const msa_pages* pages, float* idx_k_pool,
                             const float* idx_k_new, const int32_t* tok_stream, const int32_t* tok_pos,
                             int32_t n_tok, void* stream) {
  if (pages == nullptr) return MSA_ERR_NULL;
  return append_rows(shape, idx_k_pool, idx_k_new, nullptr, nullptr, tok_stream, tok_pos, n_tok,
                     128 * static_cast<int>(sizeof(float)), stream, pages);
}

int msa_indexer_append_f16_paged(const msa_shape* shape, const msa_pages* pages, msa_f16* idx_k_pool,
                                 const float* idx_k_new, const int32_t* tok_stream, const int32_t* tok_pos,
                                 int32_t n_tok, void* stream) {
  if (pages == nullptr) return MSA_ERR_NULL;
  return append_idx_f16(shape, idx_k_pool, idx_k_new, tok_stream, tok_pos, n_tok, stream, pages);
}

int msa_kv_append_paged(const msa_shape* shape, const msa_pages* pages, msa_bf16* k_pool, msa_bf16* v_pool,
                        const msa_bf16* k_new, const msa_bf16* v_new, const int32_t* tok_stream,
                        const int32_t* tok_pos, int32_t n_tok, void* stream) {
  if (pages == nullptr) return MSA_ERR_NULL;
  if (n_tok > 0 && (!v_pool || !v_new)) return MSA_ERR_NULL;
  return append_rows(shape, k_pool, k_new, v_pool, v_new, tok_stream, tok_pos, n_tok,
                     128 * static_cast<int>(sizeof(msa_bf16)), stream, pages);
}

int msa_block_scores_paged(const msa_shape* shape, const msa_pages* pages, const float* idx_q,
                           const float* idx_k_pool, const int32_t* q_stream, const int32_t* q_pos, int32_t n_q,
                           float* block_scores, void* workspace, size_t workspace_bytes, void* stream) {
  if (pages == nullptr) return MSA_ERR_NULL;
  return block_scores_impl<float>(shape, idx_q, idx_k_pool, q_stream, q_pos, n_q, block_scores, workspace,
                                  workspace_bytes, stream, pages);
}

int msa_block_scores_f16_paged(const msa_shape* shape, const msa_pages* pages, const float* idx_q,
                               const msa_f16* idx_k_pool, const int32_t* q_stream, const int32_t* q_pos,
                               int32_t n_q, float* block_scores, void* workspace, size_t workspace_bytes,
                               void* stream) {
  if (pages == nullptr) return MSA_ERR_NULL;
  return block_scores_impl<__half>(shape, idx_q, reinterpret_cast<const __half*>(idx_k_pool), q_stream, q_pos,
                                   n_q, block_scores, workspace, workspace_bytes, stream, pages);
}

int msa_sparse_attn_decode_paged(const msa_shape* shape, const msa_pages* pages, const msa_bf16* q,
                                 const msa_bf16* k_pool, const msa_bf16* v_pool, const int32_t* sel,
                                 const int32_t* q_stream, const int32_t* q_pos, int32_t n_q, float softmax_scale,
                                 msa_bf16* out, void* workspace, size_t workspace_bytes, void* stream) {
  if (pages == nullptr) return MSA_ERR_NULL;
  return sparse_attn(shape, q, k_pool, v_pool, sel, q_stream, q_pos, n_q, softmax_scale, out, workspace,
                     workspace_bytes, stream, MSA_MODE_DECODE, pages);
}

int msa_select_attn_decode_paged(const msa_shape* shape, const msa_pages* pages, const float* block_scores,
                                 const msa_bf16* q, const msa_bf16* k_pool, const msa_bf16* v_pool,
                                 const int32_t* q_stream, const int32_t* q_pos, int32_t n_q, float softmax_scale,
                                 int32_t* sel, int32_t* n_sel, msa_bf16* out, void* workspace,
                                 size_t workspace_bytes, void* stream) {
  if (pages == nullptr) return MSA_ERR_NULL;
  if (n_q > 0 && (block_scores == nullptr || sel == nullptr)) return MSA_ERR_NULL;
  if (n_q > 0 && !aligned16(block_scores)) return MSA_ERR_ALIGN;
  return sparse_attn(shape, q, k_pool, v_pool, sel, q_stream, q_pos, n_q, softmax_scale, out, workspace,
                     workspace_bytes, stream, MSA_MODE_DECODE, pages, nullptr, block_scores, sel, n_sel);
}

int msa_sparse_attn_prefill_paged(const msa_shape* shape, const msa_pages* pages, const msa_bf16* q,
                                  const msa_bf16* k_pool, const msa_bf16* v_pool, const int32_t* sel,
                                  const int32_t* q_stream, const int32_t* q_pos, int32_t n_q,
                                  float softmax_scale, msa_bf16* out, void* workspace, size_t workspace_bytes,
                                  void* stream) {
  if (pages == nullptr) return MSA_ERR_NULL;
  return sparse_attn(shape, q, k_pool, v_pool, sel, q_stream, q_pos, n_q, softmax_scale, out, workspace,
                     workspace_bytes, stream, MSA_MODE_PREFILL, pages);
}

// ---- token-level variant ---------------------------------------------------
int msa_dsa_indexer_append(const msa_dsa_shape* shape, const msa_pages* pages, msa_f16* k_idx_cache,
                           const float* k_idx_new, const int32_t* tok_stream, const int32_t* tok_pos,
                           int32_t n_tok, void* stream) {
  const int st = check_dsa_shape(shape);
  if (st != MSA_OK) return st;
  const msa_shape m = dsa_as_msa(shape);
  return append_idx_f16(&m, k_idx_cache, k_idx_new, tok_stream, tok_pos, n_tok, stream, pages);
}

int msa_dsa_token_scores(const msa_dsa_shape* shape, const msa_pages* pages, const msa_f16* q_idx,
                         const float* weights, const msa_f16* k_idx_cache, const int32_t* q_stream,
                         const int32_t* q_pos, int32_t n_q, float* scores, void* stream) {
  int st = check_dsa_shape(shape);
  if (st != MSA_OK) return st;
  if (n_q < 0) return MSA_ERR_RANGE;
  if (n_q == 0) return MSA_OK;
  if (!q_idx || !weights || !k_idx_cache || !q_stream || !q_pos || !scores) return MSA_ERR_NULL;
  if (!aligned16(q_idx) || !aligned16(weights) || !aligned16(k_idx_cache) || !aligned16(scores))
    return MSA_ERR_ALIGN;
  if (static_cast<int64_t>(n_q) * msa::dsa::kHeads >= (int64_t{1} << 31)) return MSA_ERR_RANGE;
  const msa_shape m = dsa_as_msa(shape);
  msa::KvPages pg;
  int64_t rows = 0;
  if ((st = pages_of(&m, pages, &pg, &rows)) != MSA_OK) return st;
  CUtensorMap tm_key, tm_q;
  if ((st = make_map_16bit(&tm_key, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, k_idx_cache, rows)) != MSA_OK) return st;
  if ((st = make_map_16bit(&tm_q, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, q_idx,
                           static_cast<int64_t>(n_q) * msa::dsa::kHeads, msa::dsa::kHeads)) != MSA_OK)
    return st;
  int sms = 0;
  if ((st = current_device_sms(&sms)) != MSA_OK) return st;
  static std::atomic<uint64_t> smem_done{0};
  if ((st = ensure_smem(msa::dsa::dsa_scores_kernel, msa::dsa::Smem::kBytes, smem_done)) != MSA_OK) return st;
  msa::dsa::Params P;
  P.weights = weights;
  P.q_stream = q_stream;
  P.q_pos = q_pos;
  P.scores = scores;
  P.n_q = n_q;
  P.n_streams = shape->n_streams;
  P.capacity = shape->capacity;
  P.n_tiles = shape->capacity / msa::dsa::kTile;
  P.relu = shape->relu != 0;
  P.pages = pg;
  const int64_t tasks = static_cast<int64_t>(n_q) * P.n_tiles;
  const int64_t grid = std::min<int64_t>(static_cast<int64_t>(msa::dsa::kCtasPerSm) * sms, tasks);
  launch(msa::dsa::dsa_scores_kernel, dim3(static_cast<unsigned>(grid)), dim3(msa::dsa::kThreads), msa::dsa::Smem::kBytes, static_cast<cudaStream_t>(stream), tm_key, tm_q, P);
  return cuda_status(cudaGetLastError());
}

int msa_dsa_select_topk(const msa_dsa_shape* shape, const float* scores, const int32_t* q_pos, int32_t n_q,
                        int32_t* sel, int32_t* n_sel, void* stream) {
  int st = check_dsa_shape(shape);
  if (st != MSA_OK) return st;
  if (n_q < 0) return MSA_ERR_RANGE;
  if (n_q == 0) return MSA_OK;
  if (!scores || !q_pos || !sel) return MSA_ERR_NULL;
  if (!aligned16(scores) || !aligned16(sel)) return MSA_ERR_ALIGN;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  int sms = 0;
  if ((st = current_device_sms(&sms)) != MSA_OK) return st;
  // fewer queries than SMs: a cluster of four CTAs per query, each staging a
  // quarter of the row, so a small batch of long rows uses four times the SMs
  if (n_q < sms && shape->capacity <= msa::dsa::kClusterKeys &&
      static_cast<int64_t>(n_q) * msa::dsa::kClusterCtas < (int64_t{1} << 31)) {
    const auto ck = msa::dsa::dsa_select_topk_cluster_kernel;
    static std::atomic<uint64_t> csmem_done{0};
    static std::atomic<int> cluster_ok{-1};           // can a cluster of this size be scheduled
    if ((st = ensure_smem(ck, msa::dsa::kClusterSmemBytes, csmem_done)) != MSA_OK) return st;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(n_q * msa::dsa::kClusterCtas));
    cfg.blockDim = dim3(msa::dsa::kSelThreads);
    cfg.dynamicSmemBytes = msa::dsa::kClusterSmemBytes;
    cfg.stream = cs;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = msa::dsa::kClusterCtas;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    if (cluster_ok.load() < 0) {
      int clusters = 0;
      cluster_ok.store(cudaOccupancyMaxActiveClusters(&clusters, ck, &cfg) == cudaSuccess && clusters > 0 ? 1 : 0);
      (void)cudaGetLastError();
    }
    if (cluster_ok.load() == 1) {
      if (cudaLaunchKernelEx(&cfg, ck, scores, q_pos, n_q, shape->capacity, shape->top_k, sel, n_sel) !=
          cudaSuccess)
        return MSA_ERR_CUDA;
      return cuda_status(cudaGetLastError());
    }
  }
  if (shape->capacity <= msa::dsa::kSmemKeys) {
    static std::atomic<uint64_t> smem_done{0};
    if ((st = ensure_smem(msa::dsa::dsa_select_topk_kernel<true>, msa::dsa::kSelSmemStaged, smem_done)) != MSA_OK)
      return st;
    launch(msa::dsa::dsa_select_topk_kernel<true>, dim3(static_cast<unsigned>(n_q)), dim3(msa::dsa::kSelThreads), msa::dsa::kSelSmemStaged, cs, scores, q_pos, n_q, shape->capacity,
                                                                             shape->top_k, sel, n_sel);
  } else {
    launch(msa::dsa::dsa_select_topk_kernel<false>, dim3(static_cast<unsigned>(n_q)), dim3(msa::dsa::kSelThreads), msa::dsa::kSelSmemUnstaged, cs, scores, q_pos, n_q,
                                                                                shape->capacity, shape->top_k,
                                                                                sel, n_sel);
  }
  return cuda_status(cudaGetLastError());
}

int msa_dsa_sparse_attn_decode(const msa_shape* shape, const msa_pages* pages, const msa_bf16* q,
                               const msa_bf16* k_cache, const msa_bf16* v_cache, const int32_t* sel,
                               const int32_t* q_stream, const int32_t* q_pos, int32_t n_q, float softmax_scale,
                               msa_bf16* out, void* workspace, size_t workspace_bytes, void* stream) {
  if (n_q > 0 && sel == nullptr) return MSA_ERR_NULL;
  return sparse_attn(shape, q, k_cache, v_cache, sel, q_stream, q_pos, n_q, softmax_scale, out, workspace,
                     workspace_bytes, stream, MSA_MODE_DECODE, pages, sel);
}

// ---- the whole decode step in one kernel ---------------------------------------
size_t msa_decode_step_fused_workspace_bytes(const msa_shape* shape, int32_t n_q) {
  if (check_shape(shape) != MSA_OK || n_q < 1 || scores_use_tiles(shape, n_q)) return static_cast<size_t>(-1);
  return msa::tc::align256(attn_workspace(shape, n_q, MSA_MODE_DECODE)) + 256;   // partials, then barrier words
}

int msa_decode_step_fused(const msa_shape* shape, float* idx_k_cache, msa_bf16* k_cache, msa_bf16* v_cache,
                          const float* idx_k_new, const msa_bf16* k_new, const msa_bf16* v_new,
                          const int32_t* tok_stream, const int32_t* tok_pos, int32_t n_tok, const float* idx_q,
                          const msa_bf16* q, const int32_t* q_stream, const int32_t* q_pos, int32_t n_q,
                          float softmax_scale, float* block_scores, int32_t* sel, int32_t* n_sel, msa_bf16* out,
                          void* workspace, size_t workspace_bytes, void* stream) {
  int st = check_shape(shape);
  if (st != MSA_OK) return st;
  if (n_tok < 0 || n_q < 0) return MSA_ERR_RANGE;
  if (n_q == 0 && n_tok == 0) return MSA_OK;
  if (n_q == 0) {                                            // nothing to score: the appends alone
    if ((st = msa_indexer_append(shape, idx_k_cache, idx_k_new, tok_stream, tok_pos, n_tok, stream)) != MSA_OK)
      return st;
    return msa_kv_append(shape, k_cache, v_cache, k_new, v_new, tok_stream, tok_pos, n_tok, stream);
  }
  if (!idx_k_cache || !k_cache || !v_cache || !idx_q || !q || !q_stream || !q_pos || !block_scores || !sel || !out)
    return MSA_ERR_NULL;
  if (n_tok > 0 && (!idx_k_new || !k_new || !v_new || !tok_stream || !tok_pos)) return MSA_ERR_NULL;
  if (!aligned16(idx_k_cache) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(idx_q) || !aligned16(q) ||
      !aligned16(block_scores) || !aligned16(sel) || !aligned16(out) || (n_tok > 0 && (!aligned16(idx_k_new) ||
      !aligned16(k_new) || !aligned16(v_new))))
    return MSA_ERR_ALIGN;
  if (!std::isfinite(softmax_scale)) return MSA_ERR_RANGE;
  if (scores_use_tiles(shape, n_q)) return MSA_ERR_SHAPE;       // prefill-shaped: use the separate calls
  const int G = shape->n_kv_heads;
  const int64_t n_pairs = static_cast<int64_t>(n_q) * G;
  if (static_cast<int64_t>(n_tok) * G >= (int64_t{1} << 31) || n_pairs * msa::dattn::kHpg >= (int64_t{1} << 31))
    return MSA_ERR_RANGE;
  const size_t need = msa_decode_step_fused_workspace_bytes(shape, n_q);
  if (workspace == nullptr || workspace_bytes < need) return MSA_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return MSA_ERR_ALIGN;
  int sms = 0;
  if ((st = current_device_sms(&sms)) != MSA_OK) return st;
  const auto kernel = msa::fused::decode_step_fused_kernel;
  static std::atomic<uint64_t> smem_done{0};
  if ((st = ensure_smem(kernel, msa::fused::kSmemBytes, smem_done)) != MSA_OK) return st;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, msa::fused::kThreads, msa::fused::kSmemBytes) !=
          cudaSuccess || per_sm < 1)
    return MSA_ERR_CUDA;
  const int grid = sms;                                      // one resident CTA per SM, as the separate kernels use
  const int64_t rows = static_cast<int64_t>(shape->n_streams) * G * shape->capacity;
  CUtensorMap tm_k, tm_v, tm_q;
  if ((st = make_kv_map(&tm_k, k_cache, rows)) != MSA_OK) return st;
  if ((st = make_kv_map(&tm_v, v_cache, rows)) != MSA_OK) return st;
  if ((st = make_map_16bit(&tm_q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, q, n_pairs * msa::dattn::kHpg,
                           msa::dattn::kHpg)) != MSA_OK)
    return st;

  msa::fused::Params F;
  F.idx_k_cache = idx_k_cache;
  F.idx_k_new = idx_k_new;
  F.k_cache = reinterpret_cast<uint8_t*>(k_cache);
  F.v_cache = reinterpret_cast<uint8_t*>(v_cache);
  F.k_new = reinterpret_cast<const uint8_t*>(k_new);
  F.v_new = reinterpret_cast<const uint8_t*>(v_new);
  F.tok_stream = tok_stream;
  F.tok_pos = tok_pos;
  F.n_tok = n_tok;
  msa::gemv::Params<float>& S = F.scores;
  S.idx_q = idx_q;
  S.idx_k = idx_k_cache;
  S.q_stream = q_stream;
  S.q_pos = q_pos;
  S.bs = block_scores;
  S.n_q = n_q;
  S.G = G;
  S.n_streams = shape->n_streams;
  S.capacity = shape->capacity;
  S.nblk = shape->capacity / 128;
  S.n_tasks = static_cast<long long>(n_q) * G * S.nblk;
  S.q_list = nullptr;
  S.q_count = nullptr;
  S.pages = msa::KvPages{nullptr, 0};
  F.sel = sel;
  F.n_sel = n_sel;
  msa::dattn::Params& A = F.attn;
  A.q = reinterpret_cast<const __nv_bfloat16*>(q);
  A.sel = sel;
  A.q_stream = q_stream;
  A.q_pos = q_pos;
  A.out = reinterpret_cast<__nv_bfloat16*>(out);
  A.sync = static_cast<msa::dattn::SyncSlot*>(workspace);
  A.ws = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + msa::dattn::kSyncBytes);
  A.n_q = n_q;
  A.G = G;
  A.n_streams = shape->n_streams;
  A.capacity = shape->capacity;
  A.n_units = n_pairs * msa::dattn::kTopK;
  A.n_cta = decode_attn_ctas(n_pairs, grid);                 // the separate calls' split
  A.scale_log2 = softmax_scale * 1.4426950408889634f;
  A.pages = msa::KvPages{nullptr, 0};
  A.tok_sel = nullptr;
  A.k_cache = reinterpret_cast<const __nv_bfloat16*>(k_cache);
  A.v_cache = reinterpret_cast<const __nv_bfloat16*>(v_cache);
  // the top-16 inside the attention phase when every CTA's share touches at
  // most kSelPairs pairs (no barrier between ranking and attention)
  const bool fuse_sel = max_pairs_per_cta(A.n_units, A.n_cta) <= msa::dattn::kSelPairs;
  A.bs = fuse_sel ? block_scores : nullptr;
  A.nblk = S.nblk;
  A.sel_out = fuse_sel ? sel : nullptr;
  A.n_sel_out = fuse_sel ? n_sel : nullptr;
  unsigned int* bar = reinterpret_cast<unsigned int*>(
      static_cast<uint8_t*>(workspace) + msa::tc::align256(attn_workspace(shape, n_q, MSA_MODE_DECODE)));
  F.bar_count = bar;
  F.bar_gen = bar + 1;
  F.wait_cycles = msa::kWaitCycles;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(bar, 0, 2 * sizeof(unsigned int), cs) != cudaSuccess) return MSA_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(msa::fused::kThreads);
  cfg.dynamicSmemBytes = msa::fused::kSmemBytes;
  cfg.stream = cs;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kernel, tm_k, tm_v, tm_q, F) != cudaSuccess) return MSA_ERR_CUDA;
  return cuda_status(cudaGetLastError());
}

int msa_wait_selftest(long long wait_cycles, void* workspace, size_t workspace_bytes, void* stream) {
  if (wait_cycles < 1 || wait_cycles > msa::kWaitCycles) return MSA_ERR_RANGE;
  if (workspace == nullptr) return MSA_ERR_NULL;
  if (workspace_bytes < MSA_WAIT_SELFTEST_WORKSPACE_BYTES) return MSA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return MSA_ERR_ALIGN;
  int sms = 0;
  int st = current_device_sms(&sms);
  if (st != MSA_OK) return st;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  unsigned int* bar = static_cast<unsigned int*>(workspace);
  if (cudaMemsetAsync(bar, 0, MSA_WAIT_SELFTEST_WORKSPACE_BYTES, cs) != cudaSuccess) return MSA_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(sms));
  cfg.blockDim = dim3(32);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = cs;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, msa::fused::wait_selftest_kernel, bar, wait_cycles) != cudaSuccess)
    return MSA_ERR_CUDA;
  return cuda_status(cudaGetLastError());
}

size_t msa_workspace_bytes(const msa_shape* shape, int32_t n_q, int32_t mode) {
  if (check_shape(shape) != MSA_OK || n_q < 0 || (mode != MSA_MODE_DECODE && mode != MSA_MODE_PREFILL))
    return static_cast<size_t>(-1);
  return std::max(scores_workspace(shape, n_q), attn_workspace(shape, n_q, mode));
}

const char* msa_status_string(int status) {
  switch (status) {
    case MSA_OK: return "MSA_OK";
    case MSA_ERR_NULL: return "MSA_ERR_NULL: a required pointer is NULL";
    case MSA_ERR_ALIGN: return "MSA_ERR_ALIGN: a pointer is not 16-byte aligned";
    case MSA_ERR_SHAPE: return "MSA_ERR_SHAPE: unsupported geometry";
    case MSA_ERR_RANGE: return "MSA_ERR_RANGE: count or value out of range";
    case MSA_ERR_WORKSPACE: return "MSA_ERR_WORKSPACE: workspace missing or too small";
    case MSA_ERR_CUDA: return "MSA_ERR_CUDA: CUDA launch or query failed";
    default: return "unknown MSA status";
  }
}

int msa_get_device_error(uint32_t* flags, void* stream) {
  if (flags == nullptr) return MSA_ERR_NULL;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return MSA_ERR_CUDA;
  unsigned int v = 0;
  if (cudaMemcpyFromSymbol(&v, msa::g_dev_error, sizeof(v)) != cudaSuccess) return MSA_ERR_CUDA;
  const unsigned int zero = 0;
  if (cudaMemcpyToSymbol(msa::g_dev_error, &zero, sizeof(zero)) != cudaSuccess) return MSA_ERR_CUDA;
  *flags = v;
  return MSA_OK;
}

int msa_version(void) { return kVersion; }

}  // extern "C"
