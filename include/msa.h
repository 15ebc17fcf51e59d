/*
 * msa.h - C ABI of the MiniMax Sparse Attention (MSA) hot path for NVIDIA
 * B200 (sm_100a).
 *
 * The method (llama.cpp pull request "Add MiniMax-M3 (MSA: MiniMax Sparse
 * Attention) support", sections "Overview" and "Implementation"): for every
 * query, one indexer head per GQA group scores each causally visible key as
 * idx_q . idx_k, the scores are max-pooled over 128-slot key blocks, the
 * query's own (local) block gets a large positive bias so it is always kept,
 * and the top-16 blocks are selected.  Attention then runs over only those
 * 16 x 128 = 2048 K/V rows, shared by the group's 16 query heads.
 *
 * Conventions for every call
 *  - All tensor pointers are DEVICE pointers into caller-owned memory,
 *    contiguous in the layout stated, 16-byte aligned.  The library never
 *    allocates, frees or keeps a pointer after a call returns.
 *  - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *    default stream) and returns MSA_OK or a negative MSA_ERR_* code.  On an
 *    error nothing is launched and no output is written.
 *  - Conditions only the device can see (a position or stream id outside the
 *    cache, a selected block id that is not visible) set a bit in a per-device
 *    error word and skip the affected work; kernels never trap.  Read and
 *    clear the word with msa_get_device_error().
 *  - Block scores, selection and attention read rows j <= q_pos of the query's
 *    stream: append a token's indexer key and K/V row before scoring or
 *    attending a query at that position (the query sees its own token).
 *  - Supported geometry of the CUDA kernels: head_dim = idx_dim = block = 128,
 *    top_k = 16, n_q_heads = 16 * n_kv_heads, 1 <= n_kv_heads <= 16,
 *    capacity a positive multiple of 128 (the KV length is a multiple of 128,
 *    as the MSA branch asserts).  Other shapes return MSA_ERR_SHAPE.
 *
 * Layouts (S streams, G = n_kv_heads groups, cap = capacity, nblk = cap/128,
 * Hq = n_q_heads, D = head_dim, Di = idx_dim):
 *   idx_k_cache   [S][G][cap][Di]  float32   indexer-key cache
 *   k_cache       [S][G][cap][D]   bfloat16  K cache (non-transposed)
 *   v_cache       [S][G][cap][D]   bfloat16  V cache (non-transposed)
 *   idx_q         [n_q][G][Di]     float32   one indexer query per group
 *   q             [n_q][Hq][D]     bfloat16  head h belongs to group h / 16
 *   q_stream, q_pos [n_q]          int32     stream and absolute slot
 *   block_scores  [n_q][G][nblk]   float32
 *   sel           [n_q][G][top_k]  int32     ascending block ids, -1 padded
 *   n_sel         [n_q][G]         int32
 *   out           [n_q][Hq][D]     bfloat16
 */
#ifndef MSA_H
#define MSA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MSA_API __attribute__((visibility("default")))
#else
#define MSA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ------------------------------------------------------ */
#define MSA_OK             0
#define MSA_ERR_NULL      (-1)  /* a required pointer is NULL                  */
#define MSA_ERR_ALIGN     (-2)  /* a pointer is not 16-byte aligned            */
#define MSA_ERR_SHAPE     (-3)  /* geometry not supported (see above)          */
#define MSA_ERR_RANGE     (-4)  /* a count is negative or too large            */
#define MSA_ERR_WORKSPACE (-5)  /* workspace missing or smaller than required  */
#define MSA_ERR_CUDA      (-6)  /* a CUDA launch or query failed               */

/* ---- device error word bits (msa_get_device_error) -------------------- */
#define MSA_DEVERR_QUERY_RANGE 0x1u /* q_stream/q_pos outside [0,S) x [0,cap): query skipped */
#define MSA_DEVERR_TOKEN_RANGE 0x2u /* tok_stream/tok_pos outside the cache: token skipped   */
#define MSA_DEVERR_SEL_RANGE   0x4u /* sel id not a visible block: that block skipped       */
#define MSA_DEVERR_TIMEOUT     0x8u /* a bounded wait on a copy gave up: output incomplete  */
#define MSA_DEVERR_PAGE_RANGE  0x10u /* paged cache: a touched block has no valid page: skipped */

/* The local-force bias added to the score of each query's own block
 * ("a large positive bias on each query's local block", MSA pull request,
 * section "Implementation").  2^100 exceeds twice any finite score the
 * indexer can produce in practice, so the local block always ranks first;
 * in float32 the biased score is exactly 2^100. */
#define MSA_LOCAL_BIAS 0x1p100f

/* Bit pattern of an IEEE bfloat16 value. */
typedef uint16_t msa_bf16;

/* Bit pattern of an IEEE binary16 (fp16) value. */
typedef uint16_t msa_f16;

typedef struct msa_shape {
  int32_t n_streams;   /* S: independent sequences, one cache region each      */
  int32_t capacity;    /* slots per stream, a multiple of block                */
  int32_t n_q_heads;   /* Hq: 64 for the MiniMax-M3 attention layers           */
  int32_t n_kv_heads;  /* G: KV heads = GQA groups = indexer heads (4)         */
  int32_t head_dim;    /* D: 128                                               */
  int32_t idx_dim;     /* Di: indexer dimension, 128                           */
  int32_t block;       /* key block size of the max-pool, 128                  */
  int32_t top_k;       /* blocks kept per query and group, 16                  */
} msa_shape;

/* msa_indexer_append - write new tokens' indexer keys into the F32 cache.
 * The indexer keeps its own per-layer F32 key cache beside K/V, one region
 * per stream (MSA pull request, section "Implementation").
 *   idx_k_new [n_tok][G][Di] f32; token t goes to idx_k_cache[tok_stream[t]]
 *   [g][tok_pos[t]][:] for every group g.  Tokens with an out-of-range
 *   stream or slot are skipped and set MSA_DEVERR_TOKEN_RANGE.  Two tokens
 *   naming the same slot race.  n_tok == 0 is a no-op. */
MSA_API int msa_indexer_append(const msa_shape* shape, float* idx_k_cache, const float* idx_k_new,
                       const int32_t* tok_stream, const int32_t* tok_pos, int32_t n_tok,
                       void* stream);

/* msa_kv_append - write new tokens' K and V rows ([n_tok][G][D] bf16 each)
 * into the bf16 caches at (tok_stream[t], tok_pos[t]); same rules as
 * msa_indexer_append.  The main K/V cache keeps the non-transposed V layout
 * (MSA pull request, section "Requirements and fallbacks"). */
MSA_API int msa_kv_append(const msa_shape* shape, msa_bf16* k_cache, msa_bf16* v_cache,
                  const msa_bf16* k_new, const msa_bf16* v_new, const int32_t* tok_stream,
                  const int32_t* tok_pos, int32_t n_tok, void* stream);

/* msa_step_append - msa_indexer_append and msa_kv_append in one launch: each
 * new token's F32 indexer key and its K and V rows are written at the same
 * slots, with the same arguments, layouts, checks and error bits as the two
 * calls (the indexer keeps its own key cache beside K/V: MSA pull request,
 * "Implementation").  One kernel instead of two per step, which matters
 * when a step is launch-bound (a decode batch of a few streams).  All six
 * cache and row pointers are required and 16-byte aligned. */
MSA_API int msa_step_append(const msa_shape* shape, float* idx_k_cache, msa_bf16* k_cache, msa_bf16* v_cache,
                            const float* idx_k_new, const msa_bf16* k_new, const msa_bf16* v_new,
                            const int32_t* tok_stream, const int32_t* tok_pos, int32_t n_tok, void* stream);

/* msa_block_scores - fused indexer score, causal mask, max-pool and local
 * bias: block_scores[i][g][b] = max over slots j of block b with j <= q_pos[i]
 * of idx_q[i][g] . idx_k_cache[q_stream[i]][g][j], accumulated in float32
 * ("force F32 indexer score accum", MSA branch commit message); blocks with
 * no visible slot are -inf; the local block q_pos[i]/128 gets
 * + MSA_LOCAL_BIAS (MSA pull request, section "Implementation":
 * bs = maxpool_128(idx_q*idx_k^T + causal mask) plus the local-force bias).
 * NaN scores are treated as -inf.  An out-of-range query writes -inf
 * everywhere and sets MSA_DEVERR_QUERY_RANGE.
 *
 * Two kernels implement it.  Decode-shaped batches (fewer than 256 queries,
 * or fewer than 64 per stream on average) stream the F32 keys through a
 * GEMV; they need no workspace.  Prefill-shaped batches run tiles of 128
 * consecutive queries against 128-key blocks on the tcgen05 tensor cores:
 * each F32 row is split exactly as 2^-e (hi + lo) with fp16 hi, lo and three
 * MMAs (hi.hi + hi.lo + lo.hi) accumulate in F32, which keeps the score within
 * about 2^-21 of sum |q_d k_d|.  Tiles whose queries span several streams
 * fall back to the GEMV for the queries of the other streams.  The tile path
 * needs `workspace` of at least msa_workspace_bytes(shape, n_q, mode) bytes,
 * 256-byte aligned (its contents need not be initialised). */
MSA_API int msa_block_scores(const msa_shape* shape, const float* idx_q, const float* idx_k_cache,
                     const int32_t* q_stream, const int32_t* q_pos, int32_t n_q,
                     float* block_scores, void* workspace, size_t workspace_bytes,
                     void* stream);

/* F16 indexer-key cache variant.  The MSA pull request keeps the indexer
 * cache in F32 by default ("set default cache type to F32", MSA branch
 * commit message) and its review thread compares F16 against F32 indexer
 * precision (IF16 vs IF32 KL divergence); these two calls are the F16 cache
 * type: keys are stored as fp16, which halves the bytes a decode step
 * streams.  msa_indexer_append_f16 rounds each F32 key value to fp16
 * (nearest even) as it writes idx_k_cache [S][G][cap][Di] (fp16 bits);
 * msa_block_scores_f16 computes exactly what msa_block_scores computes on the
 * fp16 keys (each converted exactly to F32, F32 accumulation, same pooling,
 * bias, layouts, workspace and errors).  Selection and attention calls are
 * unchanged. */
MSA_API int msa_indexer_append_f16(const msa_shape* shape, msa_f16* idx_k_cache, const float* idx_k_new,
                                   const int32_t* tok_stream, const int32_t* tok_pos, int32_t n_tok,
                                   void* stream);
MSA_API int msa_block_scores_f16(const msa_shape* shape, const float* idx_q, const msa_f16* idx_k_cache,
                                 const int32_t* q_stream, const int32_t* q_pos, int32_t n_q,
                                 float* block_scores, void* workspace, size_t workspace_bytes,
                                 void* stream);

/* msa_select_topk - top-k block selection per (query, group).
 * Ranks the visible blocks b <= q_pos/128 by (score descending, block index
 * ascending) and keeps the first min(top_k, q_pos/128 + 1): with fewer
 * visible blocks than top_k every visible block is taken (MSA pull request,
 * RADV review comment: k = min(indexer_top_k, n_blocks)).  Ids are written
 * ascending into sel, padded with -1; n_sel (may be NULL) gets the count.
 * Equal scores go to the lower block index; NaN ranks as -inf.  A q_pos
 * outside [0, capacity) writes an empty selection and sets
 * MSA_DEVERR_QUERY_RANGE. */
MSA_API int msa_select_topk(const msa_shape* shape, const float* block_scores, const int32_t* q_pos,
                    int32_t n_q, int32_t* sel, int32_t* n_sel, void* stream);

/* msa_sparse_attn_decode - block-sparse GQA attention for a few queries
 * (decode: one new token per stream).  For query i and head h (group
 * g = h/16): out[i][h] = softmax(softmax_scale * q[i][h] . K_j) . V_j over
 * rows j of the blocks in sel[i][g] with j <= q_pos[i] (MSA pull request,
 * section "Overview": attention runs only over the selected blocks; the
 * token-level causal mask applies inside the local block).  Softmax and
 * accumulation in float32, output rounded to bf16 (nearest even).  A query
 * with no attended row writes zeros.  A persistent grid of at most one CTA
 * per SM splits the (pair, selected block) units into equal contiguous
 * shares, in one launch (when the pairs fit, k CTAs per pair, so that the
 * shares line up with the pairs); a pair cut between CTAs is merged by the
 * CTA holding its first unit from the partial results the later CTAs
 * publish.  `workspace` (at least
 * msa_workspace_bytes(shape, n_q, MSA_MODE_DECODE) bytes, 16-byte aligned)
 * holds, in its first 4096 bytes, the merge bookkeeping of 256 CTA slots
 * (per slot: a 64-bit publication flag and a 32-bit epoch that the merging
 * CTA raises), then one partial result per CTA (16 x 130 floats).  The
 * bookkeeping carries over from call to call and needs no initial value: a
 * merger waits for a flag equal to a tag, its own index and its epoch + 1,
 * which no earlier call (and, short of that exact 64-bit pattern, no other
 * contents of a reused buffer) leaves behind.  Calls that may run at the
 * same time on the GPU need separate workspaces.  A merge whose partial
 * never appears gives up after the library's bounded wait and sets
 * MSA_DEVERR_TIMEOUT. */
MSA_API int msa_sparse_attn_decode(const msa_shape* shape, const msa_bf16* q, const msa_bf16* k_cache,
                           const msa_bf16* v_cache, const int32_t* sel, const int32_t* q_stream,
                           const int32_t* q_pos, int32_t n_q, float softmax_scale, msa_bf16* out,
                           void* workspace, size_t workspace_bytes, void* stream);

/* msa_select_attn_decode - msa_select_topk followed by
 * msa_sparse_attn_decode in one call, bit-identical to the two: block_scores
 * [n_q][G][capacity/128] f32 in, the selection written to sel [n_q][G][16]
 * and n_sel [n_q][G] (n_sel may be NULL), the attention to out.  MSA pull
 * request, "Implementation": the block scores are ranked for the top-k and
 * attention runs over the kept blocks.  Each CTA of the persistent attention
 * grid ranks the pairs its units touch before it starts loading K/V, so a
 * decode step has one launch fewer; when a CTA's share would touch more
 * than 8 pairs (more than about 900 (query, group) pairs on 148 SMs) the
 * call runs the selection kernel first instead, with the same results.
 * Same arguments, layouts, workspace (msa_workspace_bytes(shape, n_q,
 * MSA_MODE_DECODE)) and device errors as the two calls. */
MSA_API int msa_select_attn_decode(const msa_shape* shape, const float* block_scores, const msa_bf16* q,
                                   const msa_bf16* k_cache, const msa_bf16* v_cache, const int32_t* q_stream,
                                   const int32_t* q_pos, int32_t n_q, float softmax_scale, int32_t* sel,
                                   int32_t* n_sel, msa_bf16* out, void* workspace, size_t workspace_bytes,
                                   void* stream);

/* msa_sparse_attn_prefill - the same computation as msa_sparse_attn_decode,
 * for batches of many queries (prefill: every appended token is a query).
 * MSA pull request, "Implementation", batch case: the query's block-level
 * selection combined with the token-level causal mask.  Workspace:
 * msa_workspace_bytes(shape, n_q, MSA_MODE_PREFILL) bytes, 16-byte aligned:
 * it holds the plan of every tile of 8 queries (the union of their selected
 * blocks), written by a first kernel and read by the attention kernel. */
MSA_API int msa_sparse_attn_prefill(const msa_shape* shape, const msa_bf16* q, const msa_bf16* k_cache,
                            const msa_bf16* v_cache, const int32_t* sel, const int32_t* q_stream,
                            const int32_t* q_pos, int32_t n_q, float softmax_scale, msa_bf16* out,
                            void* workspace, size_t workspace_bytes, void* stream);

#define MSA_MODE_DECODE  0
#define MSA_MODE_PREFILL 1

/* Size of the fixed device buffer used by msa_sparse_attn_decode_noalloc. */
#define MSA_NOALLOC_SCRATCH_BYTES (8u * 1024u * 1024u)

/* msa_sparse_attn_decode_noalloc - msa_sparse_attn_decode without a
 * caller-provided workspace.  The pages describe no such call; it exists for
 * callers that cannot allocate device memory when they run attention, for
 * example a runtime whose device memory is all handed out by a pool sized at
 * start-up, or a program driving the C ABI from a language that has no CUDA
 * allocator of its own.  Such a caller still owns q, the caches, sel and out.
 *
 * The workspace (merge bookkeeping and partial results) is one file-scope
 * device buffer of MSA_NOALLOC_SCRATCH_BYTES that every GPU loading this
 * library holds until the process exits.  A call whose
 * msa_workspace_bytes(shape, n_q, MSA_MODE_DECODE) exceeded that size would
 * be rejected with MSA_ERR_WORKSPACE; decode needs at most 4096 + 256 CTAs x
 * 8320 bytes = 2,134,016 bytes, so every batch fits.  The first call on each
 * device looks up the buffer's device address (with that device current);
 * make that first call before any stream capture.  The address is looked up
 * again when the device's current context is not the one it was found in
 * (after cudaDeviceReset, or when the primary context was released and
 * created anew), since each context holds its own copy of the buffer; that
 * first call in a new context, too, belongs before any capture.  All calls share the
 * buffer: calls that can run at the same time on the GPU (different streams,
 * or different host threads on one device) race and must be serialised by
 * the caller.  Nothing in the buffer needs to start at zero: every call
 * writes each partial it reads, and the bookkeeping needs no initial value.
 * Allocates nothing, on the host or the device. */
MSA_API int msa_sparse_attn_decode_noalloc(const msa_shape* shape, const msa_bf16* q,
                                           const msa_bf16* k_cache, const msa_bf16* v_cache,
                                           const int32_t* sel, const int32_t* q_stream,
                                           const int32_t* q_pos, int32_t n_q, float softmax_scale,
                                           msa_bf16* out, void* stream);

/* ---- paged caches --------------------------------------------------------
 * The calls above address a cache as one region per stream, so logical slot
 * j of stream s is physical slot j of region s.  The MSA pull request's
 * issue thread on unified KV caches finds that block scoring and gathering
 * by absolute slot breaks once streams share one buffer, and that a fix
 * needs a sequence-relative page indirection consulted by the scoring and
 * gather steps (what the reference MSA kernel's page index provides).  These
 * calls are that indirection.
 *
 * A page holds the 128 slots of one key block for every group.  Pools:
 *   idx_k_pool [n_pages][G][128][Di] f32 (or fp16 for the _f16 calls),
 *   k_pool, v_pool [n_pages][G][128][D] bf16.
 * block_table [n_streams][capacity / 128] int32 (device memory, 4-byte
 * aligned) names the page that holds logical block b of stream s; capacity
 * is the logical length of a stream.  Several streams may name the same
 * page (a shared prefix) for reading; writing a shared page is the caller's
 * race.  Each paged call computes exactly what its contiguous counterpart
 * computes on the logical cache cache[s][g][j] = pool[block_table[s][j/128]]
 * [g][j % 128]: same arguments otherwise, same layouts of every other array,
 * same workspace (msa_workspace_bytes).  Only blocks a call touches are
 * looked up (a token's block for the appends, blocks b <= q_pos/128 for
 * scores, selected blocks for attention).  A touched block whose entry is
 * negative or >= n_pages is skipped and sets MSA_DEVERR_PAGE_RANGE: the
 * token is not written, the block scores -inf, attention leaves the block
 * out.  Host-side errors: pages or block_table NULL (MSA_ERR_NULL),
 * n_pages < 1 (MSA_ERR_RANGE), n_pages * G * 128 >= 2^31 (MSA_ERR_SHAPE). */
typedef struct msa_pages {
  const int32_t* block_table;  /* [n_streams][capacity / block], page ids      */
  int32_t n_pages;             /* pages in each pool                           */
} msa_pages;

MSA_API int msa_indexer_append_paged(const msa_shape* shape, const msa_pages* pages, float* idx_k_pool,
                                     const float* idx_k_new, const int32_t* tok_stream, const int32_t* tok_pos,
                                     int32_t n_tok, void* stream);
MSA_API int msa_indexer_append_f16_paged(const msa_shape* shape, const msa_pages* pages, msa_f16* idx_k_pool,
                                         const float* idx_k_new, const int32_t* tok_stream,
                                         const int32_t* tok_pos, int32_t n_tok, void* stream);
MSA_API int msa_kv_append_paged(const msa_shape* shape, const msa_pages* pages, msa_bf16* k_pool,
                                msa_bf16* v_pool, const msa_bf16* k_new, const msa_bf16* v_new,
                                const int32_t* tok_stream, const int32_t* tok_pos, int32_t n_tok, void* stream);
MSA_API int msa_step_append_paged(const msa_shape* shape, const msa_pages* pages, float* idx_k_pool,
                                  msa_bf16* k_pool, msa_bf16* v_pool, const float* idx_k_new,
                                  const msa_bf16* k_new, const msa_bf16* v_new, const int32_t* tok_stream,
                                  const int32_t* tok_pos, int32_t n_tok, void* stream);
MSA_API int msa_block_scores_paged(const msa_shape* shape, const msa_pages* pages, const float* idx_q,
                                   const float* idx_k_pool, const int32_t* q_stream, const int32_t* q_pos,
                                   int32_t n_q, float* block_scores, void* workspace, size_t workspace_bytes,
                                   void* stream);
MSA_API int msa_block_scores_f16_paged(const msa_shape* shape, const msa_pages* pages, const float* idx_q,
                                       const msa_f16* idx_k_pool, const int32_t* q_stream, const int32_t* q_pos,
                                       int32_t n_q, float* block_scores, void* workspace,
                                       size_t workspace_bytes, void* stream);
MSA_API int msa_sparse_attn_decode_paged(const msa_shape* shape, const msa_pages* pages, const msa_bf16* q,
                                         const msa_bf16* k_pool, const msa_bf16* v_pool, const int32_t* sel,
                                         const int32_t* q_stream, const int32_t* q_pos, int32_t n_q,
                                         float softmax_scale, msa_bf16* out, void* workspace,
                                         size_t workspace_bytes, void* stream);
MSA_API int msa_select_attn_decode_paged(const msa_shape* shape, const msa_pages* pages,
                                         const float* block_scores, const msa_bf16* q, const msa_bf16* k_pool,
                                         const msa_bf16* v_pool, const int32_t* q_stream, const int32_t* q_pos,
                                         int32_t n_q, float softmax_scale, int32_t* sel, int32_t* n_sel,
                                         msa_bf16* out, void* workspace, size_t workspace_bytes, void* stream);
MSA_API int msa_sparse_attn_prefill_paged(const msa_shape* shape, const msa_pages* pages, const msa_bf16* q,
                                          const msa_bf16* k_pool, const msa_bf16* v_pool, const int32_t* sel,
                                          const int32_t* q_stream, const int32_t* q_pos, int32_t n_q,
                                          float softmax_scale, msa_bf16* out, void* workspace,
                                          size_t workspace_bytes, void* stream);

/* ---- token-level variant: the lightning indexer ---------------------------
 * "deepseek2 : GLM-DSA sparse attention (lightning indexer)" (ik_llama.cpp
 * pull request), section "What this does": instead of max-pooled blocks, the
 * indexer scores every visible token and the top-k tokens of each query are
 * kept (GLM-5.2 keeps 2048); attention then runs over those tokens only.  The
 * indexer-key cache holds one F16 key per token ([head_size, kv_size]); a
 * query has H_I indexer heads whose products with a key are weighted per head
 * and summed (the review thread's element-wise product with a weight matrix
 * followed by the reduction over indexer heads).  The caller applies the
 * Hadamard rotation of queries and keys before these calls.
 *
 *   I[t][s] = sum_h weights[t][h] * act(q_idx[t][h] . k_idx[stream(t)][s])
 *
 * for s <= q_pos[t] (-inf beyond), act = ReLU when shape->relu is nonzero
 * (the published lightning-indexer definition; the page does not print the
 * formula), identity otherwise.  Supported: index_dim 128, n_index_heads
 * 64, 1 <= top_k <= 2048, capacity % 128 == 0, n_streams * capacity < 2^31.
 * Every call takes an optional page table (NULL: contiguous caches); a page
 * of the key pool [n_pages][128][Di] holds 128 consecutive tokens of one
 * stream, as for the MSA caches with one group. */
typedef struct msa_dsa_shape {
  int32_t n_streams;
  int32_t capacity;       /* tokens per stream (logical length when paged)     */
  int32_t n_index_heads;  /* H_I: 64                                           */
  int32_t index_dim;      /* 128                                               */
  int32_t top_k;          /* tokens kept per query, 1..2048                    */
  int32_t relu;           /* nonzero: ReLU on each head's product              */
} msa_dsa_shape;

#define MSA_DSA_SEL_WIDTH 2048   /* entries of one selection row */

/* Append: k_idx_new [n_tok][Di] f32, rounded to fp16 (nearest even) and
 * written at (tok_stream[t], tok_pos[t]) of k_idx_cache [S][cap][Di] fp16
 * (or of its page).  Same rules as msa_indexer_append. */
MSA_API int msa_dsa_indexer_append(const msa_dsa_shape* shape, const msa_pages* pages, msa_f16* k_idx_cache,
                                   const float* k_idx_new, const int32_t* tok_stream, const int32_t* tok_pos,
                                   int32_t n_tok, void* stream);

/* Token scores: q_idx [n_q][H_I][Di] fp16, weights [n_q][H_I] f32 ->
 * scores [n_q][capacity] f32, -inf past each query's position.  Each head's
 * product of fp16 vectors accumulates in f32 on the tensor cores; the
 * weighted sum over heads runs in f32 in a fixed order (deterministic).  An out-of-range query
 * writes -inf everywhere and sets MSA_DEVERR_QUERY_RANGE. */
MSA_API int msa_dsa_token_scores(const msa_dsa_shape* shape, const msa_pages* pages, const msa_f16* q_idx,
                                 const float* weights, const msa_f16* k_idx_cache, const int32_t* q_stream,
                                 const int32_t* q_pos, int32_t n_q, float* scores, void* stream);

/* Top-k tokens: sel [n_q][MSA_DSA_SEL_WIDTH] int32, ascending token ids,
 * -1 padded; n_sel [n_q] (may be NULL) gets min(top_k, q_pos + 1).  Every
 * visible token is kept when there are at most top_k; otherwise the top_k
 * largest scores, equal scores keeping the lower index (NaN ranks as -inf,
 * -0 equals +0). */
MSA_API int msa_dsa_select_topk(const msa_dsa_shape* shape, const float* scores, const int32_t* q_pos,
                                int32_t n_q, int32_t* sel, int32_t* n_sel, void* stream);

/* Attention over the kept tokens: for query i and head h (group h/16),
 * softmax(softmax_scale * q . K_j) . V_j over the tokens j of sel[i] (the
 * same tokens for every group), rows of the MSA K/V caches of `shape`
 * (contiguous, or pools addressed through `pages`).  Same layouts, workspace
 * (msa_workspace_bytes(shape, n_q, MSA_MODE_DECODE)), rounding and errors
 * as msa_sparse_attn_decode; a kept token past the query sets
 * MSA_DEVERR_SEL_RANGE, one in an unmapped page MSA_DEVERR_PAGE_RANGE, and
 * is left out. */
MSA_API int msa_dsa_sparse_attn_decode(const msa_shape* shape, const msa_pages* pages, const msa_bf16* q,
                                       const msa_bf16* k_cache, const msa_bf16* v_cache, const int32_t* sel,
                                       const int32_t* q_stream, const int32_t* q_pos, int32_t n_q,
                                       float softmax_scale, msa_bf16* out, void* workspace,
                                       size_t workspace_bytes, void* stream);

/* msa_decode_step_fused - one whole decode step in a single persistent
 * kernel: append the new tokens (msa_indexer_append + msa_kv_append), block
 * scores (msa_block_scores), top-16 (msa_select_topk) and block-sparse
 * attention (msa_sparse_attn_decode), with the same arguments, layouts,
 * rounding and errors as those calls and bit-identical results.  The MSA
 * pull request runs the step as separate graph nodes per layer; here the
 * phases are separated by grid-wide barriers of one cooperative launch (one
 * CTA per SM), so a small decode batch pays one launch instead of six.  F32
 * indexer cache, contiguous caches and decode-shaped batches only (fewer
 * than 256 queries, or fewer than 64 per stream on average; otherwise
 * MSA_ERR_SHAPE).  n_sel may be NULL.  workspace: at least
 * msa_decode_step_fused_workspace_bytes(shape, n_q) bytes, 256-byte aligned
 * (the attention's merge bookkeeping and partials, and the barrier words, which the call
 * zeroes on `stream` before the launch).  A barrier wait that gives up sets
 * MSA_DEVERR_TIMEOUT and leaves the outputs incomplete.  n_q == 0 only
 * appends. */
MSA_API int msa_decode_step_fused(const msa_shape* shape, float* idx_k_cache, msa_bf16* k_cache, msa_bf16* v_cache,
                                  const float* idx_k_new, const msa_bf16* k_new, const msa_bf16* v_new,
                                  const int32_t* tok_stream, const int32_t* tok_pos, int32_t n_tok,
                                  const float* idx_q, const msa_bf16* q, const int32_t* q_stream,
                                  const int32_t* q_pos, int32_t n_q, float softmax_scale, float* block_scores,
                                  int32_t* sel, int32_t* n_sel, msa_bf16* out, void* workspace,
                                  size_t workspace_bytes, void* stream);
/* Workspace bytes of msa_decode_step_fused, or (size_t)-1 for an
 * unsupported shape or batch. */
MSA_API size_t msa_decode_step_fused_workspace_bytes(const msa_shape* shape, int32_t n_q);

/* Bytes of device workspace msa_wait_selftest needs. */
#define MSA_WAIT_SELFTEST_WORKSPACE_BYTES 16u

/* msa_wait_selftest - drives the library's bounded device waits to their
 * limit, so that a caller (or a test) can see that a wait which never ends
 * gives up, records MSA_DEVERR_TIMEOUT and lets its kernel return with the
 * context still usable.  The pages have no counterpart: it checks the
 * library's own failure handling (no kernel here traps or spins without a
 * limit).  One cooperative launch with one CTA per SM: every CTA meets at
 * the grid barrier of msa_decode_step_fused set to expect one more arrival
 * than the grid gives, then one thread per CTA waits on an mbarrier that
 * nothing arrives on.  Each wait gives up after wait_cycles SM clock cycles
 * (1 ..= 1e9; the library's own kernels use 1e9, about half a second).
 * workspace: MSA_WAIT_SELFTEST_WORKSPACE_BYTES of device memory, 16-byte
 * aligned, zeroed by the call on `stream`; afterwards its third 32-bit word
 * is 0 when every wait ran out as it should.  Asynchronous on `stream`;
 * read the result with msa_get_device_error.  MSA_ERR_RANGE for a limit out
 * of range. */
MSA_API int msa_wait_selftest(long long wait_cycles, void* workspace, size_t workspace_bytes, void* stream);

/* Bytes of workspace that msa_block_scores and the attention call of `mode`
 * need for n_q queries (the larger of the two; one buffer serves both calls
 * of a step, since they run in stream order).  0 when neither needs any.
 * Returns (size_t)-1 for an unsupported shape. */
MSA_API size_t msa_workspace_bytes(const msa_shape* shape, int32_t n_q, int32_t mode);

/* Human-readable name of a status code (static string). */
MSA_API const char* msa_status_string(int status);

/* Wait for `stream`, then read and clear the calling thread's current
 * device's error word into *flags (MSA_DEVERR_* bits). */
MSA_API int msa_get_device_error(uint32_t* flags, void* stream);

/* Library version, major*10000 + minor*100 + patch. */
MSA_API int msa_version(void);

#ifdef __cplusplus
}
#endif
#endif /* MSA_H */
