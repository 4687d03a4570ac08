/*
 * qsa.h -- C ABI of a B200 (sm_100a) implementation of one Qwen Sparse
 * Attention layer with compression ratio 4 (QSA c4).
 *
 * The method is the one the SGLang day-0 blog for Qwen3.8-Flash-Next describes
 * in its sections "Qwen Sparse Attention: Retrieve Coarsely, Attend Precisely"
 * and "IndexShare MTP: Reusing the QSA Selection Across Draft Steps":
 *
 *   indexer  every 4 raw 128-d index keys -> one compressed key (FP32 mean,
 *            L2-normalised, RoPE-rotated at the block's first position, BF16);
 *            the raw keys of an unfinished block wait in a 4-slot ring;
 *            a query's 4 index heads score every complete block,
 *            score_b = sum_h w_h * max(0, q~_h . k^_b), and the best 512 blocks
 *            are kept (ties: lower block index first);
 *   expand   512 blocks -> 2048 token positions, plus the 0..3 tokens of the
 *            unfinished block: at most 2051 positions;
 *   attend   GQA (16 query heads, 2 KV heads, d = 128) over the raw, paged BF16
 *            K/V at exactly those positions.
 *
 * Conventions for every entry point
 *   - All tensor pointers are DEVICE pointers owned by the caller; the library
 *     allocates nothing, never synchronises the stream (except
 *     qsa_device_error, which says so) and only enqueues work on `stream`
 *     (a cudaStream_t; NULL = the legacy default stream).
 *   - bf16 tensors are passed as void* holding IEEE bfloat16 values.
 *   - Row-major layouts; shapes are given in brackets, innermost last.
 *   - Host-checkable errors (null pointers, bad sizes, a workspace that is too
 *     small, unsupported shapes) return an error status before anything is
 *     enqueued.  Data-dependent errors found on the device (a page id outside
 *     the pool, a length beyond the stated maximum, a position past the pages
 *     of its request) set bits of the device error word in the workspace and
 *     the offending rows are skipped; read it with qsa_device_error.
 *   - Positions are logical token indices of a request.  Logical position p of
 *     request r lives in physical slot page_table[r][p / 64] * 64 + p % 64.
 *   - Lengths: L is a context length INCLUDING the query token, whose position
 *     is L - 1.  A query sees floor(L/4) complete blocks and L mod 4 tail tokens.
 */
#ifndef QSA_H
#define QSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define QSA_HEAD_DIM 128    /* dims of every index head and attention head       */
#define QSA_INDEX_HEADS 4   /* index query heads (one shared index key head)     */
#define QSA_Q_HEADS 16      /* attention query heads                              */
#define QSA_KV_HEADS 2      /* attention KV heads; head h reads KV head h / 8    */
#define QSA_BLOCK 4         /* compression ratio c4                              */
#define QSA_TOPK 512        /* kept blocks                                        */
#define QSA_MAX_SEL 2051    /* 512 * 4 + 3 positions                              */
#define QSA_PAGE_SIZE 64    /* tokens per K/V page (16 compressed entries)        */
#define QSA_MAX_DRAFT 8     /* largest n_plus_1 of qsa_decode_indexshare          */
#define QSA_MAX_CONTEXT (1 << 20) /* largest context length accepted (1,048,576)    */
/* Outputs of the index projection per token: 4 x 128 query dims, 128 key dims, 4 head weights. */
#define QSA_PROJ_FEATURES (QSA_INDEX_HEADS * QSA_HEAD_DIM + QSA_HEAD_DIM + QSA_INDEX_HEADS) /* 644 */
#define QSA_MAX_HIDDEN 32768 /* largest hidden size of the index projection (a multiple of 128) */

typedef enum {
  QSA_OK = 0,
  QSA_ERR_INVALID_ARG = 1, /* null pointer, negative or inconsistent size          */
  QSA_ERR_UNSUPPORTED = 2, /* shape or configuration this build does not handle   */
  QSA_ERR_WORKSPACE = 3,   /* workspace null, misaligned or smaller than required */
  QSA_ERR_CUDA = 4         /* a CUDA launch or driver call failed                 */
} qsa_status;

/* Device error word bits (qsa_device_error). */
#define QSA_DEVERR_PAGE 1       /* page id outside [0, num_slots / 64)           */
#define QSA_DEVERR_LENGTH 2     /* length < 1, beyond max_len or past the pages  */
#define QSA_DEVERR_POSITION 4   /* an explicit position outside its request      */
#define QSA_DEVERR_REQUEST 8    /* a request index outside [0, batch)            */
#define QSA_DEVERR_SELECTION 16 /* a selection count outside [0, 512]            */
#define QSA_DEVERR_TIMEOUT 32   /* a bounded wait inside a kernel gave up        */

/*
 * The layer's cache.  All pointers are device pointers owned by the caller.
 *   k, v        bf16 raw attention keys / values of the paged pool: slot s holds
 *               its two KV heads' 128-d rows at k + s * kv_stride (and likewise v)
 *   cidx        bf16 [num_slots / 4][128] compressed index keys; block b of request r
 *               lives at entry (page_table[r][4b / 64] * 64 + 4b % 64) / 4, so one
 *               page's 16 entries are contiguous (page-aligned full_slot / 4 rule)
 *   ring        bf16 [batch][4][128]      raw index keys of each request's
 *               unfinished block, slot = position mod 4
 *   page_table  int32 [batch][max_pages]  physical page of each logical page
 *   num_slots   multiple of page_size; page_size must be 64
 *   kv_stride   bf16 elements from one slot to the next in k (and in v): 0 means
 *               256, i.e. separate [num_slots][2][128] arrays; 512 with
 *               v = k + 256 interleaves each slot's K and V rows, so that the
 *               4 slots of a compressed block are one 4 KiB run (the sparse
 *               GQA then reads whole 4 KiB runs instead of two 2 KiB pieces).
 *               Otherwise a multiple of 8, at least 256.
 *   rope_theta  RoPE base of the index keys/queries (1e7 for the workloads here)
 * Alignment: k, v, cidx, ring 16-byte aligned; page_table 4-byte aligned.
 */
typedef struct {
  void* k;
  void* v;
  void* cidx;
  void* ring;
  const int32_t* page_table;
  int64_t num_slots;
  int32_t page_size;
  int32_t max_pages;
  int32_t batch;
  int32_t kv_stride;
  double rope_theta;
} qsa_cache;

/* Operation ids for qsa_workspace_bytes. */
typedef enum {
  QSA_OP_INDEX_SCORE_TOPK = 1,
  QSA_OP_SPARSE_GQA = 2,
  QSA_OP_DECODE = 3,
  QSA_OP_DECODE_INDEXSHARE = 4,
  QSA_OP_COMPRESS_APPEND = 5,
  QSA_OP_PREFILL_SCORE_TOPK = 6,
  QSA_OP_DECODE_INDEXER = 7, /* qsa_decode_indexer: rows = batch, max_len = longest context */
  QSA_OP_DECODE_ATTEND = 8,  /* qsa_decode_attend:  rows = batch, max_len = longest context */
  QSA_OP_SPLIT_SCORE = 9     /* qsa_split_score_topk: rows = batch, max_len = longest context */
} qsa_op;

/*
 * Workspace bytes an operation needs for `rows` rows (queries for
 * QSA_OP_INDEX_SCORE_TOPK / QSA_OP_SPARSE_GQA, requests for the decode ops)
 * whose contexts are at most `max_len` tokens (for QSA_OP_SPARSE_GQA:
 * positions per query; for QSA_OP_DECODE_INDEXSHARE pass the capture length
 * L0).  Returns 0 for invalid arguments.  The workspace must be 256-byte
 * aligned and must be zeroed once with qsa_workspace_init before its first
 * use; the kernels leave it ready for the next call (after a call that
 * returned QSA_ERR_CUDA, zero it again).  Calls that share one workspace must
 * be ordered on the GPU (same stream or synchronised).
 */
size_t qsa_workspace_bytes(int32_t op, int32_t rows, int32_t max_len);

/* Zero a workspace (enqueued on `stream`). */
qsa_status qsa_workspace_init(void* ws, size_t ws_bytes, void* stream);

/*
 * Append new raw index keys to the cache (prefill / chunked prefill / decode).
 * Blog section "Qwen Sparse Attention: Retrieve Coarsely, Attend Precisely":
 * each group of 4 raw index keys becomes one compressed key (FP32 mean,
 * normalised, rotated at its first token's position, stored BF16); the keys
 * of the unfinished block wait in the 4-slot ring.
 *   idx_k_new   bf16 [total_new][128]  raw index keys, request r's keys in rows
 *               cu_new[r] .. cu_new[r+1]-1, at positions len_before[r] + j
 *   cu_new      int32 [batch + 1]      prefix offsets (device)
 *   len_before  int32 [batch]          tokens already appended per request (device)
 *   max_new     upper bound of cu_new[r+1]-cu_new[r] over r (host), >= 0
 * Completed blocks are written to cidx; the ring ends up holding the keys of
 * each request's unfinished block (slots of positions past the last appended
 * token keep whatever they held).  Appending a prefix in one call, token by
 * token, or in chunks gives bit-identical caches.
 */
qsa_status qsa_compress_append(const qsa_cache* cache, const void* idx_k_new, const int32_t* cu_new,
                               const int32_t* len_before, int32_t total_new, int32_t max_new, void* stream);

/*
 * Score the visible compressed blocks of each query and keep the top 512.
 * Blog section "Qwen Sparse Attention: Retrieve Coarsely, Attend Precisely"
 * (score formula as stated in this header's preamble; the text's own formula
 * is lost).  Query i belongs to request q_req[i] and sits at position
 * q_pos[i]; it scores blocks b < floor((q_pos[i]+1)/4).
 *   idx_q     bf16 [nq][4][128]  unrotated index queries (rotated here at q_pos)
 *   w         f32  [nq][4]       per-query head weights
 *   q_req     int32 [nq], q_pos int32 [nq]   (device)
 *   max_len   host bound of q_pos[i] + 1
 *   blocks    int32 [nq][512]  out: kept block ids, ascending; unused tail untouched
 *   nblocks   int32 [nq]       out: min(512, floor((q_pos+1)/4))
 *   ws        workspace of qsa_workspace_bytes(QSA_OP_INDEX_SCORE_TOPK, nq, max_len)
 */
qsa_status qsa_index_score_topk(const qsa_cache* cache, const void* idx_q, const float* w, const int32_t* q_req,
                                const int32_t* q_pos, int32_t nq, int32_t max_len, int32_t* blocks,
                                int32_t* nblocks, void* ws, size_t ws_bytes, void* stream);

/*
 * Prefill scoring of one causal chunk on the tensor cores: the queries at
 * positions pos0 .. pos0+T-1 of request `req` each score their complete
 * blocks b < floor((pos+1)/4) and keep the top 512.  Same result as
 * qsa_index_score_topk on those queries; built for long chunks, where the
 * chunk's queries share every compressed-key tile.  For queries that see
 * more than 8192 blocks scores do not go to memory: a sampled threshold per
 * query lets only likely members of its top 512 through as candidates, the
 * exact top 512 is taken among them, and a row the candidates cannot settle is
 * re-scored in full (exact either way); queries of shorter contexts write all
 * their score keys to the workspace and select from those.
 * Blog section "Qwen Sparse Attention: Retrieve Coarsely, Attend Precisely"
 * (prefill: a GPU kernel computes the index scores, a fast top-k selects).
 *   idx_q     bf16 [T][4][128] unrotated index queries
 *   w         f32  [T][4] head weights, 16-byte aligned
 *   req, pos0 host values; the cache must already hold the chunk's blocks
 *             (qsa_compress_append of positions up to pos0+T-1)
 *   blocks    int32 [T][512] out, ascending; nblocks int32 [T] out
 *   ws        workspace of qsa_workspace_bytes(QSA_OP_PREFILL_SCORE_TOPK, T, pos0+T)
 */
qsa_status qsa_prefill_score_topk(const qsa_cache* cache, const void* idx_q, const float* w, int32_t req,
                                  int32_t pos0, int32_t T, int32_t* blocks, int32_t* nblocks, void* ws,
                                  size_t ws_bytes, void* stream);

/*
 * Prefill scoring of a ragged batch of causal chunks in one call (chunked
 * prefill of several sequences at once: the aik8s.run deployment page runs
 * chunked prefill of 8192 tokens over concurrent requests).  Segment i is the
 * queries at positions seg_pos0[i] .. seg_pos0[i]+T_i-1 of request seg_req[i],
 * T_i = cu_q[i+1] - cu_q[i], stored at rows cu_q[i] .. cu_q[i+1]-1 of idx_q,
 * w, blocks and nblocks.  Each segment's result equals a
 * qsa_prefill_score_topk call on it alone.  Requests may share pages: when
 * two page tables map a shared prefix to the same physical pages, the
 * compressed keys of that prefix are one copy (block b of a request lives at
 * its own physical slot / 4, blog section "Qwen Sparse Attention: Retrieve
 * Coarsely, Attend Precisely", page-aligned full_slot / 4 addressing), and
 * both requests' queries score it.
 *   nseg         1 .. 64 (host); seg_req, seg_pos0 int32 [nseg] and cu_q int32 [nseg+1]
 *                are HOST arrays, cu_q[0] = 0, non-decreasing
 *   max_len      host bound of seg_pos0[i] + T_i
 *   idx_q        bf16 [cu_q[nseg]][4][128]; w f32 [cu_q[nseg]][4] (16-byte aligned)
 *   blocks, nblocks   int32 [cu_q[nseg]][512], [cu_q[nseg]] out
 *   ws           workspace of qsa_workspace_bytes(QSA_OP_PREFILL_SCORE_TOPK, cu_q[nseg], max_len)
 */
qsa_status qsa_prefill_score_topk_varlen(const qsa_cache* cache, const void* idx_q, const float* w, int32_t nseg,
                                         const int32_t* seg_req, const int32_t* seg_pos0, const int32_t* cu_q,
                                         int32_t max_len, int32_t* blocks, int32_t* nblocks, void* ws,
                                         size_t ws_bytes, void* stream);

/*
 * Expand kept blocks to token positions: block b -> 4b..4b+3 in block order,
 * then the tail 4*floor(L/4) .. L-1 with L = q_pos[i] + 1.
 * Blog section "Qwen Sparse Attention: Retrieve Coarsely, Attend Precisely".
 *   blocks  int32 [nq][512], nblocks int32 [nq], q_pos int32 [nq] (device)
 *   pos     int32 [nq][2051] out, npos int32 [nq] out (= 4*nblocks + L mod 4)
 */
qsa_status qsa_expand_indices(const int32_t* blocks, const int32_t* nblocks, const int32_t* q_pos, int32_t nq,
                              int32_t* pos, int32_t* npos, void* stream);

/*
 * Sparse GQA of nq query tokens, each over its own list of positions.
 * Blog section "Qwen Sparse Attention: Retrieve Coarsely, Attend Precisely":
 * softmax and value sum run over the raw, uncompressed K/V of the cache.
 *   q        bf16 [nq][16][128]
 *   q_req    int32 [nq] request of each query (device)
 *   pos      int32 [nq][pos_stride] positions (device); npos int32 [nq]
 *   max_pos  host bound of npos[i] (<= pos_stride and <= QSA_MAX_SEL, else
 *            QSA_ERR_UNSUPPORTED); a row whose npos exceeds 2051 is skipped
 *            and flagged QSA_DEVERR_SELECTION
 *   scale    softmax scale (1/sqrt(128) for the layer)
 *   out      bf16 [nq][16][128] out; lse f32 [nq][16] out (natural log) or NULL
 *   ws       workspace of qsa_workspace_bytes(QSA_OP_SPARSE_GQA, nq, max_pos)
 * A query with no positions gets zeros (lse = -inf).
 */
qsa_status qsa_sparse_gqa(const qsa_cache* cache, const void* q, const int32_t* q_req, const int32_t* pos,
                          const int32_t* npos, int32_t pos_stride, int32_t max_pos, int32_t nq, float scale,
                          void* out, float* lse, void* ws, size_t ws_bytes, void* stream);

/*
 * One decode step of the whole layer for every request of the cache:
 * append the new index key (ring; compress when it completes a block), rotate
 * the index query at seq_len[r]-1, score the complete blocks, keep the top
 * 512, and attend over the kept positions plus the tail.
 * Blog section "Qwen Sparse Attention: Retrieve Coarsely, Attend Precisely".
 *   idx_k_new  bf16 [batch][128]     index key of each request's new token
 *   idx_q      bf16 [batch][4][128]  unrotated index queries
 *   w          f32  [batch][4]       index head weights
 *   q          bf16 [batch][16][128] attention queries
 *   seq_len    int32 [batch] context length including the new token (device);
 *              the new token's K/V must already be in the pool
 *   max_len    host bound of seq_len
 *   out        bf16 [batch][16][128] out; lse f32 [batch][16] out or NULL
 *   blocks_out int32 [batch][512], nblocks_out int32 [batch]: the kept blocks
 *              (out, may both be NULL; IndexShare captures them from here)
 *   ws         workspace of qsa_workspace_bytes(QSA_OP_DECODE, batch, max_len)
 * Calling it twice with the same inputs gives the same result (the append is
 * idempotent).  The attention kernel is launched as a programmatic dependent
 * of the scoring kernel: it may start while the scorer finishes and waits, per
 * request, for that request's selection (bounded wait; QSA_DEVERR_TIMEOUT).
 */
qsa_status qsa_decode(const qsa_cache* cache, const void* idx_k_new, const void* idx_q, const float* w,
                      const void* q, const int32_t* seq_len, int32_t max_len, float scale, void* out, float* lse,
                      int32_t* blocks_out, int32_t* nblocks_out, void* ws, size_t ws_bytes, void* stream);

/*
 * FP8 K/V variants of qsa_sparse_gqa and qsa_decode.  The pages run FP8
 * checkpoints and an FP8 KV cache (the aik8s.run deployment page and the
 * ailone.io model page) but do not state its format; the reading used here:
 * the raw attention keys and values are E4M3 bytes with one FP32 scale for K
 * and one for V (value = code * scale); everything else, the compressed index
 * keys and the ring included, stays as in the bf16 calls.
 *   cache->k, cache->v   E4M3 bytes: slot s holds its two KV heads' 128-byte rows at
 *                        k + s * kv_stride (bytes; 0 means 256, separate arrays; 512 with
 *                        v = k + 256 interleaves K and V); kv_stride a multiple of 16
 *   k_scale, v_scale     positive, finite
 * Every other argument is that of qsa_sparse_gqa / qsa_decode (same workspaces).
 * Attention is computed on the exact dequantized values (each E4M3 value is a
 * bf16 value; the K scale joins the softmax scale and the V scale the output).
 */
qsa_status qsa_sparse_gqa_fp8(const qsa_cache* cache, float k_scale, float v_scale, const void* q,
                              const int32_t* q_req, const int32_t* pos, const int32_t* npos, int32_t pos_stride,
                              int32_t max_pos, int32_t nq, float scale, void* out, float* lse, void* ws,
                              size_t ws_bytes, void* stream);
qsa_status qsa_decode_fp8(const qsa_cache* cache, float k_scale, float v_scale, const void* idx_k_new,
                          const void* idx_q, const float* w, const void* q, const int32_t* seq_len, int32_t max_len,
                          float scale, void* out, float* lse, int32_t* blocks_out, int32_t* nblocks_out, void* ws,
                          size_t ws_bytes, void* stream);

/*
 * IndexShare draft step: attention only, the indexer is skipped.
 * Blog section "IndexShare MTP: Reusing the QSA Selection Across Draft Steps":
 * the selection captured at the last accepted token (position len0[r]-1) is
 * frozen; draft query i (i = 0 .. n_plus_1-1, position len0[r]+i) attends to
 * the frozen positions plus the drafted positions len0[r] .. len0[r]+i.
 *   frozen_pos  int32 [batch][frozen_stride] frozen positions (e.g. from
 *               qsa_expand_indices on qsa_decode's blocks_out), all < len0[r]
 *   frozen_n    int32 [batch]
 *   len0        int32 [batch] context length at capture (device)
 *   n_plus_1    drafted positions per request, 1 .. QSA_MAX_DRAFT (host)
 *   q           bf16 [batch][n_plus_1][16][128]
 *   out         bf16 [batch][n_plus_1][16][128] out
 *   ws          workspace of qsa_workspace_bytes(QSA_OP_DECODE_INDEXSHARE, batch, max_len0)
 */
qsa_status qsa_decode_indexshare(const qsa_cache* cache, const int32_t* frozen_pos, const int32_t* frozen_n,
                                 int32_t frozen_stride, const int32_t* len0, int32_t n_plus_1, const void* q,
                                 float scale, void* out, void* ws, size_t ws_bytes, void* stream);

/*
 * Index projection: hidden states -> index queries, index keys, head weights.
 * Blog section "Qwen Sparse Attention: Retrieve Coarsely, Attend Precisely":
 * the indexer has 4 query heads of 128 dims and one shared 128-dim key per
 * token.  The pages give no hidden size and do not say how the head weights
 * are formed; this library reads them as one bias-free linear map:
 *   [idx_q (4 x 128) | idx_k (128) | w (4)] = W_proj x
 * accumulated in FP32; idx_q and idx_k rounded once to bf16, w kept FP32.
 *   x       bf16 [n][hidden]                       hidden states (16-byte aligned rows)
 *   w_proj  bf16 [QSA_PROJ_FEATURES][hidden]       rows 0..511: query head h dim d at 128h + d;
 *                                                   rows 512..639: key dims; rows 640..643: head weights
 *   hidden  multiple of 128, at most QSA_MAX_HIDDEN
 *   idx_q   bf16 [n][4][128] out; idx_k bf16 [n][128] out; w f32 [n][4] out
 */
qsa_status qsa_index_project(const void* x, const void* w_proj, int32_t n, int32_t hidden, void* idx_q, void* idx_k,
                             float* w, void* stream);

/*
 * The decode step in two phases, so that the indexer can run on a second CUDA
 * stream while the caller computes the layer's main Q/K/V projection (blog
 * section "Qwen Sparse Attention: Retrieve Coarsely, Attend Precisely": the
 * indexer can overlap the main Q/K/V projection on a second stream).
 *
 * qsa_decode_indexer needs only the new tokens' hidden states: it projects
 * them (qsa_index_project), appends each request's new index key (ring, and
 * the compressed key when it completes a block), rotates the index queries,
 * scores the complete blocks and keeps the top 512.
 *   x        bf16 [batch][hidden] hidden state of each request's new token
 *   w_proj   bf16 [QSA_PROJ_FEATURES][hidden] (see qsa_index_project)
 *   seq_len  int32 [batch] context length including the new token (device)
 *   max_len  host bound of seq_len
 *   blocks   int32 [batch][512] out, ascending; nblocks int32 [batch] out
 *   ws       workspace of qsa_workspace_bytes(QSA_OP_DECODE_INDEXER, batch, max_len)
 * qsa_decode_attend then runs the sparse GQA over the kept blocks plus each
 * request's tail; it needs the attention queries and the new token's K/V in
 * the pool (the caller's main projection), and the indexer's blocks/nblocks
 * (order the streams with an event).
 *   q        bf16 [batch][16][128]; out bf16 [batch][16][128]; lse f32 [batch][16] or NULL
 *   ws       workspace of qsa_workspace_bytes(QSA_OP_DECODE_ATTEND, batch, max_len)
 *            (its own: the two phases of consecutive steps may run at once)
 * Together they compute what qsa_decode computes from the projected inputs.
 */
qsa_status qsa_decode_indexer(const qsa_cache* cache, const void* x, const void* w_proj, int32_t hidden,
                              const int32_t* seq_len, int32_t max_len, int32_t* blocks, int32_t* nblocks, void* ws,
                              size_t ws_bytes, void* stream);
qsa_status qsa_decode_attend(const qsa_cache* cache, const void* q, const int32_t* seq_len, int32_t max_len,
                             const int32_t* blocks, const int32_t* nblocks, float scale, void* out, float* lse,
                             void* ws, size_t ws_bytes, void* stream);

/*
 * Split-context decode: a request's context divided over several GPUs (ranks)
 * by page ranges, for one very long request that one GPU would decode slowly.
 * The pages describe no such split (the layer runs on one GPU there); this is
 * the plainest exact split of the decode step of blog section "Qwen Sparse
 * Attention: Retrieve Coarsely, Attend Precisely".  Each rank holds pages
 * [page_lo[r], page_lo[r] + page_cnt[r]) of request r in a cache of its own
 * whose page-table row is indexed by the request's logical page (only those
 * pages mapped), so positions and block numbers are the request's own
 * everywhere.  A step, on every rank:
 *   1. the rank holding position L-1 appends the new index key
 *      (qsa_compress_append at len_before = L-1);
 *   2. qsa_split_score_topk: its best min(512, its blocks) (score key, block)
 *      in block order, the index query rotated at L-1;
 *   3. an all-gather of the candidates in rank order (ranks hold increasing
 *      page ranges), then qsa_split_merge: the exact top 512 of the request,
 *      the same on every rank;
 *   4. qsa_split_positions: the kept positions the rank holds (plus the tail
 *      on the rank holding L-1), then qsa_sparse_gqa with lse;
 *   5. an all-gather of (out, lse) and qsa_split_combine.
 * qsa_split_score_topk:
 *   seq_len, page_lo, page_cnt   int32 [batch] (device)
 *   cand_key uint32 [batch][512], cand_id int32 [batch][512], cand_n int32 [batch] out
 *   ws  workspace of qsa_workspace_bytes(QSA_OP_SPLIT_SCORE, batch, max_len)
 * qsa_split_merge: cand_key / cand_id [world][rows][512], cand_n [world][rows]
 *   (the ranks' outputs stacked in rank order) -> blocks [rows][512] ascending,
 *   nblocks [rows]; world <= 64.
 * qsa_split_positions: -> pos int32 [rows][2051], npos int32 [rows].
 * qsa_split_combine: outs bf16 [world][rows][16][128], lses f32 [world][rows][16]
 *   (natural-log LSE; -inf for a rank without positions) -> out bf16 [rows][16][128].
 */
qsa_status qsa_split_score_topk(const qsa_cache* cache, const void* idx_q, const float* w, const int32_t* seq_len,
                                const int32_t* page_lo, const int32_t* page_cnt, int32_t max_len, uint32_t* cand_key,
                                int32_t* cand_id, int32_t* cand_n, void* ws, size_t ws_bytes, void* stream);
qsa_status qsa_split_merge(const uint32_t* cand_key, const int32_t* cand_id, const int32_t* cand_n, int32_t world,
                           int32_t rows, int32_t* blocks, int32_t* nblocks, void* stream);
qsa_status qsa_split_positions(const int32_t* seq_len, const int32_t* page_lo, const int32_t* page_cnt,
                               const int32_t* blocks, const int32_t* nblocks, int32_t rows, int32_t* pos,
                               int32_t* npos, void* stream);
qsa_status qsa_split_combine(const void* outs, const float* lses, int32_t world, int32_t rows, void* out,
                             void* stream);

/*
 * Sparse GQA without a workspace: the same computation as qsa_sparse_gqa
 * (same arguments minus ws / ws_bytes), for callers that cannot allocate
 * device memory or pass the library scratch space -- e.g. a plugin whose host
 * hands it only input and output buffers, code running during CUDA-graph
 * capture where cudaMalloc is not allowed, or a deployment whose device memory
 * is fixed at start-up.  The QSA description has no counterpart: this is an
 * interface convenience of this library, not a step of the method.
 *   Scratch: a file-scope device array of QSA_NOALLOC_SCRATCH_BYTES (about
 *   4.1 MiB) that every GPU which loads the library keeps until the process
 *   exits.  It holds split-K partials for at most QSA_NOALLOC_ROW_SPLITS
 *   (query, split) pairs, so fewer splits are used for large nq.
 *   Limit: nq <= QSA_NOALLOC_MAX_QUERIES, else QSA_ERR_UNSUPPORTED is returned
 *   before anything is enqueued.
 *   The entry point allocates nothing (no cudaMalloc / cudaFree, no allocating
 *   library call).  Its first call on a device looks up the array's device
 *   address (cudaGetSymbolAddress) with that device current; make that first
 *   call before any stream capture.  Each call zeroes the arrival counters it
 *   uses (cudaMemsetAsync on `stream`).
 *   All calls share the one array, which keeps the last call's contents: calls
 *   that overlap on the GPU (different streams, no ordering) race and give
 *   wrong results.  Device-side data errors are not reported (there is no
 *   error word): a position whose page lies outside the request's page-table row, or whose
 *   page id lies outside the pool, is skipped (a position past the request's length on a
 *   page it owns is read like any other).
 */
#define QSA_NOALLOC_MAX_QUERIES 4096
#define QSA_NOALLOC_ROW_SPLITS 512
#define QSA_NOALLOC_SCRATCH_BYTES                                          \
  (256 + 4 * QSA_NOALLOC_MAX_QUERIES + 4 * QSA_NOALLOC_ROW_SPLITS * 16 * 2 + \
   4 * QSA_NOALLOC_ROW_SPLITS * 16 * 128)
qsa_status qsa_sparse_gqa_noalloc(const qsa_cache* cache, const void* q, const int32_t* q_req, const int32_t* pos,
                                  const int32_t* npos, int32_t pos_stride, int32_t max_pos, int32_t nq, float scale,
                                  void* out, float* lse, void* stream);

/*
 * Failure detection without a GPU fault: a check that the kernels' bounded
 * waits end.  Every wait inside a kernel of this library (the decode attention
 * waiting for its request's selection, the prefill scorer's pipeline barriers)
 * gives up after a limit (2 s), records QSA_DEVERR_TIMEOUT and lets the kernel
 * finish, so no wait can hang the GPU.  This call launches the decode attention
 * kernel for request 0 of `cache` with a selection that nothing publishes and a
 * limit of `limit_ns` nanoseconds: the kernel waits, gives up, sets
 * QSA_DEVERR_TIMEOUT in the workspace's error word and writes zeros to `out`.
 * The CUDA context stays usable; read the outcome with qsa_device_error.
 * Not a step of the method (the QSA description has no counterpart).
 *   q         bf16 [16][128] a query (device; read, its values do not matter)
 *   out       bf16 [16][128] out (zeros)
 *   limit_ns  1 .. 2e9
 *   ws        workspace of qsa_workspace_bytes(QSA_OP_DECODE, 1, 8), zeroed
 */
qsa_status qsa_check_bounded_wait(const qsa_cache* cache, const void* q, void* out, uint64_t limit_ns, void* ws,
                                  size_t ws_bytes, void* stream);

/*
 * Read (and optionally clear) the device error word of a workspace.  This
 * call synchronises `stream`.  Returns the QSA_DEVERR_* bits, or -1 if the
 * copy failed.
 */
int32_t qsa_device_error(void* ws, int32_t clear, void* stream);

/*
 * Measurement hook: when `events` is non-NULL, qsa_decode records
 * events[2*i] before and events[2*i+1] after its i-th kernel (i < n_pairs)
 * on its stream; qsa_prefill_score_topk does the same around its rotation
 * (i = 0), scoring (i = 1) and finalize (i = 2) kernels.  Each entry is a cudaEvent_t.  Pass NULL to switch it off.
 * Not thread-safe with concurrent qsa_decode calls from several host threads.
 */
void qsa_set_profile_events(void* const* events, int32_t n_pairs);

/*
 * Measurement hook of qsa_prefill_score_topk: how many rows of the last call
 * made with workspace `ws` (sized for T queries and contexts up to max_len)
 * could not be settled from their filtered candidates and were re-scored in
 * full.  Synchronises `stream`.  Returns -1 on error.
 */
int32_t qsa_prefill_rescored_rows(void* ws, int32_t T, int32_t max_len, void* stream);

/*
 * Measurement hook of qsa_prefill_score_topk: copies the rotated index queries
 * of the last call made with workspace `ws` (sized for T queries and contexts
 * up to max_len), bf16 [T][4][128] as uint16 bit patterns, into `out`, a HOST
 * buffer of T*4*128*2 bytes owned by the caller, so that the rotation can be
 * checked against its plain definition (blog section "Qwen Sparse Attention:
 * Retrieve Coarsely, Attend Precisely": the index query is rotated at its own
 * position).  Synchronises `stream`.  QSA_ERR_INVALID_ARG for a null pointer or
 * sizes no workspace layout has; QSA_ERR_CUDA when the copy fails.
 */
qsa_status qsa_prefill_rotated_queries(const void* ws, int32_t T, int32_t max_len, void* out, void* stream);

/* Number of kernels qsa_decode launches per call for `batch` requests: 2 up to
 * 512 requests (the scorer runs the indexer front end itself, then the sparse
 * GQA), 3 above (a separate front-end kernel first). */
int32_t qsa_decode_kernel_count(int32_t batch);

const char* qsa_status_string(qsa_status s);
/* Text of the CUDA error behind the calling thread's last QSA_ERR_CUDA. */
const char* qsa_last_error_string(void);
const char* qsa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* QSA_H */
