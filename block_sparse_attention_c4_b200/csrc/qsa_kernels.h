// Internal launch interface between the C-ABI layer (qsa_api.cu) and the
// kernel translation units.  Not part of the public ABI.
#pragma once

#include "qsa_common.cuh"

namespace qsa {

// Host checks of the paged K/V part of a cache (what the sparse GQA reads), shared by every entry
// point that attends: pointers, page size, pool size, strides and alignment.
inline bool host_aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

inline qsa_status check_kv_cache(const qsa_cache* c) {
  if (!c) return QSA_ERR_INVALID_ARG;
  if (!c->k || !c->v || !c->page_table) return QSA_ERR_INVALID_ARG;
  if (c->page_size != QSA_PAGE_SIZE) return QSA_ERR_UNSUPPORTED;
  if (c->num_slots <= 0 || c->num_slots % QSA_PAGE_SIZE != 0) return QSA_ERR_INVALID_ARG;
  if (c->num_slots / QSA_PAGE_SIZE > (int64_t)INT32_MAX / QSA_PAGE_SIZE) return QSA_ERR_UNSUPPORTED;
  if (c->max_pages <= 0 || c->batch < 0) return QSA_ERR_INVALID_ARG;
  if (c->kv_stride != 0 && (c->kv_stride < HKV * D || c->kv_stride % 8 != 0)) return QSA_ERR_INVALID_ARG;
  if (!host_aligned(c->k, 16) || !host_aligned(c->v, 16) || !host_aligned(c->page_table, 4))
    return QSA_ERR_INVALID_ARG;
  return QSA_OK;
}

// A softmax scale the kernels accept: positive and finite.
inline bool valid_scale(float scale) { return scale > 0.f && scale <= 3.4e38f; }

// ---- indexer front end (qsa_indexer.cu) ----
cudaError_t launch_compress_append(const CacheView& c, const __nv_bfloat16* knew, const int32_t* cu_new,
                                   const int32_t* len_before, int total_new, int max_new, const RopeFreqs& fr,
                                   int* err, cudaStream_t st);
// Rotates each row's index query (and, for decode, appends the new index key),
// writes the row's number of pages to score, and -- in the CTA that finishes
// last -- the exclusive prefix of those page counts (page_off[rows + 1]).
cudaError_t launch_index_prologue(const CacheView& c, const __nv_bfloat16* knew, const __nv_bfloat16* idx_q,
                                  const int32_t* row_req, const int32_t* row_len, int len_offset, int rows,
                                  int max_len, const RopeFreqs& fr, __nv_bfloat16* qrot, int32_t* row_pages,
                                  int32_t* page_off, int* ticket, int* err, cudaStream_t st);
cudaError_t launch_expand(const int32_t* blocks, const int32_t* nblocks, const int32_t* q_pos, int nq, int32_t* pos,
                          int32_t* npos, int* err, cudaStream_t st);

// ---- streaming scorer + top-512 (qsa_score.cu) ----
#ifndef QSA_SC_WARPS
#define QSA_SC_WARPS 16
#endif
// pages of one segment (16 blocks of score keys each, all in shared memory)
constexpr int SC_MAX_SEG_PAGES = QSA_SC_WARPS >= 16 ? 1024 : 512;
constexpr int SC_MAX_SEGS = 64;        // segments per row a merge can order
constexpr int SC_MIN_PPC = 32;         // pages per CTA range, lower bound
// Work of starting a row's segment (row setup, a partial top-512, its hand-over), in pages of
// streaming: the page list gives every row this many empty pages in front of its own, so a range
// that crosses into a row streams that many fewer pages.
#ifndef QSA_SC_ROW_COST
#define QSA_SC_ROW_COST 64
#endif
constexpr int SC_ROW_COST = QSA_SC_ROW_COST;

struct ScoreParams {
  CacheView c;
  const int32_t* row_req;  // nullable: row r is request r
  const int32_t* row_len;  // L = row_len[row] + len_offset
  int len_offset;
  int max_len;
  int rows;
  const __nv_bfloat16* qrot;  // [rows][4][128] rotated index queries
  const float* w;             // [rows][4]
  const int32_t* page_off;    // [rows + 1] exclusive prefix of pages to score per row
  int ppc_min;                // pages per CTA range, lower bound
  int seg_cap;                // segment slots per row (a partial segment's 512 candidates go to slot j,
                              // its rank among the row's segments in block order)
  int* pages_done;            // [rows], zero between calls
  uint32_t* cand_key;         // [rows][seg_cap * 512]
  int32_t* cand_id;           // [rows][seg_cap * 512]
  int32_t* sel;               // [rows][512] out
  int32_t* sel_n;             // [rows] out
  int* err;
  // Fused front end (rows <= SC_ROWS_SMEM): with idx_q set, every CTA computes the page prefix
  // itself (page_off unused), the CTA starting a row rotates that row's index query (qrot unused),
  // and with knew set the CTA owning a row's last page first appends the row's new index key.
  const __nv_bfloat16* idx_q;  // nullable: [rows][4][128] unrotated index queries
  const __nv_bfloat16* knew;   // nullable: [rows][128] decode index keys
  RopeFreqs fr;
  int* row_ready;              // nullable: [rows][READY_STRIDE] set to 1 once a row's selection is final
};
constexpr int SC_ROWS_SMEM = 512;  // rows whose page offsets fit shared memory (fused front end)

// Launches the persistent scorer on every SM (as many CTAs per SM as are resident).
cudaError_t launch_score_topk(const ScoreParams& p, int num_sms, cudaStream_t st);

// ---- sparse GQA (qsa_gqa.cu) ----
constexpr int GQ_MAX_SPLITS = 16;

struct GqaParams {
  CacheView c;
  const __nv_bfloat16* q;   // [rows][nq_row][16][128]
  int nq_row;               // queries per row sharing one position list
  const int32_t* row_req;   // nullable
  int mode;                 // 0: kept blocks + tail, 1: explicit list
  const int32_t* sel;       // mode 0: [rows][512]
  const int32_t* sel_n;     // mode 0: [rows]
  const int32_t* row_len;   // mode 0: L = row_len[row] + len_offset
  int len_offset;
  int max_len;
  const int32_t* list;      // mode 1: [rows][list_stride]
  const int32_t* list_n;    // mode 1: [rows]
  int list_stride;
  const int32_t* extra_base;  // nullable: extra positions extra_base[row] + e, e < n_extra
  int n_extra;                // query i sees extra e <= i
  float scale_log2;           // softmax scale * log2(e)
  __nv_bfloat16* out;         // [rows][nq_row][16][128]
  float* lse;                 // nullable, [rows][nq_row][16]
  float* part_o;              // [rows][splits][nq_row*16][128]
  float* part_ml;             // [rows][splits][nq_row*16][2]
  int* counters;              // [rows]
  int splits;                 // set by launch_gqa
  int tiles_per_split;        // set by launch_gqa
  int* err;
  int* row_ready;             // nullable (mode 0, [rows][READY_STRIDE]): wait for the row's flag, then clear it;
                              // the kernel is then launched as a programmatic dependent of the scorer
  int cluster_merge;          // 1: a row's splits may form one thread-block cluster and merge their partials
                              // through distributed shared memory (part_o, part_ml, counters unused);
                              // 0: partials go through global memory, the last split merges them
  uint64_t wait_ns;           // limit of the row-flag wait (0: WAIT_LIMIT_NS)
  int fp8;                    // 1: K/V are E4M3 bytes (c.kv_stride in bytes), scale_log2 includes the K scale
  float v_scale;              // fp8: scale of the V values
};
constexpr int GQ_CLUSTER_MAX = 8;  // splits of one row in a cluster (portable cluster size)

// Upper bound of the split count launch_gqa may choose (workspace sizing).
int gqa_split_bound(int rows, int max_pos);
// Chooses the split count (one wave of resident CTAs, at most split_bound) and launches.
cudaError_t launch_gqa(const GqaParams& p, int rows, int max_pos, int num_sms, int split_bound, cudaStream_t st);

// ---- prefill scorer on tcgen05 (qsa_prefill.cu) ----
constexpr int PF_QCAP = 512;            // candidates kept per (query, TMEM quadrant) list
constexpr int PF_EMIT_ALL = 4 * PF_QCAP - 128;  // queries with at most this many blocks emit every block
constexpr int PF_NO_BASE = -(1 << 30);  // a query whose scores are all <= 0 (no histogram range)
constexpr int PF_DENSE_MAX = 8192;      // work tiles whose queries see at most this many blocks write every
                                        // score key instead of filtered candidates
// 8-byte words of one query row's area: its 4 candidate lists, or its dense score keys (4 bytes each)
constexpr int PF_ROW_WORDS = 4 * PF_QCAP > PF_DENSE_MAX / 2 ? 4 * PF_QCAP : PF_DENSE_MAX / 2;
// A work tile of 64 consecutive queries of a segment (first position pos0, T queries), tile qt: its
// queries see at most this many blocks; the tile is dense when that is at most PF_DENSE_MAX.
__host__ __device__ inline int pf_tile_nbv_hi(int pos0, int T, int qt) {
  const int last = (qt + 1) * 64 < T ? (qt + 1) * 64 : T;
  return (pos0 + last) >> 2;
}

// One sequence of a (ragged) prefill call: request req, queries at positions pos0 .. pos0+T-1, stored
// at rows q_off .. q_off+T-1 of the call's query arrays.  The segments are listed in the order their
// work is scheduled (longest contexts first); tile_off / row_off are prefix sums in that order.
constexpr int PF_MAX_SEGS = 64;
struct PfSeg {
  int req, pos0, T, q_off, tile_off, row_off;
};

struct PrefillParams {
  CacheView c;
  int nseg;                // segments (1 .. PF_MAX_SEGS)
  int T;                   // queries of the call (all segments)
  int ntiles;              // work tiles of 64 queries (all segments)
  PfSeg seg[PF_MAX_SEGS];
  const float* w;          // [T][4] head weights (16-byte aligned)
  __nv_bfloat16* qrot;     // [T*4][128] rotated index queries (written by the rotation kernel)
  int32_t* qbase;          // [T] histogram base of each query (rotation kernel), or PF_NO_BASE
  unsigned long long* cand;  // [T][PF_ROW_WORDS] per query row: 4 lists of PF_QCAP candidates (key << 32 | ~block),
                             // one per TMEM quadrant; or, in a dense tile, the score key of every block (uint32)
  int32_t* cand_n;         // [T][4] candidates emitted per list (may exceed PF_QCAP: overflow)
  int32_t* sel;            // [T][512] out
  int32_t* sel_n;          // [T] out
  int* fb_n;               // rows handed to the exact re-scoring (zeroed per call)
  int32_t* fb_list;        // [T]
  uint32_t* fb_keys;       // [fb_ctas][fb_cap] score keys of the rows being re-scored
  int fb_cap;              // >= blocks visible to the chunk's last query, a multiple of 16
  int fb_ctas;             // CTAs of the re-scoring kernel (rows of fb_keys)
  int* err;
  uint64_t wait_ns;        // limit of each mbarrier wait (0: WAIT_LIMIT_NS)
  int* stats;              // nullable [4]: rows selected from candidates, rows re-scored, candidates, -
  int sel_r0, sel_pivot;   // one segment, sel_pivot > 0: the selection's row order (see k_prefill_select)
};

// ---- index projection (qsa_proj.cu) ----
struct ProjParams {
  const __nv_bfloat16* x;  // [n][hidden] hidden states
  const __nv_bfloat16* w;  // [QSA_PROJ_FEATURES][hidden] projection weights
  int n, hidden;           // hidden: a multiple of 128
  __nv_bfloat16* idx_q;    // [n][4][128] out
  __nv_bfloat16* idx_k;    // [n][128] out
  float* wout;             // [n][4] out
};
cudaError_t launch_index_proj(const ProjParams& p, cudaStream_t st);

// ---- split-context decode (qsa_split.cu) ----
constexpr int SPLIT_MAX_LISTS = 64;  // candidate lists a merge takes: ranks, or chunks of one rank
constexpr int SPLIT_CHUNK_BLOCKS = 8192;  // most blocks one CTA of the split scorer takes
constexpr int SPLIT_CHUNK_MIN = 2048;     // fewest (fewer, longer chunks: a row's merge has fewer lists)
// Blocks per CTA of the split scorer for contexts up to max_len: the smallest multiple of 16 (at least
// SPLIT_CHUNK_MIN) that keeps a row's chunks within SPLIT_MAX_LISTS, so a rank's blocks spread over
// many CTAs; 0 when even SPLIT_CHUNK_BLOCKS per CTA leaves too many chunks.
inline int split_chunk(int max_len) {
  const int nb = max_len / QSA_BLOCK > 1 ? max_len / QSA_BLOCK : 1;
  int c = (nb + SPLIT_MAX_LISTS - 1) / SPLIT_MAX_LISTS;
  c = (c + 15) / 16 * 16;
  if (c < SPLIT_CHUNK_MIN) c = SPLIT_CHUNK_MIN;
  return c <= SPLIT_CHUNK_BLOCKS ? c : 0;
}
struct SplitParams {
  CacheView c;                 // the rank's cache (page-table rows indexed by global logical page)
  const __nv_bfloat16* idx_q;  // [rows][4][128] unrotated index queries
  const float* w;              // [rows][4]
  const int32_t* seq_len;      // [rows] context length including the query token
  const int32_t* page_lo;      // [rows] first page this rank holds
  const int32_t* page_cnt;     // [rows] pages this rank holds
  int max_len;
  RopeFreqs fr;
  int chunk;                   // blocks per chunk (one CTA), a multiple of 16, <= SPLIT_CHUNK_BLOCKS
  int nchunks;                 // chunks per row
  uint32_t* cand_key;          // [rows][nchunks][512]
  int32_t* cand_id;            // [rows][nchunks][512]
  int32_t* cand_n;             // [rows][nchunks]
  uint32_t* out_key;           // [rows][512] the rank's best 512 (key, block), block order
  int32_t* out_id;             // [rows][512]
  int32_t* out_n;              // [rows]
  int* err;
};
cudaError_t launch_split_score(const SplitParams& p, int rows, cudaStream_t st);
cudaError_t launch_split_merge(const uint32_t* keys, const int32_t* ids, const int32_t* n, int world, int rows,
                               int32_t* blocks, int32_t* nblocks, cudaStream_t st);
cudaError_t launch_split_positions(const SplitParams& p, const int32_t* blocks, const int32_t* nblocks, int rows,
                                   int32_t* pos, int32_t* npos, cudaStream_t st);
cudaError_t launch_split_combine(const __nv_bfloat16* outs, const float* lses, int world, int rows,
                                 __nv_bfloat16* out, cudaStream_t st);

// ev (nullable): n_ev event pairs recorded around the rotation, scoring and finalize kernels.
cudaError_t launch_prefill(PrefillParams p, const __nv_bfloat16* idx_q, const RopeFreqs& fr, int num_sms,
                           cudaStream_t st, const cudaEvent_t* ev, int n_ev);

}  // namespace qsa
