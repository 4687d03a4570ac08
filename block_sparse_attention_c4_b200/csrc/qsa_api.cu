// C ABI of the QSA c4 layer (declared in include/qsa.h): argument checks,
// workspace carving, TMA descriptors and the launch sequences.  Every step of
// the computation runs in the kernels of qsa_indexer.cu, qsa_score.cu and
// qsa_gqa.cu; this file only marshals arguments.
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "qsa_common.cuh"
#include "qsa_kernels.h"

using namespace qsa;

namespace {

constexpr int MAX_DEVICES = 64;
constexpr int SIZING_SMS = 256;  // upper bound of SMs used to size workspaces without a device

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

struct WsLayout {
  size_t cnt_score = 0, cnt_gqa = 0, qrot = 0, sel = 0, sel_n = 0, cand_key = 0, cand_id = 0, part_o = 0,
         part_ml = 0, total = 0;
  int max_chunks_bound = 0;
  int splits_bound = 0;
};

int positions_bound(int op, int max_len) {
  if (op == QSA_OP_SPARSE_GQA) return max_len;
  if (op == QSA_OP_DECODE_INDEXSHARE) return QSA_MAX_SEL + QSA_MAX_DRAFT;
  return std::min(QSA_TOPK * QSA_BLOCK, (max_len / QSA_BLOCK) * QSA_BLOCK) + QSA_BLOCK - 1;
}

// Workspace carving.  Returns false for invalid arguments.
bool layout(int op, int rows, int max_len, WsLayout& w) {
  if (rows < 0 || max_len < 0 || max_len > QSA_MAX_CONTEXT) return false;
  const bool scorer = op == QSA_OP_INDEX_SCORE_TOPK || op == QSA_OP_DECODE;
  const bool gqa = op == QSA_OP_SPARSE_GQA || op == QSA_OP_DECODE || op == QSA_OP_DECODE_INDEXSHARE;
  if (!scorer && !gqa && op != QSA_OP_COMPRESS_APPEND) return false;
  size_t off = 256;  // error word and spare
  w.cnt_score = off;
  off += align256(sizeof(int) * (size_t)rows);
  w.cnt_gqa = off;
  off += align256(sizeof(int) * (size_t)rows);
  if (scorer) {
    const int nb = max_len / QSA_BLOCK;
    w.max_chunks_bound = std::max(1, ceil_div(nb, SC_MIN_CHUNK));
    w.qrot = off;
    off += align256((size_t)rows * HI * D * 2);
    w.sel = off;
    off += align256((size_t)rows * TOPK * 4);
    w.sel_n = off;
    off += align256((size_t)rows * 4);
    w.cand_key = off;
    off += align256((size_t)rows * w.max_chunks_bound * TOPK * 4);
    w.cand_id = off;
    off += align256((size_t)rows * w.max_chunks_bound * TOPK * 4);
  }
  if (gqa) {
    const int nq_row = op == QSA_OP_DECODE_INDEXSHARE ? QSA_MAX_DRAFT : 1;
    w.splits_bound = gqa_splits_for(rows, positions_bound(op, max_len), nq_row, SIZING_SMS);
    const size_t heads = (size_t)nq_row * HQ;
    w.part_o = off;
    off += align256((size_t)rows * w.splits_bound * heads * D * 4);
    w.part_ml = off;
    off += align256((size_t)rows * w.splits_bound * heads * 2 * 4);
  }
  w.total = off;
  return true;
}

int num_sms() {
  static int cached[MAX_DEVICES] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= MAX_DEVICES) return 148;
  if (cached[dev] == 0) {
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    cached[dev] = n > 0 ? std::min(n, SIZING_SMS) : 148;
  }
  return cached[dev];
}

RopeFreqs make_freqs(double theta) {
  RopeFreqs f;
  for (int i = 0; i < D / 2; ++i) f.f[i] = std::pow(theta, -static_cast<double>(i) / (D / 2));
  return f;
}

qsa_status check_cache(const qsa_cache* c) {
  if (!c) return QSA_ERR_INVALID_ARG;
  if (!c->k || !c->v || !c->cidx || !c->ring || !c->page_table) return QSA_ERR_INVALID_ARG;
  if (c->page_size != QSA_PAGE_SIZE) return QSA_ERR_UNSUPPORTED;
  if (c->num_slots <= 0 || c->num_slots % QSA_PAGE_SIZE != 0) return QSA_ERR_INVALID_ARG;
  if (c->num_slots / QSA_PAGE_SIZE > (int64_t)INT32_MAX / QSA_PAGE_SIZE) return QSA_ERR_UNSUPPORTED;
  if (c->max_pages <= 0 || c->batch < 0) return QSA_ERR_INVALID_ARG;
  if (!(c->rope_theta > 0.0) || !std::isfinite(c->rope_theta)) return QSA_ERR_INVALID_ARG;
  if (!aligned(c->k, 16) || !aligned(c->v, 16) || !aligned(c->cidx, 16) || !aligned(c->ring, 16) ||
      !aligned(c->page_table, 4))
    return QSA_ERR_INVALID_ARG;
  return QSA_OK;
}

CacheView view_of(const qsa_cache* c) {
  CacheView v;
  v.k = static_cast<const __nv_bfloat16*>(c->k);
  v.v = static_cast<const __nv_bfloat16*>(c->v);
  v.cidx = static_cast<__nv_bfloat16*>(c->cidx);
  v.ring = static_cast<__nv_bfloat16*>(c->ring);
  v.page_table = c->page_table;
  v.num_pages = c->num_slots / QSA_PAGE_SIZE;
  v.max_pages = c->max_pages;
  v.batch = c->batch;
  return v;
}

qsa_status check_ws(void* ws, size_t ws_bytes, size_t need) {
  if (!ws || !aligned(ws, 256)) return QSA_ERR_WORKSPACE;
  if (ws_bytes < need) return QSA_ERR_WORKSPACE;
  return QSA_OK;
}

template <typename T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<uint8_t*>(ws) + off);
}

// ---- TMA descriptor of the compressed cache: [num_slots/4 rows][128 bf16] ----
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

bool make_cidx_map(const qsa_cache* c, CUtensorMap* map) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)(c->num_slots / QSA_BLOCK)};
  const cuuint64_t strides[1] = {(cuuint64_t)D * 2};
  const cuuint32_t box[2] = {64, (cuuint32_t)PAGE_BLOCKS};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, c->cidx, dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ---- measurement hook ----
std::mutex g_prof_mu;
cudaEvent_t g_prof[16];
int g_prof_pairs = 0;

struct ProfScope {
  cudaStream_t st;
  int idx;
  ProfScope(cudaStream_t s, int i) : st(s), idx(i) {
    if (idx < g_prof_pairs) cudaEventRecord(g_prof[2 * idx], st);
  }
  ~ProfScope() {
    if (idx < g_prof_pairs) cudaEventRecord(g_prof[2 * idx + 1], st);
  }
};

qsa_status cuda_status(cudaError_t e) { return e == cudaSuccess ? QSA_OK : QSA_ERR_CUDA; }

// Scorer pass shared by qsa_decode and qsa_index_score_topk (after the prologue).
qsa_status run_scorer(const qsa_cache* cache, const CacheView& cv, const int32_t* row_req, const int32_t* row_len,
                      int len_offset, int rows, int max_len, const __nv_bfloat16* qrot, const float* w, int32_t* sel,
                      int32_t* sel_n, void* ws, const WsLayout& L, int* err, cudaStream_t st) {
  CUtensorMap map;
  if (!make_cidx_map(cache, &map)) return QSA_ERR_CUDA;
  ScoreParams p;
  p.c = cv;
  p.row_req = row_req;
  p.row_len = row_len;
  p.len_offset = len_offset;
  p.max_len = max_len;
  p.qrot = qrot;
  p.w = w;
  p.chunk = score_chunk_for(rows, max_len, num_sms());
  p.max_chunks = std::max(1, ceil_div(max_len / QSA_BLOCK, p.chunk));
  if (p.max_chunks > L.max_chunks_bound) return QSA_ERR_WORKSPACE;
  p.cand_key = at<uint32_t>(ws, L.cand_key);
  p.cand_id = at<int32_t>(ws, L.cand_id);
  p.counters = at<int>(ws, L.cnt_score);
  p.sel = sel;
  p.sel_n = sel_n;
  p.err = err;
  return cuda_status(launch_score_topk(p, rows, &map, st));
}

}  // namespace

extern "C" {

const char* qsa_version(void) { return "qsa-b200 0.1 (sm_100a)"; }

const char* qsa_status_string(qsa_status s) {
  switch (s) {
    case QSA_OK: return "ok";
    case QSA_ERR_INVALID_ARG: return "invalid argument";
    case QSA_ERR_UNSUPPORTED: return "unsupported configuration";
    case QSA_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case QSA_ERR_CUDA: return "CUDA error";
  }
  return "unknown status";
}

size_t qsa_workspace_bytes(int32_t op, int32_t rows, int32_t max_len) {
  WsLayout w;
  return layout(op, rows, max_len, w) ? w.total : 0;
}

qsa_status qsa_workspace_init(void* ws, size_t ws_bytes, void* stream) {
  if (!ws || !aligned(ws, 256) || ws_bytes < 256) return QSA_ERR_WORKSPACE;
  return cuda_status(cudaMemsetAsync(ws, 0, ws_bytes, static_cast<cudaStream_t>(stream)));
}

int32_t qsa_device_error(void* ws, int32_t clear, void* stream) {
  if (!ws) return -1;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int v = 0;
  if (cudaMemcpyAsync(&v, ws, sizeof(int), cudaMemcpyDeviceToHost, st) != cudaSuccess) return -1;
  if (cudaStreamSynchronize(st) != cudaSuccess) return -1;
  if (clear && cudaMemsetAsync(ws, 0, sizeof(int), st) != cudaSuccess) return -1;
  return v;
}

void qsa_set_profile_events(void* const* events, int32_t n_pairs) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  if (!events || n_pairs <= 0) {
    g_prof_pairs = 0;
    return;
  }
  n_pairs = std::min(n_pairs, 8);
  for (int i = 0; i < 2 * n_pairs; ++i) g_prof[i] = static_cast<cudaEvent_t>(events[i]);
  g_prof_pairs = n_pairs;
}

int32_t qsa_decode_kernel_count(void) { return 3; }

qsa_status qsa_compress_append(const qsa_cache* cache, const void* idx_k_new, const int32_t* cu_new,
                               const int32_t* len_before, int32_t total_new, int32_t max_new, void* stream) {
  qsa_status s = check_cache(cache);
  if (s != QSA_OK) return s;
  if (total_new < 0 || max_new < 0) return QSA_ERR_INVALID_ARG;
  if (!cu_new || !len_before) return QSA_ERR_INVALID_ARG;
  if (cache->batch == 0 || total_new == 0) return QSA_OK;
  if (!idx_k_new || !aligned(idx_k_new, 16)) return QSA_ERR_INVALID_ARG;
  if (max_new > total_new) max_new = total_new;
  const RopeFreqs fr = make_freqs(cache->rope_theta);
  return cuda_status(launch_compress_append(view_of(cache), static_cast<const __nv_bfloat16*>(idx_k_new), cu_new,
                                            len_before, total_new, max_new, fr, nullptr,
                                            static_cast<cudaStream_t>(stream)));
}

qsa_status qsa_index_score_topk(const qsa_cache* cache, const void* idx_q, const float* w, const int32_t* q_req,
                                const int32_t* q_pos, int32_t nq, int32_t max_len, int32_t* blocks,
                                int32_t* nblocks, void* ws, size_t ws_bytes, void* stream) {
  qsa_status s = check_cache(cache);
  if (s != QSA_OK) return s;
  if (nq < 0 || max_len < 1 || max_len > QSA_MAX_CONTEXT) return QSA_ERR_INVALID_ARG;
  if (nq == 0) return QSA_OK;
  if (!idx_q || !w || !q_req || !q_pos || !blocks || !nblocks) return QSA_ERR_INVALID_ARG;
  if (!aligned(idx_q, 16) || !aligned(w, 4)) return QSA_ERR_INVALID_ARG;
  WsLayout L;
  if (!layout(QSA_OP_INDEX_SCORE_TOPK, nq, max_len, L)) return QSA_ERR_INVALID_ARG;
  if ((s = check_ws(ws, ws_bytes, L.total)) != QSA_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const CacheView cv = view_of(cache);
  const RopeFreqs fr = make_freqs(cache->rope_theta);
  int* err = at<int>(ws, 0);
  __nv_bfloat16* qrot = at<__nv_bfloat16>(ws, L.qrot);
  s = cuda_status(launch_index_prologue(cv, nullptr, static_cast<const __nv_bfloat16*>(idx_q), q_req, q_pos, 1, nq,
                                        max_len, fr, qrot, err, st));
  if (s != QSA_OK) return s;
  return run_scorer(cache, cv, q_req, q_pos, 1, nq, max_len, qrot, w, blocks, nblocks, ws, L, err, st);
}

qsa_status qsa_expand_indices(const int32_t* blocks, const int32_t* nblocks, const int32_t* q_pos, int32_t nq,
                              int32_t* pos, int32_t* npos, void* stream) {
  if (nq < 0) return QSA_ERR_INVALID_ARG;
  if (nq == 0) return QSA_OK;
  if (!blocks || !nblocks || !q_pos || !pos || !npos) return QSA_ERR_INVALID_ARG;
  return cuda_status(launch_expand(blocks, nblocks, q_pos, nq, pos, npos, nullptr, static_cast<cudaStream_t>(stream)));
}

qsa_status qsa_sparse_gqa(const qsa_cache* cache, const void* q, const int32_t* q_req, const int32_t* pos,
                          const int32_t* npos, int32_t pos_stride, int32_t max_pos, int32_t nq, float scale,
                          void* out, float* lse, void* ws, size_t ws_bytes, void* stream) {
  qsa_status s = check_cache(cache);
  if (s != QSA_OK) return s;
  if (nq < 0 || pos_stride < 0 || max_pos < 0 || max_pos > pos_stride || !(scale > 0.f) || !std::isfinite(scale))
    return QSA_ERR_INVALID_ARG;
  if (nq == 0) return QSA_OK;
  if (!q || !q_req || !pos || !npos || !out) return QSA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(out, 16) || (lse && !aligned(lse, 4))) return QSA_ERR_INVALID_ARG;
  WsLayout L;
  if (!layout(QSA_OP_SPARSE_GQA, nq, max_pos, L)) return QSA_ERR_INVALID_ARG;
  if ((s = check_ws(ws, ws_bytes, L.total)) != QSA_OK) return s;
  GqaParams p{};
  p.c = view_of(cache);
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.nq_row = 1;
  p.row_req = q_req;
  p.mode = 1;
  p.list = pos;
  p.list_n = npos;
  p.list_stride = pos_stride;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  p.part_o = at<float>(ws, L.part_o);
  p.part_ml = at<float>(ws, L.part_ml);
  p.counters = at<int>(ws, L.cnt_gqa);
  p.splits = std::min(L.splits_bound, gqa_splits_for(nq, max_pos, 1, num_sms()));
  p.err = at<int>(ws, 0);
  return cuda_status(launch_gqa(p, nq, static_cast<cudaStream_t>(stream)));
}

qsa_status qsa_decode(const qsa_cache* cache, const void* idx_k_new, const void* idx_q, const float* w,
                      const void* q, const int32_t* seq_len, int32_t max_len, float scale, void* out, float* lse,
                      int32_t* blocks_out, int32_t* nblocks_out, void* ws, size_t ws_bytes, void* stream) {
  qsa_status s = check_cache(cache);
  if (s != QSA_OK) return s;
  if (max_len < 1 || max_len > QSA_MAX_CONTEXT || !(scale > 0.f) || !std::isfinite(scale))
    return QSA_ERR_INVALID_ARG;
  if ((int64_t)max_len > (int64_t)cache->max_pages * QSA_PAGE_SIZE) return QSA_ERR_INVALID_ARG;
  if ((blocks_out == nullptr) != (nblocks_out == nullptr)) return QSA_ERR_INVALID_ARG;
  const int B = cache->batch;
  if (B == 0) return QSA_OK;
  if (!idx_k_new || !idx_q || !w || !q || !seq_len || !out) return QSA_ERR_INVALID_ARG;
  if (!aligned(idx_k_new, 16) || !aligned(idx_q, 16) || !aligned(q, 16) || !aligned(out, 16) || !aligned(w, 4))
    return QSA_ERR_INVALID_ARG;
  WsLayout L;
  if (!layout(QSA_OP_DECODE, B, max_len, L)) return QSA_ERR_INVALID_ARG;
  if ((s = check_ws(ws, ws_bytes, L.total)) != QSA_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const CacheView cv = view_of(cache);
  const RopeFreqs fr = make_freqs(cache->rope_theta);
  int* err = at<int>(ws, 0);
  __nv_bfloat16* qrot = at<__nv_bfloat16>(ws, L.qrot);
  int32_t* sel = blocks_out ? blocks_out : at<int32_t>(ws, L.sel);
  int32_t* sel_n = nblocks_out ? nblocks_out : at<int32_t>(ws, L.sel_n);
  std::lock_guard<std::mutex> lk(g_prof_mu);
  {
    ProfScope ps(st, 0);
    s = cuda_status(launch_index_prologue(cv, static_cast<const __nv_bfloat16*>(idx_k_new),
                                          static_cast<const __nv_bfloat16*>(idx_q), nullptr, seq_len, 0, B, max_len,
                                          fr, qrot, err, st));
  }
  if (s != QSA_OK) return s;
  {
    ProfScope ps(st, 1);
    s = run_scorer(cache, cv, nullptr, seq_len, 0, B, max_len, qrot, w, sel, sel_n, ws, L, err, st);
  }
  if (s != QSA_OK) return s;
  GqaParams p{};
  p.c = cv;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.nq_row = 1;
  p.mode = 0;
  p.sel = sel;
  p.sel_n = sel_n;
  p.row_len = seq_len;
  p.len_offset = 0;
  p.max_len = max_len;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  p.part_o = at<float>(ws, L.part_o);
  p.part_ml = at<float>(ws, L.part_ml);
  p.counters = at<int>(ws, L.cnt_gqa);
  p.splits = std::min(L.splits_bound, gqa_splits_for(B, positions_bound(QSA_OP_DECODE, max_len), 1, num_sms()));
  p.err = err;
  ProfScope ps(st, 2);
  return cuda_status(launch_gqa(p, B, st));
}

qsa_status qsa_decode_indexshare(const qsa_cache* cache, const int32_t* frozen_pos, const int32_t* frozen_n,
                                 int32_t frozen_stride, const int32_t* len0, int32_t n_plus_1, const void* q,
                                 float scale, void* out, void* ws, size_t ws_bytes, void* stream) {
  qsa_status s = check_cache(cache);
  if (s != QSA_OK) return s;
  if (n_plus_1 < 1 || n_plus_1 > QSA_MAX_DRAFT) return QSA_ERR_UNSUPPORTED;
  if (frozen_stride < 0 || frozen_stride > QSA_MAX_SEL || !(scale > 0.f) || !std::isfinite(scale))
    return QSA_ERR_INVALID_ARG;
  const int B = cache->batch;
  if (B == 0) return QSA_OK;
  if (!frozen_pos || !frozen_n || !len0 || !q || !out) return QSA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(out, 16)) return QSA_ERR_INVALID_ARG;
  WsLayout L;
  if (!layout(QSA_OP_DECODE_INDEXSHARE, B, 1, L)) return QSA_ERR_INVALID_ARG;
  if ((s = check_ws(ws, ws_bytes, L.total)) != QSA_OK) return s;
  GqaParams p{};
  p.c = view_of(cache);
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.nq_row = n_plus_1;
  p.mode = 1;
  p.list = frozen_pos;
  p.list_n = frozen_n;
  p.list_stride = frozen_stride;
  p.extra_base = len0;
  p.n_extra = n_plus_1;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.part_o = at<float>(ws, L.part_o);
  p.part_ml = at<float>(ws, L.part_ml);
  p.counters = at<int>(ws, L.cnt_gqa);
  p.splits = std::min(L.splits_bound,
                      gqa_splits_for(B, positions_bound(QSA_OP_DECODE_INDEXSHARE, 1), n_plus_1, num_sms()));
  p.err = at<int>(ws, 0);
  return cuda_status(launch_gqa(p, B, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
