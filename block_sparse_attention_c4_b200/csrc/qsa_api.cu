// C ABI of the QSA c4 layer (declared in include/qsa.h): argument checks,
// workspace carving, TMA descriptors and the launch sequences.  Every step of
// the computation runs in the kernels of qsa_indexer.cu, qsa_score.cu and
// qsa_gqa.cu; this file only marshals arguments.
#include <cmath>
#include <cstdio>
#include <cstring>
#include <algorithm>
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
  size_t cnt_gqa = 0, qrot = 0, sel = 0, sel_n = 0, row_pages = 0, page_off = 0, pages_done = 0, cand_key = 0,
         cand_id = 0, part_o = 0, part_ml = 0, total = 0;
  size_t pf_qbase = 0, pf_cand = 0, pf_cand_n = 0, pf_fb_n = 0, pf_fb_list = 0, pf_fb_keys = 0;
  size_t ready = 0;  // decode: per-row flag, selection final (scorer -> sparse GQA)
  size_t pj_q = 0, pj_k = 0, pj_w = 0;  // decode indexer: projected index queries, keys, head weights
  size_t sp_key = 0, sp_id = 0, sp_n = 0;  // split scoring: per-chunk candidates
  int sp_chunks = 0, sp_chunk = 0;
  int ppc_min = 0;
  int seg_cap = 0;
  int splits_bound = 0;
  int cap = 0;
};

constexpr size_t WS_ERR = 0;     // int: device error word
constexpr size_t WS_TICKET = 64;  // int: prologue arrival ticket

// Scorer range sizing from the longest context: ranges of at least ppc_min
// pages keep the segments of one row at or below seg_cap.  A row of np pages
// meets at most ceil(np / ppc) + 1 ranges, and each range piece is cut every
// SC_MAX_SEG_PAGES pages.
void scorer_sizing(int max_len, int& ppc_min, int& seg_cap) {
  const int np_max = std::max(1, ceil_div(max_len / QSA_BLOCK, PAGE_BLOCKS));
  ppc_min = std::max(SC_MIN_PPC, ceil_div(np_max, 14));
  seg_cap = ceil_div(np_max, ppc_min) + ceil_div(np_max, SC_MAX_SEG_PAGES) + 2;
}


int positions_bound(int op, int max_len) {
  if (op == QSA_OP_SPARSE_GQA) return max_len;
  if (op == QSA_OP_DECODE_INDEXSHARE) return QSA_MAX_SEL + QSA_MAX_DRAFT;
  return std::min(QSA_TOPK * QSA_BLOCK, (max_len / QSA_BLOCK) * QSA_BLOCK) + QSA_BLOCK - 1;
}

// Workspace carving.  Returns false for invalid arguments.
bool layout(int op, int rows, int max_len, WsLayout& w) {
  if (rows < 0 || max_len < 0 || max_len > QSA_MAX_CONTEXT) return false;
  const bool scorer = op == QSA_OP_INDEX_SCORE_TOPK || op == QSA_OP_DECODE || op == QSA_OP_DECODE_INDEXER;
  const bool gqa = op == QSA_OP_SPARSE_GQA || op == QSA_OP_DECODE || op == QSA_OP_DECODE_INDEXSHARE ||
                   op == QSA_OP_DECODE_ATTEND;
  const bool prefill = op == QSA_OP_PREFILL_SCORE_TOPK;
  if (!scorer && !gqa && !prefill && op != QSA_OP_COMPRESS_APPEND && op != QSA_OP_SPLIT_SCORE) return false;
  if (op == QSA_OP_DECODE_ATTEND) op = QSA_OP_DECODE;  // the decode step's attention part
  size_t off = 256;  // error word, prologue ticket, spare
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off += align256(bytes);
    return at;
  };
  if (op == QSA_OP_SPLIT_SCORE) {
    w.sp_chunk = split_chunk(max_len);
    if (w.sp_chunk == 0) return false;
    w.sp_chunks = ceil_div(std::max(1, max_len / QSA_BLOCK), w.sp_chunk);
    w.sp_key = take((size_t)rows * w.sp_chunks * TOPK * 4);
    w.sp_id = take((size_t)rows * w.sp_chunks * TOPK * 4);
    w.sp_n = take((size_t)rows * w.sp_chunks * 4);
    w.total = off;
    return true;
  }
  if (prefill) {
    w.cap = (std::max(1, max_len / QSA_BLOCK) + 31) / 32 * 32;  // blocks of the longest row, whole words
    w.qrot = take((size_t)rows * HI * D * 2);
    w.pf_qbase = take((size_t)rows * 4);
    w.pf_cand = take((size_t)rows * PF_ROW_WORDS * 8);
    w.pf_cand_n = take((size_t)rows * 4 * 4);
    w.pf_fb_n = take(4);
    w.pf_fb_list = take((size_t)rows * 4);
    w.pf_fb_keys = take((size_t)SIZING_SMS * w.cap * 4);
    w.total = off;
    return true;
  }
  w.cnt_gqa = take(sizeof(int) * (size_t)rows);
  if (op == QSA_OP_DECODE) w.ready = take(sizeof(int) * READY_STRIDE * (size_t)rows);
  if (op == QSA_OP_DECODE_INDEXER) {
    w.pj_q = take((size_t)rows * HI * D * 2);
    w.pj_k = take((size_t)rows * D * 2);
    w.pj_w = take((size_t)rows * HI * 4);
  }
  if (scorer) {
    scorer_sizing(max_len, w.ppc_min, w.seg_cap);
    if (w.seg_cap > SC_MAX_SEGS) return false;
    const int np_max = ceil_div(max_len / QSA_BLOCK, PAGE_BLOCKS);
    if ((int64_t)rows * (np_max + SC_ROW_COST) >= (int64_t)INT32_MAX) return false;
    w.qrot = take((size_t)rows * HI * D * 2);
    w.sel = take((size_t)rows * TOPK * 4);
    w.sel_n = take((size_t)rows * 4);
    w.row_pages = take((size_t)rows * 4);
    w.page_off = take((size_t)(rows + 1) * 4);
    w.pages_done = take((size_t)rows * 4);
    w.cand_key = take((size_t)rows * w.seg_cap * TOPK * 4);
    w.cand_id = take((size_t)rows * w.seg_cap * TOPK * 4);
  }
  if (gqa) {
    const int nq_row = op == QSA_OP_DECODE_INDEXSHARE ? QSA_MAX_DRAFT : 1;
    w.splits_bound = gqa_split_bound(rows, positions_bound(op, max_len));
    const size_t heads = (size_t)nq_row * HQ;
    w.part_o = take((size_t)rows * w.splits_bound * heads * D * 4);
    w.part_ml = take((size_t)rows * w.splits_bound * heads * 2 * 4);
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
  const qsa_status s = check_kv_cache(c);
  if (s != QSA_OK) return s;
  if (!c->cidx || !c->ring) return QSA_ERR_INVALID_ARG;
  if (!(c->rope_theta > 0.0) || !std::isfinite(c->rope_theta)) return QSA_ERR_INVALID_ARG;
  if (!aligned(c->cidx, 16) || !aligned(c->ring, 16)) return QSA_ERR_INVALID_ARG;
  return QSA_OK;
}

// FP8 K/V: rows of 128 E4M3 bytes per KV head; kv_stride (bytes) 0 (= 256) or a multiple of 16, at least 256.
qsa_status check_fp8(const qsa_cache* c, float k_scale, float v_scale) {
  if (c->kv_stride != 0 && c->kv_stride % 16 != 0) return QSA_ERR_INVALID_ARG;
  if (!valid_scale(k_scale) || !valid_scale(v_scale)) return QSA_ERR_INVALID_ARG;
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
  v.kv_stride = c->kv_stride ? c->kv_stride : HKV * D;
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

thread_local cudaError_t g_last_cuda_error = cudaSuccess;

qsa_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return QSA_OK;
  g_last_cuda_error = e;
  return QSA_ERR_CUDA;
}

// Prologue (rotation, decode append, page offsets) and scorer, shared by
// qsa_decode and qsa_index_score_topk.
qsa_status run_indexer(const qsa_cache* cache, const CacheView& cv, const __nv_bfloat16* knew,
                       const __nv_bfloat16* idx_q, const int32_t* row_req, const int32_t* row_len, int len_offset,
                       int rows, int max_len, const float* w, int32_t* sel, int32_t* sel_n, void* ws,
                       const WsLayout& L, cudaStream_t st, int* row_ready = nullptr, int ev0 = 0) {
  const RopeFreqs fr = make_freqs(cache->rope_theta);
  int* err = at<int>(ws, WS_ERR);
  __nv_bfloat16* qrot = at<__nv_bfloat16>(ws, L.qrot);
  // Up to SC_ROWS_SMEM rows the scorer runs the front end itself (append, rotation, page prefix);
  // above that a separate prologue kernel does it first.
  const bool fused = rows <= SC_ROWS_SMEM;
  int ev = ev0;
  if (!fused) {
    ProfScope ps(st, ev++);
    cudaError_t e = launch_index_prologue(cv, knew, idx_q, row_req, row_len, len_offset, rows, max_len, fr, qrot,
                                          at<int32_t>(ws, L.row_pages), at<int32_t>(ws, L.page_off),
                                          at<int>(ws, WS_TICKET), err, st);
    if (e != cudaSuccess) return cuda_status(e);
  }
  ScoreParams p;
  p.c = cv;
  p.row_req = row_req;
  p.row_len = row_len;
  p.len_offset = len_offset;
  p.max_len = max_len;
  p.rows = rows;
  p.qrot = qrot;
  p.w = w;
  p.page_off = at<int32_t>(ws, L.page_off);
  p.ppc_min = L.ppc_min;
  p.seg_cap = L.seg_cap;
  p.pages_done = at<int>(ws, L.pages_done);
  p.cand_key = at<uint32_t>(ws, L.cand_key);
  p.cand_id = at<int32_t>(ws, L.cand_id);
  p.sel = sel;
  p.sel_n = sel_n;
  p.err = err;
  p.idx_q = fused ? idx_q : nullptr;
  p.knew = fused ? knew : nullptr;
  p.fr = fr;
  p.row_ready = row_ready;
  ProfScope ps(st, ev);
  return cuda_status(launch_score_topk(p, num_sms(), st));
}

}  // namespace

extern "C" {

const char* qsa_version(void) { return "qsa-b200 0.1 (sm_100a)"; }

const char* qsa_last_error_string(void) {
  return g_last_cuda_error == cudaSuccess ? "no CUDA error" : cudaGetErrorString(g_last_cuda_error);
}

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

int32_t qsa_prefill_rescored_rows(void* ws, int32_t T, int32_t max_len, void* stream) {
  WsLayout L;
  if (!ws || T < 1 || !layout(QSA_OP_PREFILL_SCORE_TOPK, T, max_len, L)) return -1;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int v = 0;
  if (cudaMemcpyAsync(&v, at<int>(ws, L.pf_fb_n), sizeof(int), cudaMemcpyDeviceToHost, st) != cudaSuccess) return -1;
  if (cudaStreamSynchronize(st) != cudaSuccess) return -1;
  return v;
}

qsa_status qsa_prefill_rotated_queries(const void* ws, int32_t T, int32_t max_len, void* out, void* stream) {
  WsLayout L;
  if (!ws || !out || T < 1 || !layout(QSA_OP_PREFILL_SCORE_TOPK, T, max_len, L)) return QSA_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(out, static_cast<const uint8_t*>(ws) + L.qrot, (size_t)T * HI * D * 2, cudaMemcpyDeviceToHost,
                      st) != cudaSuccess)
    return cuda_status(cudaGetLastError());
  return cuda_status(cudaStreamSynchronize(st));
}

int32_t qsa_decode_kernel_count(int32_t batch) { return batch <= SC_ROWS_SMEM ? 2 : 3; }

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
  return run_indexer(cache, view_of(cache), nullptr, static_cast<const __nv_bfloat16*>(idx_q), q_req, q_pos, 1, nq,
                     max_len, w, blocks, nblocks, ws, L, static_cast<cudaStream_t>(stream));
}

qsa_status qsa_prefill_score_topk_varlen(const qsa_cache* cache, const void* idx_q, const float* w, int32_t nseg,
                                         const int32_t* seg_req, const int32_t* seg_pos0, const int32_t* cu_q,
                                         int32_t max_len, int32_t* blocks, int32_t* nblocks, void* ws,
                                         size_t ws_bytes, void* stream) {
  qsa_status s = check_cache(cache);
  if (s != QSA_OK) return s;
  if (nseg < 0 || nseg > PF_MAX_SEGS) return nseg < 0 ? QSA_ERR_INVALID_ARG : QSA_ERR_UNSUPPORTED;
  if (nseg == 0) return QSA_OK;
  if (!seg_req || !seg_pos0 || !cu_q || cu_q[0] != 0) return QSA_ERR_INVALID_ARG;
  if (max_len < 1 || max_len > QSA_MAX_CONTEXT || (int64_t)max_len > (int64_t)cache->max_pages * QSA_PAGE_SIZE)
    return QSA_ERR_INVALID_ARG;
  PrefillParams p{};
  int order[PF_MAX_SEGS], n_live = 0;
  for (int i = 0; i < nseg; ++i) {
    const int T = cu_q[i + 1] - cu_q[i];
    if (T < 0 || seg_pos0[i] < 0 || (int64_t)seg_pos0[i] + T > max_len) return QSA_ERR_INVALID_ARG;
    if (seg_req[i] < 0 || seg_req[i] >= cache->batch) return QSA_ERR_INVALID_ARG;
    if (T > 0) order[n_live++] = i;
  }
  const int total = cu_q[nseg];
  if (n_live == 0) return QSA_OK;
  if (!idx_q || !w || !blocks || !nblocks) return QSA_ERR_INVALID_ARG;
  if (!aligned(idx_q, 16) || !aligned(w, 16)) return QSA_ERR_INVALID_ARG;
  // longest contexts first: their tiles are the most expensive, so they start first
  std::stable_sort(order, order + n_live, [&](int a, int b) {
    return (int64_t)seg_pos0[a] + (cu_q[a + 1] - cu_q[a]) > (int64_t)seg_pos0[b] + (cu_q[b + 1] - cu_q[b]);
  });
  int tiles = 0, rows = 0;
  for (int k = 0; k < n_live; ++k) {
    const int i = order[k];
    PfSeg& sg = p.seg[k];
    sg.req = seg_req[i];
    sg.pos0 = seg_pos0[i];
    sg.T = cu_q[i + 1] - cu_q[i];
    sg.q_off = cu_q[i];
    sg.tile_off = tiles;
    sg.row_off = rows;
    tiles += ceil_div(sg.T, 64);
    rows += sg.T;
  }
  WsLayout L;
  if (!layout(QSA_OP_PREFILL_SCORE_TOPK, total, max_len, L)) return QSA_ERR_INVALID_ARG;
  if ((s = check_ws(ws, ws_bytes, L.total)) != QSA_OK) return s;
  p.c = view_of(cache);
  p.nseg = n_live;
  p.T = total;
  p.ntiles = tiles;
  p.w = w;
  p.qrot = at<__nv_bfloat16>(ws, L.qrot);
  p.qbase = at<int32_t>(ws, L.pf_qbase);
  p.cand = at<unsigned long long>(ws, L.pf_cand);
  p.cand_n = at<int32_t>(ws, L.pf_cand_n);
  p.fb_n = at<int>(ws, L.pf_fb_n);
  p.fb_list = at<int32_t>(ws, L.pf_fb_list);
  p.fb_keys = at<uint32_t>(ws, L.pf_fb_keys);
  p.fb_cap = L.cap;
  p.fb_ctas = std::min(num_sms(), SIZING_SMS);
  p.wait_ns = 0;
  p.stats = nullptr;
  p.sel = blocks;
  p.sel_n = nblocks;
  p.err = at<int>(ws, WS_ERR);
  std::lock_guard<std::mutex> lk(g_prof_mu);
  return cuda_status(launch_prefill(p, static_cast<const __nv_bfloat16*>(idx_q), make_freqs(cache->rope_theta),
                                    num_sms(), static_cast<cudaStream_t>(stream), g_prof_pairs ? g_prof : nullptr,
                                    g_prof_pairs));
}

qsa_status qsa_prefill_score_topk(const qsa_cache* cache, const void* idx_q, const float* w, int32_t req,
                                  int32_t pos0, int32_t T, int32_t* blocks, int32_t* nblocks, void* ws,
                                  size_t ws_bytes, void* stream) {
  if (T < 0 || pos0 < 0 || (int64_t)pos0 + T > QSA_MAX_CONTEXT) return QSA_ERR_INVALID_ARG;
  if (T == 0) return check_cache(cache);
  const int32_t cu[2] = {0, T};
  return qsa_prefill_score_topk_varlen(cache, idx_q, w, 1, &req, &pos0, cu, pos0 + T, blocks, nblocks, ws, ws_bytes,
                                       stream);
}

qsa_status qsa_expand_indices(const int32_t* blocks, const int32_t* nblocks, const int32_t* q_pos, int32_t nq,
                              int32_t* pos, int32_t* npos, void* stream) {
  if (nq < 0) return QSA_ERR_INVALID_ARG;
  if (nq == 0) return QSA_OK;
  if (!blocks || !nblocks || !q_pos || !pos || !npos) return QSA_ERR_INVALID_ARG;
  return cuda_status(launch_expand(blocks, nblocks, q_pos, nq, pos, npos, nullptr, static_cast<cudaStream_t>(stream)));
}

}  // extern "C" (reopened below)

static qsa_status sparse_gqa_impl(const qsa_cache* cache, const void* q, const int32_t* q_req, const int32_t* pos,
                                  const int32_t* npos, int32_t pos_stride, int32_t max_pos, int32_t nq, float scale,
                                  void* out, float* lse, void* ws, size_t ws_bytes, void* stream, int fp8,
                                  float k_scale, float v_scale) {
  qsa_status s = check_cache(cache);
  if (s != QSA_OK) return s;
  if (nq < 0 || pos_stride < 0 || max_pos < 0 || max_pos > pos_stride || !valid_scale(scale))
    return QSA_ERR_INVALID_ARG;
  if (max_pos > QSA_MAX_SEL) return QSA_ERR_UNSUPPORTED;
  if (nq == 0) return QSA_OK;
  if (!q || !q_req || !pos || !npos || !out) return QSA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(out, 16) || (lse && !aligned(lse, 4))) return QSA_ERR_INVALID_ARG;
  WsLayout L;
  if (!layout(QSA_OP_SPARSE_GQA, nq, max_pos, L)) return QSA_ERR_INVALID_ARG;
  if ((s = check_ws(ws, ws_bytes, L.total)) != QSA_OK) return s;
  GqaParams p{};
  p.cluster_merge = 1;
  p.c = view_of(cache);
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.nq_row = 1;
  p.row_req = q_req;
  p.mode = 1;
  p.list = pos;
  p.list_n = npos;
  p.list_stride = pos_stride;
  p.scale_log2 = scale * k_scale * 1.4426950408889634f;
  p.fp8 = fp8;
  p.v_scale = v_scale;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  p.part_o = at<float>(ws, L.part_o);
  p.part_ml = at<float>(ws, L.part_ml);
  p.counters = at<int>(ws, L.cnt_gqa);
  p.err = at<int>(ws, WS_ERR);
  return cuda_status(launch_gqa(p, nq, max_pos, num_sms(), L.splits_bound, static_cast<cudaStream_t>(stream)));
}

static qsa_status decode_impl(const qsa_cache* cache, const void* idx_k_new, const void* idx_q, const float* w,
                              const void* q, const int32_t* seq_len, int32_t max_len, float scale, void* out,
                              float* lse, int32_t* blocks_out, int32_t* nblocks_out, void* ws, size_t ws_bytes,
                              void* stream, int fp8, float k_scale, float v_scale) {
  qsa_status s = check_cache(cache);
  if (s != QSA_OK) return s;
  if (max_len < 1 || max_len > QSA_MAX_CONTEXT || !valid_scale(scale))
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
  int* err = at<int>(ws, WS_ERR);
  int32_t* sel = blocks_out ? blocks_out : at<int32_t>(ws, L.sel);
  int32_t* sel_n = nblocks_out ? nblocks_out : at<int32_t>(ws, L.sel_n);
  std::lock_guard<std::mutex> lk(g_prof_mu);
  // The sparse GQA is launched as a programmatic dependent of the scorer: it starts on the SMs the
  // scorer frees and waits per row for the row's ready flag, overlapping the scorer's last merges.
  int* ready = at<int>(ws, L.ready);
  s = run_indexer(cache, cv, static_cast<const __nv_bfloat16*>(idx_k_new), static_cast<const __nv_bfloat16*>(idx_q),
                  nullptr, seq_len, 0, B, max_len, w, sel, sel_n, ws, L, st, ready);
  if (s != QSA_OK) return s;
  GqaParams p{};
  p.cluster_merge = 1;
  p.c = cv;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.nq_row = 1;
  p.mode = 0;
  p.sel = sel;
  p.sel_n = sel_n;
  p.row_len = seq_len;
  p.len_offset = 0;
  p.max_len = max_len;
  p.scale_log2 = scale * k_scale * 1.4426950408889634f;
  p.fp8 = fp8;
  p.v_scale = v_scale;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  p.part_o = at<float>(ws, L.part_o);
  p.part_ml = at<float>(ws, L.part_ml);
  p.counters = at<int>(ws, L.cnt_gqa);
  p.err = err;
  p.row_ready = ready;
  ProfScope ps(st, qsa_decode_kernel_count(B) - 1);
  return cuda_status(launch_gqa(p, B, positions_bound(QSA_OP_DECODE, max_len), num_sms(), L.splits_bound, st));
}

extern "C" {

qsa_status qsa_sparse_gqa(const qsa_cache* cache, const void* q, const int32_t* q_req, const int32_t* pos,
                          const int32_t* npos, int32_t pos_stride, int32_t max_pos, int32_t nq, float scale,
                          void* out, float* lse, void* ws, size_t ws_bytes, void* stream) {
  return sparse_gqa_impl(cache, q, q_req, pos, npos, pos_stride, max_pos, nq, scale, out, lse, ws, ws_bytes, stream,
                         0, 1.f, 1.f);
}

qsa_status qsa_sparse_gqa_fp8(const qsa_cache* cache, float k_scale, float v_scale, const void* q,
                              const int32_t* q_req, const int32_t* pos, const int32_t* npos, int32_t pos_stride,
                              int32_t max_pos, int32_t nq, float scale, void* out, float* lse, void* ws,
                              size_t ws_bytes, void* stream) {
  if (!cache) return QSA_ERR_INVALID_ARG;
  const qsa_status s = check_fp8(cache, k_scale, v_scale);
  if (s != QSA_OK) return s;
  return sparse_gqa_impl(cache, q, q_req, pos, npos, pos_stride, max_pos, nq, scale, out, lse, ws, ws_bytes, stream,
                         1, k_scale, v_scale);
}

qsa_status qsa_decode(const qsa_cache* cache, const void* idx_k_new, const void* idx_q, const float* w,
                      const void* q, const int32_t* seq_len, int32_t max_len, float scale, void* out, float* lse,
                      int32_t* blocks_out, int32_t* nblocks_out, void* ws, size_t ws_bytes, void* stream) {
  return decode_impl(cache, idx_k_new, idx_q, w, q, seq_len, max_len, scale, out, lse, blocks_out, nblocks_out, ws,
                     ws_bytes, stream, 0, 1.f, 1.f);
}

qsa_status qsa_decode_fp8(const qsa_cache* cache, float k_scale, float v_scale, const void* idx_k_new,
                          const void* idx_q, const float* w, const void* q, const int32_t* seq_len, int32_t max_len,
                          float scale, void* out, float* lse, int32_t* blocks_out, int32_t* nblocks_out, void* ws,
                          size_t ws_bytes, void* stream) {
  if (!cache) return QSA_ERR_INVALID_ARG;
  const qsa_status s = check_fp8(cache, k_scale, v_scale);
  if (s != QSA_OK) return s;
  return decode_impl(cache, idx_k_new, idx_q, w, q, seq_len, max_len, scale, out, lse, blocks_out, nblocks_out, ws,
                     ws_bytes, stream, 1, k_scale, v_scale);
}

qsa_status qsa_index_project(const void* x, const void* w_proj, int32_t n, int32_t hidden, void* idx_q, void* idx_k,
                             float* w, void* stream) {
  if (n < 0 || hidden < QSA_HEAD_DIM || hidden > QSA_MAX_HIDDEN || hidden % QSA_HEAD_DIM != 0)
    return QSA_ERR_INVALID_ARG;
  if (n == 0) return QSA_OK;
  if (!x || !w_proj || !idx_q || !idx_k || !w) return QSA_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(w_proj, 16) || !aligned(idx_q, 2) || !aligned(idx_k, 2) || !aligned(w, 4))
    return QSA_ERR_INVALID_ARG;
  ProjParams p;
  p.x = static_cast<const __nv_bfloat16*>(x);
  p.w = static_cast<const __nv_bfloat16*>(w_proj);
  p.n = n;
  p.hidden = hidden;
  p.idx_q = static_cast<__nv_bfloat16*>(idx_q);
  p.idx_k = static_cast<__nv_bfloat16*>(idx_k);
  p.wout = w;
  return cuda_status(launch_index_proj(p, static_cast<cudaStream_t>(stream)));
}

qsa_status qsa_decode_indexer(const qsa_cache* cache, const void* x, const void* w_proj, int32_t hidden,
                              const int32_t* seq_len, int32_t max_len, int32_t* blocks, int32_t* nblocks, void* ws,
                              size_t ws_bytes, void* stream) {
  qsa_status s = check_cache(cache);
  if (s != QSA_OK) return s;
  if (max_len < 1 || max_len > QSA_MAX_CONTEXT) return QSA_ERR_INVALID_ARG;
  if ((int64_t)max_len > (int64_t)cache->max_pages * QSA_PAGE_SIZE) return QSA_ERR_INVALID_ARG;
  if (hidden < QSA_HEAD_DIM || hidden > QSA_MAX_HIDDEN || hidden % QSA_HEAD_DIM != 0) return QSA_ERR_INVALID_ARG;
  const int B = cache->batch;
  if (B == 0) return QSA_OK;
  if (!x || !w_proj || !seq_len || !blocks || !nblocks) return QSA_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(w_proj, 16)) return QSA_ERR_INVALID_ARG;
  WsLayout L;
  if (!layout(QSA_OP_DECODE_INDEXER, B, max_len, L)) return QSA_ERR_INVALID_ARG;
  if ((s = check_ws(ws, ws_bytes, L.total)) != QSA_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  ProjParams pj;
  pj.x = static_cast<const __nv_bfloat16*>(x);
  pj.w = static_cast<const __nv_bfloat16*>(w_proj);
  pj.n = B;
  pj.hidden = hidden;
  pj.idx_q = at<__nv_bfloat16>(ws, L.pj_q);
  pj.idx_k = at<__nv_bfloat16>(ws, L.pj_k);
  pj.wout = at<float>(ws, L.pj_w);
  std::lock_guard<std::mutex> lk(g_prof_mu);
  {
    ProfScope ps(st, 0);
    cudaError_t e = launch_index_proj(pj, st);
    if (e != cudaSuccess) return cuda_status(e);
  }
  // the projected key, queries and weights feed the same front end and scorer as qsa_decode
  return run_indexer(cache, view_of(cache), pj.idx_k, pj.idx_q, nullptr, seq_len, 0, B, max_len, pj.wout, blocks,
                     nblocks, ws, L, st, nullptr, 1);
}

qsa_status qsa_decode_attend(const qsa_cache* cache, const void* q, const int32_t* seq_len, int32_t max_len,
                             const int32_t* blocks, const int32_t* nblocks, float scale, void* out, float* lse,
                             void* ws, size_t ws_bytes, void* stream) {
  qsa_status s = check_kv_cache(cache);
  if (s != QSA_OK) return s;
  if (max_len < 1 || max_len > QSA_MAX_CONTEXT || !valid_scale(scale)) return QSA_ERR_INVALID_ARG;
  if ((int64_t)max_len > (int64_t)cache->max_pages * QSA_PAGE_SIZE) return QSA_ERR_INVALID_ARG;
  const int B = cache->batch;
  if (B == 0) return QSA_OK;
  if (!q || !seq_len || !blocks || !nblocks || !out) return QSA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(out, 16) || (lse && !aligned(lse, 4))) return QSA_ERR_INVALID_ARG;
  WsLayout L;
  if (!layout(QSA_OP_DECODE_ATTEND, B, max_len, L)) return QSA_ERR_INVALID_ARG;
  if ((s = check_ws(ws, ws_bytes, L.total)) != QSA_OK) return s;
  GqaParams p{};
  p.cluster_merge = 1;
  p.c = view_of(cache);
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.nq_row = 1;
  p.mode = 0;
  p.sel = blocks;
  p.sel_n = nblocks;
  p.row_len = seq_len;
  p.len_offset = 0;
  p.max_len = max_len;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  p.part_o = at<float>(ws, L.part_o);
  p.part_ml = at<float>(ws, L.part_ml);
  p.counters = at<int>(ws, L.cnt_gqa);
  p.err = at<int>(ws, WS_ERR);
  return cuda_status(launch_gqa(p, B, positions_bound(QSA_OP_DECODE, max_len), num_sms(), L.splits_bound,
                                static_cast<cudaStream_t>(stream)));
}

qsa_status qsa_split_score_topk(const qsa_cache* cache, const void* idx_q, const float* w, const int32_t* seq_len,
                                const int32_t* page_lo, const int32_t* page_cnt, int32_t max_len, uint32_t* cand_key,
                                int32_t* cand_id, int32_t* cand_n, void* ws, size_t ws_bytes, void* stream) {
  qsa_status s = check_cache(cache);
  if (s != QSA_OK) return s;
  if (max_len < 1 || max_len > QSA_MAX_CONTEXT) return QSA_ERR_INVALID_ARG;
  const int B = cache->batch;
  if (B == 0) return QSA_OK;
  if (!idx_q || !w || !seq_len || !page_lo || !page_cnt || !cand_key || !cand_id || !cand_n) return QSA_ERR_INVALID_ARG;
  if (!aligned(idx_q, 16) || !aligned(w, 4)) return QSA_ERR_INVALID_ARG;
  WsLayout L;
  if (!layout(QSA_OP_SPLIT_SCORE, B, max_len, L)) return QSA_ERR_INVALID_ARG;
  if ((s = check_ws(ws, ws_bytes, L.total)) != QSA_OK) return s;
  SplitParams p{};
  p.c = view_of(cache);
  p.idx_q = static_cast<const __nv_bfloat16*>(idx_q);
  p.w = w;
  p.seq_len = seq_len;
  p.page_lo = page_lo;
  p.page_cnt = page_cnt;
  p.max_len = max_len;
  p.fr = make_freqs(cache->rope_theta);
  p.chunk = L.sp_chunk;
  p.nchunks = L.sp_chunks;
  p.cand_key = at<uint32_t>(ws, L.sp_key);
  p.cand_id = at<int32_t>(ws, L.sp_id);
  p.cand_n = at<int32_t>(ws, L.sp_n);
  p.out_key = cand_key;
  p.out_id = cand_id;
  p.out_n = cand_n;
  p.err = at<int>(ws, WS_ERR);
  return cuda_status(launch_split_score(p, B, static_cast<cudaStream_t>(stream)));
}

qsa_status qsa_split_merge(const uint32_t* cand_key, const int32_t* cand_id, const int32_t* cand_n, int32_t world,
                           int32_t rows, int32_t* blocks, int32_t* nblocks, void* stream) {
  if (world < 1 || world > SPLIT_MAX_LISTS || rows < 0) return world > SPLIT_MAX_LISTS ? QSA_ERR_UNSUPPORTED
                                                                                       : QSA_ERR_INVALID_ARG;
  if (rows == 0) return QSA_OK;
  if (!cand_key || !cand_id || !cand_n || !blocks || !nblocks) return QSA_ERR_INVALID_ARG;
  return cuda_status(launch_split_merge(cand_key, cand_id, cand_n, world, rows, blocks, nblocks,
                                        static_cast<cudaStream_t>(stream)));
}

qsa_status qsa_split_positions(const int32_t* seq_len, const int32_t* page_lo, const int32_t* page_cnt,
                               const int32_t* blocks, const int32_t* nblocks, int32_t rows, int32_t* pos,
                               int32_t* npos, void* stream) {
  if (rows < 0) return QSA_ERR_INVALID_ARG;
  if (rows == 0) return QSA_OK;
  if (!seq_len || !page_lo || !page_cnt || !blocks || !nblocks || !pos || !npos) return QSA_ERR_INVALID_ARG;
  SplitParams p{};
  p.seq_len = seq_len;
  p.page_lo = page_lo;
  p.page_cnt = page_cnt;
  return cuda_status(launch_split_positions(p, blocks, nblocks, rows, pos, npos, static_cast<cudaStream_t>(stream)));
}

qsa_status qsa_split_combine(const void* outs, const float* lses, int32_t world, int32_t rows, void* out,
                             void* stream) {
  if (world < 1 || rows < 0) return QSA_ERR_INVALID_ARG;
  if (rows == 0) return QSA_OK;
  if (!outs || !lses || !out || !aligned(outs, 8) || !aligned(out, 8)) return QSA_ERR_INVALID_ARG;
  return cuda_status(launch_split_combine(static_cast<const __nv_bfloat16*>(outs), lses, world, rows,
                                          static_cast<__nv_bfloat16*>(out), static_cast<cudaStream_t>(stream)));
}

qsa_status qsa_check_bounded_wait(const qsa_cache* cache, const void* q, void* out, uint64_t limit_ns, void* ws,
                                  size_t ws_bytes, void* stream) {
  qsa_status s = check_cache(cache);
  if (s != QSA_OK) return s;
  if (cache->batch < 1 || !q || !out || limit_ns < 1 || limit_ns > WAIT_LIMIT_NS) return QSA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(out, 16)) return QSA_ERR_INVALID_ARG;
  WsLayout L;
  if (!layout(QSA_OP_DECODE, 1, 8, L)) return QSA_ERR_INVALID_ARG;
  if ((s = check_ws(ws, ws_bytes, L.total)) != QSA_OK) return s;
  // The decode attention of one row, launched exactly as qsa_decode launches it, but with no scorer
  // before it: the row's ready flag (zeroed workspace) is never set.  Its length and selection are
  // read from the zeroed workspace too, and only after the wait, which gives up first.
  GqaParams p{};
  p.cluster_merge = 1;
  p.c = view_of(cache);
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.nq_row = 1;
  p.mode = 0;
  p.sel = at<int32_t>(ws, L.sel);
  p.sel_n = at<int32_t>(ws, L.sel_n);
  p.row_len = at<int32_t>(ws, L.sel_n);
  p.len_offset = 0;
  p.max_len = 8;
  p.scale_log2 = 1.f;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.part_o = at<float>(ws, L.part_o);
  p.part_ml = at<float>(ws, L.part_ml);
  p.counters = at<int>(ws, L.cnt_gqa);
  p.err = at<int>(ws, WS_ERR);
  p.row_ready = at<int>(ws, L.ready);
  p.wait_ns = limit_ns;
  return cuda_status(launch_gqa(p, 1, positions_bound(QSA_OP_DECODE, 8), num_sms(), L.splits_bound,
                                static_cast<cudaStream_t>(stream)));
}

qsa_status qsa_decode_indexshare(const qsa_cache* cache, const int32_t* frozen_pos, const int32_t* frozen_n,
                                 int32_t frozen_stride, const int32_t* len0, int32_t n_plus_1, const void* q,
                                 float scale, void* out, void* ws, size_t ws_bytes, void* stream) {
  qsa_status s = check_cache(cache);
  if (s != QSA_OK) return s;
  if (n_plus_1 < 1 || n_plus_1 > QSA_MAX_DRAFT) return QSA_ERR_UNSUPPORTED;
  if (frozen_stride < 0 || frozen_stride > QSA_MAX_SEL || !valid_scale(scale))
    return QSA_ERR_INVALID_ARG;
  const int B = cache->batch;
  if (B == 0) return QSA_OK;
  if (!frozen_pos || !frozen_n || !len0 || !q || !out) return QSA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(out, 16)) return QSA_ERR_INVALID_ARG;
  WsLayout L;
  if (!layout(QSA_OP_DECODE_INDEXSHARE, B, 1, L)) return QSA_ERR_INVALID_ARG;
  if ((s = check_ws(ws, ws_bytes, L.total)) != QSA_OK) return s;
  GqaParams p{};
  p.cluster_merge = 1;
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
  p.err = at<int>(ws, WS_ERR);
  return cuda_status(launch_gqa(p, B, frozen_stride + n_plus_1, num_sms(), L.splits_bound,
                                static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
