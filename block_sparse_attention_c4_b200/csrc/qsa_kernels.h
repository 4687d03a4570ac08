// Internal launch interface between the C-ABI layer (qsa_api.cu) and the
// kernel translation units.  Not part of the public ABI.
#pragma once

#include "qsa_common.cuh"

namespace qsa {

// ---- indexer front end (qsa_indexer.cu) ----
cudaError_t launch_compress_append(const CacheView& c, const __nv_bfloat16* knew, const int32_t* cu_new,
                                   const int32_t* len_before, int total_new, int max_new, const RopeFreqs& fr,
                                   int* err, cudaStream_t st);
cudaError_t launch_index_prologue(const CacheView& c, const __nv_bfloat16* knew, const __nv_bfloat16* idx_q,
                                  const int32_t* row_req, const int32_t* row_len, int len_offset, int rows,
                                  int max_len, const RopeFreqs& fr, __nv_bfloat16* qrot, int* err, cudaStream_t st);
cudaError_t launch_expand(const int32_t* blocks, const int32_t* nblocks, const int32_t* q_pos, int nq, int32_t* pos,
                          int32_t* npos, int* err, cudaStream_t st);

// ---- streaming scorer + top-512 (qsa_score.cu) ----
constexpr int SC_MIN_CHUNK = 1024;  // blocks per CTA, lower bound (workspace sizing)
constexpr int SC_MAX_CHUNK = 4096;  // upper bound (shared memory sizing)

struct ScoreParams {
  CacheView c;
  const int32_t* row_req;  // nullable: row r is request r
  const int32_t* row_len;  // L = row_len[row] + len_offset
  int len_offset;
  int max_len;
  const __nv_bfloat16* qrot;  // [rows][4][128] rotated index queries
  const float* w;             // [rows][4]
  int chunk;                  // blocks per CTA (multiple of 16, SC_MIN_CHUNK..SC_MAX_CHUNK)
  int max_chunks;             // grid.x; candidate buffer stride
  uint32_t* cand_key;         // [rows][max_chunks][512]
  int32_t* cand_id;           // [rows][max_chunks][512]
  int* counters;              // [rows], zero between calls
  int32_t* sel;               // [rows][512] out
  int32_t* sel_n;             // [rows] out
  int* err;
};

int score_chunk_for(int rows, int max_len, int num_sms);
cudaError_t launch_score_topk(const ScoreParams& p, int rows, const CUtensorMap* tmap, cudaStream_t st);

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
  int splits;
  int* err;
};

int gqa_splits_for(int rows, int max_pos, int nq_row, int num_sms);
cudaError_t launch_gqa(const GqaParams& p, int rows, cudaStream_t st);

}  // namespace qsa
