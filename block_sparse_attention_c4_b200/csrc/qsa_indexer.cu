// Indexer front end of the QSA c4 layer: ring append and block compression,
// index-query rotation, and block -> position expansion.
//
// Blog section "Qwen Sparse Attention: Retrieve Coarsely, Attend Precisely"
// (SGLang day-0 blog for Qwen3.8-Flash-Next): every four raw index keys are
// averaged in FP32, normalised and rotated with the first token's position to
// form one BF16 compressed key; the raw keys of the unfinished block wait in a
// four-slot ring per request; kept blocks expand to 4 positions each plus the
// 0..3 tail tokens.
//
// Numerics (shared with nothing else): the mean is an FP32 sum in token order
// times 0.25; the L2 norm, the division and the RoPE rotation run in FP64 with
// host-computed inverse frequencies; the result is rounded once to bf16.  The
// index query is rotated the same way at its own position and rounded to bf16.
#include "qsa_common.cuh"
#include "qsa_kernels.h"

namespace qsa {

// --------------------------------------------------------------------------
// Bulk append.  grid = (ceil(max_tasks / 4), batch), 128 threads = 4 warps,
// one block task per warp.  Task t of request r compresses block
// b_first + t (b_first = len_before / 4) when that block completes in this
// call; the warp of task 0 is also the only one that touches the ring: it
// reads the ring for the block that straddles len_before, then writes the
// keys of the request's final unfinished block.
// --------------------------------------------------------------------------
__global__ void __launch_bounds__(128) k_compress_append(CacheView c, const __nv_bfloat16* __restrict__ knew,
                                                         const int32_t* __restrict__ cu_new,
                                                         const int32_t* __restrict__ len_before, int total_new,
                                                         RopeFreqs fr, int* err) {
  const int r = blockIdx.y;
  const int task = blockIdx.x * 4 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  const int64_t lb = len_before[r];
  const int64_t c0 = cu_new[r], c1 = cu_new[r + 1];
  if (c0 < 0 || c1 < c0 || c1 > total_new || lb < 0) {
    if (task == 0 && lane == 0) set_error(err, QSA_DEVERR_LENGTH);
    return;
  }
  const int64_t la = lb + (c1 - c0);
  if (la > (int64_t)c.max_pages * PAGE) {
    if (task == 0 && lane == 0) set_error(err, QSA_DEVERR_LENGTH);
    return;
  }
  const int64_t b_first = lb / CBLK;
  const int64_t n_done = la / CBLK - b_first;  // blocks completed by this call
  const int64_t n_tasks = n_done > 0 ? n_done : 1;
  if (task >= n_tasks) return;
  __nv_bfloat16* ring = c.ring + (int64_t)r * CBLK * D;

  if (task < n_done) {
    const int64_t b = b_first + task;
    const __nv_bfloat16* k4[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int64_t pos = CBLK * b + j;
      k4[j] = pos < lb ? ring + (pos % CBLK) * D : knew + (c0 + pos - lb) * D;
    }
    const int64_t e = cidx_entry(c, r, b, err);
    if (e >= 0) warp_compress_block(k4, b, fr, c.cidx + e * D);
  }
  if (task == 0) {
    __syncwarp();
    const int64_t start = max(lb, (la / CBLK) * CBLK);
    for (int64_t pos = start; pos < la; ++pos) {
      const uint32_t* src = reinterpret_cast<const uint32_t*>(knew + (c0 + pos - lb) * D);
      uint32_t* dst = reinterpret_cast<uint32_t*>(ring + (pos % CBLK) * D);
      for (int i = lane; i < D / 2; i += 32) dst[i] = src[i];
    }
  }
}

// --------------------------------------------------------------------------
// Decode prologue / query rotation.  grid = rows, 128 threads.
// If `knew` is non-null (decode): the new index key of position L-1 goes to
// ring slot (L-1) mod 4, and when it completes block b = L/4 - 1 that block is
// compressed from the ring slots 0..2 and the new key.  Always: the 4 index
// query heads are rotated at position L-1 (L = row_len[row] + len_offset) and
// stored as bf16 in qrot [rows][4][128]; row_pages[row] gets the length of the
// row in the scorer's page list: the 64-token pages it streams plus
// SC_ROW_COST empty ones in front (0 when it keeps every block or the row is
// invalid), and the last CTA to finish (atomic ticket) writes their exclusive
// prefix to page_off[0..rows].
// --------------------------------------------------------------------------
__global__ void __launch_bounds__(128) k_index_prologue(CacheView c, const __nv_bfloat16* __restrict__ knew,
                                                        const __nv_bfloat16* __restrict__ idx_q,
                                                        const int32_t* __restrict__ row_req,
                                                        const int32_t* __restrict__ row_len, int len_offset,
                                                        int max_len, int rows, RopeFreqs fr,
                                                        __nv_bfloat16* __restrict__ qrot, int32_t* row_pages,
                                                        int32_t* page_off, int* ticket, int* err) {
  const int row = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5;
  const int req = row_req ? row_req[row] : row;
  const int L = row_len[row] + len_offset;
  const bool valid = req >= 0 && req < c.batch && L >= 1 && L <= max_len;
  __shared__ double cs_s[D / 2], sn_s[D / 2];
  __shared__ int warp_tot[33];
  __shared__ int is_last;
  if (!valid) {
    if (tid == 0) set_error(err, (req < 0 || req >= c.batch) ? QSA_DEVERR_REQUEST : QSA_DEVERR_LENGTH);
  } else {
    const int pos = L - 1;
    if (tid < D / 2) sincos((double)pos * fr.f[tid], &sn_s[tid], &cs_s[tid]);
    if (knew != nullptr && warp == 0) {
      __nv_bfloat16* ring = c.ring + (int64_t)req * CBLK * D;
      const __nv_bfloat16* key = knew + (int64_t)row * D;
      if ((pos & 3) == 3) {
        const __nv_bfloat16* k4[4] = {ring, ring + D, ring + 2 * D, key};
        const int64_t b = pos >> 2;
        const int64_t e = cidx_entry(c, req, b, err);
        if (e >= 0) warp_compress_block(k4, b, fr, c.cidx + e * D);
        __syncwarp();
      }
      const uint32_t* src = reinterpret_cast<const uint32_t*>(key);
      uint32_t* dst = reinterpret_cast<uint32_t*>(ring + (pos & 3) * D);
      for (int i = tid; i < D / 2; i += 32) dst[i] = src[i];
    }
  }
  __syncthreads();
  if (valid) {
    // rotate: thread t handles head t / 32 and pairs i = t % 32, t % 32 + 32
    const int h = tid >> 5, lane = tid & 31;
    const uint16_t* qin = reinterpret_cast<const uint16_t*>(idx_q + ((int64_t)row * HI + h) * D);
    uint16_t* qo = reinterpret_cast<uint16_t*>(qrot + ((int64_t)row * HI + h) * D);
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int i = lane + 32 * e;
      const double x0 = (double)bf16_bits_to_f32(qin[i]);
      const double x1 = (double)bf16_bits_to_f32(qin[i + D / 2]);
      qo[i] = f64_to_bf16_bits(x0 * cs_s[i] - x1 * sn_s[i]);
      qo[i + D / 2] = f64_to_bf16_bits(x0 * sn_s[i] + x1 * cs_s[i]);
    }
  }
  if (row_pages == nullptr) return;
  const int nb = valid ? (L >> 2) : 0;
  if (tid == 0) row_pages[row] = nb > TOPK ? SC_ROW_COST + ceil_div(nb, PAGE_BLOCKS) : 0;
  __threadfence();
  __syncthreads();
  if (tid == 0) is_last = atomicAdd(ticket, 1) == rows - 1;
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  using All = Group<128, 0>;
  int running = 0;
  for (int base = 0; base < rows; base += 128) {
    const int v = base + tid < rows ? __ldcg(row_pages + base + tid) : 0;
    int tot;
    const int ex = group_exclusive_scan<All>(v, warp_tot, &tot);
    if (base + tid < rows) page_off[base + tid] = running + ex;
    running += tot;
  }
  if (tid == 0) {
    page_off[rows] = running;
    *ticket = 0;  // ready for the next call
  }
}

// --------------------------------------------------------------------------
// Expansion: grid = nq, 256 threads.
// --------------------------------------------------------------------------
__global__ void __launch_bounds__(256) k_expand(const int32_t* __restrict__ blocks, const int32_t* __restrict__ nblocks,
                                                const int32_t* __restrict__ q_pos, int32_t* __restrict__ pos,
                                                int32_t* __restrict__ npos, int* err) {
  const int i = blockIdx.x;
  const int L = q_pos[i] + 1;
  int n = nblocks[i];
  const int nb = L >> 2;
  if (n < 0 || n > TOPK || n > nb || L < 1) {
    if (threadIdx.x == 0) set_error(err, QSA_DEVERR_SELECTION);
    n = 0;
  }
  const int tail = L & 3;
  const int total = 4 * n + (L >= 1 ? tail : 0);
  int32_t* out = pos + (int64_t)i * MAX_SEL;
  for (int j = threadIdx.x; j < total; j += blockDim.x)
    out[j] = j < 4 * n ? blocks[(int64_t)i * TOPK + (j >> 2)] * CBLK + (j & 3) : 4 * nb + (j - 4 * n);
  if (threadIdx.x == 0) npos[i] = total;
}

// --------------------------------------------------------------------------
// host launchers
// --------------------------------------------------------------------------
cudaError_t launch_compress_append(const CacheView& c, const __nv_bfloat16* knew, const int32_t* cu_new,
                                   const int32_t* len_before, int total_new, int max_new, const RopeFreqs& fr,
                                   int* err, cudaStream_t st) {
  const int max_tasks = max_new / CBLK + 2;
  dim3 grid(ceil_div(max_tasks, 4), c.batch);
  k_compress_append<<<grid, 128, 0, st>>>(c, knew, cu_new, len_before, total_new, fr, err);
  return cudaGetLastError();
}

cudaError_t launch_index_prologue(const CacheView& c, const __nv_bfloat16* knew, const __nv_bfloat16* idx_q,
                                  const int32_t* row_req, const int32_t* row_len, int len_offset, int rows,
                                  int max_len, const RopeFreqs& fr, __nv_bfloat16* qrot, int32_t* row_pages,
                                  int32_t* page_off, int* ticket, int* err, cudaStream_t st) {
  k_index_prologue<<<rows, 128, 0, st>>>(c, knew, idx_q, row_req, row_len, len_offset, max_len, rows, fr, qrot,
                                         row_pages, page_off, ticket, err);
  return cudaGetLastError();
}

cudaError_t launch_expand(const int32_t* blocks, const int32_t* nblocks, const int32_t* q_pos, int nq, int32_t* pos,
                          int32_t* npos, int* err, cudaStream_t st) {
  k_expand<<<nq, 256, 0, st>>>(blocks, nblocks, q_pos, pos, npos, err);
  return cudaGetLastError();
}

}  // namespace qsa
