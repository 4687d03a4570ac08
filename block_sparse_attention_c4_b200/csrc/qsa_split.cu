// Split-context decode: one request's context divided over several GPUs by page ranges.
//
// The QSA layer's decode (blog section "Qwen Sparse Attention: Retrieve Coarsely, Attend
// Precisely", SGLang day-0 blog for Qwen3.8-Flash-Next) scores every complete block and attends to
// the best 512 plus the tail.  Split over ranks, each rank holds the pages [page_lo, page_lo +
// page_cnt) of a request: its K/V and compressed index keys live in a cache of the rank's own whose
// page-table row is indexed by the request's (global) logical page and maps only those pages, so
// positions and blocks keep their global numbers everywhere (the compressed keys are appended at
// their global positions by qsa_compress_append on the owning rank, hence rotated correctly).
// A step is:
//   (1) qsa_split_score_topk: score the rank's complete blocks (the index query rotated at the
//       request's global position) and keep its best 512 with their score keys;
//   (2) exchange: all ranks' candidates, concatenated in rank order (an all-gather);
//   (3) qsa_split_merge: the best 512 of the concatenation.  Every block of the global top 512 is
//       in its owner's top 512, and rank order is block order, so this is the exact top 512 with
//       ties to the lower block, identical on every rank;
//   (4) qsa_split_positions + qsa_sparse_gqa (with LSE): attention over the kept positions the
//       rank holds, plus the tail if it holds the request's last position;
//   (5) exchange of (output, LSE) and qsa_split_combine: the LSE-weighted mean of the ranks'
//       outputs, which is the attention over all kept positions.
// The pages describe no such split; the reading is the plainest exact one.
#include "qsa_common.cuh"
#include "qsa_kernels.h"

namespace qsa {

constexpr int SP_WARPS = 16;
constexpr int SP_THREADS = SP_WARPS * 32;
constexpr int SP_CHUNK = SPLIT_CHUNK_BLOCKS;          // most blocks a CTA scores (512 pages)
using SpCta = Group<SP_THREADS, 0>;

struct SpSmem {
  uint32_t keys[SP_CHUNK];
  int32_t pid[SP_CHUNK / PAGE_BLOCKS];  // physical pages of the chunk
  alignas(16) uint32_t hist[HT_WORDS];
  HistTopScratch ht;
  double cs[D / 2], sn[D / 2];
  uint32_t qraw[HI * D / 2];
};
static_assert(SP_CHUNK <= HT_MAX_N && SP_CHUNK <= 32 * SP_THREADS, "a chunk's keys fit one selection");

// The complete blocks of row r held by this rank: [b_lo, b_hi) (global block numbers); the rotation
// position is the request's last position L - 1.
struct SpRow {
  int L, b_lo, b_hi;
};
__device__ __forceinline__ SpRow sp_row(const SplitParams& p, int r) {
  SpRow g;
  g.L = __ldg(p.seq_len + r);
  const int lo = __ldg(p.page_lo + r), cnt = __ldg(p.page_cnt + r);
  g.b_lo = lo * PAGE_BLOCKS;
  g.b_hi = max(g.b_lo, min((lo + cnt) * PAGE_BLOCKS, g.L >> 2));
  return g;
}

// grid = (chunks, rows): chunk c of row r scores the rank's blocks [b_lo + c * chunk, ...) and writes
// its best min(512, n) (key, block) to slot c of the row's candidate list, in block order.
__global__ void __launch_bounds__(SP_THREADS) k_split_score(SplitParams p) {
  extern __shared__ uint8_t smem_raw[];
  SpSmem& S = *reinterpret_cast<SpSmem*>(smem_aligned<128>(smem_raw));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int r = blockIdx.y, c = blockIdx.x;
  const SpRow g = sp_row(p, r);
  const int b0 = g.b_lo + c * p.chunk;
  const int n = min(p.chunk, g.b_hi - b0);
  int* slot_n = p.cand_n + (int64_t)r * p.nchunks + c;
  if (g.L < 1 || g.L > p.max_len || __ldg(p.page_lo + r) < 0 || __ldg(p.page_cnt + r) < 0) {
    if (tid == 0) {
      set_error(p.err, QSA_DEVERR_LENGTH);
      *slot_n = 0;
    }
    return;
  }
  if (n <= 0) {
    if (tid == 0) *slot_n = 0;
    return;
  }
  // the index query rotated at L - 1 (FP64 angles, one bf16 rounding), as the decode scorer does
  if (tid < HI * D / 2) S.qraw[tid] = __ldg(reinterpret_cast<const uint32_t*>(p.idx_q + (int64_t)r * HI * D) + tid);
  if (tid < D / 2) sincos((double)(g.L - 1) * p.fr.f[tid], &S.sn[tid], &S.cs[tid]);
  ht_zero<SpCta>(S.hist);
  __syncthreads();
  {
    const int h = tid >> 6, i = tid & 63;
    uint16_t y0 = 0, y1 = 0;
    if (tid < HI * D / 2) {
      const uint16_t* q16 = reinterpret_cast<const uint16_t*>(S.qraw) + h * D;
      const double x0 = (double)bf16_bits_to_f32(q16[i]);
      const double x1 = (double)bf16_bits_to_f32(q16[i + D / 2]);
      y0 = f64_to_bf16_bits(x0 * S.cs[i] - x1 * S.sn[i]);
      y1 = f64_to_bf16_bits(x0 * S.sn[i] + x1 * S.cs[i]);
    }
    __syncthreads();
    if (tid < HI * D / 2) {
      uint16_t* o16 = reinterpret_cast<uint16_t*>(S.qraw) + h * D;
      o16[i] = y0;
      o16[i + D / 2] = y1;
    }
    __syncthreads();
  }
  const int g8 = lane >> 2, cq = lane & 3;
  uint32_t bq[8][2];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int d0 = 8 * (cq + 4 * (j >> 1)) + 4 * (j & 1);
    bq[j][0] = g8 < HI ? S.qraw[(g8 * D + d0) >> 1] : 0u;
    bq[j][1] = g8 < HI ? S.qraw[(g8 * D + d0 + 2) >> 1] : 0u;
  }
  const float wa = cq < 2 ? __ldg(p.w + (int64_t)r * HI + 2 * cq) : 0.f;
  const float wb = cq < 2 ? __ldg(p.w + (int64_t)r * HI + 2 * cq + 1) : 0.f;
  const int32_t* pt = p.c.page_table + (int64_t)r * p.c.max_pages;
  const uint4* cidx = reinterpret_cast<const uint4*>(p.c.cidx);
  const int np = ceil_div(n, PAGE_BLOCKS), lp0 = b0 / PAGE_BLOCKS;
  // the chunk's physical pages, looked up together (-1: outside the table or the pool, flagged)
  for (int k = tid; k < np; k += SP_THREADS) {
    const int lp = lp0 + k;
    int phys = lp < p.c.max_pages ? __ldg(pt + lp) : -1;
    if (phys < 0 || phys >= p.c.num_pages) {
      set_error(p.err, QSA_DEVERR_PAGE);
      phys = -1;
    }
    S.pid[k] = phys;
  }
  __syncthreads();
  // each warp scores its pages two at a time (both loads in flight before either is used)
  auto finish = [&](int k, const PageRegs& pr, bool ok) {
    float lo = 0.f, hi = 0.f;
    if (ok) score_page(pr, bq, wa, wb, lo, hi);
    if (cq < 2) {
      const int local = k * PAGE_BLOCKS + g8 + 8 * cq;
      if (local < n) {
        const uint32_t key = score_key(cq ? hi : lo);
        S.keys[local] = key;
        ht_count(S.hist, key);
      }
    }
  };
  for (int k = warp; k < np; k += 2 * SP_WARPS) {
    const int k2 = k + SP_WARPS;
    const int ph1 = S.pid[k], ph2 = k2 < np ? S.pid[k2] : -1;
    PageRegs pr1, pr2;
    if (ph1 >= 0) load_page(pr1, cidx + (int64_t)ph1 * (PAGE_BLOCKS * D / 8), g8, cq);
    if (ph2 >= 0) load_page(pr2, cidx + (int64_t)ph2 * (PAGE_BLOCKS * D / 8), g8, cq);
    finish(k, pr1, ph1 >= 0);
    if (k2 < np) finish(k2, pr2, ph2 >= 0);
  }
  __syncthreads();
  const int k_keep = min(TOPK, n);
  uint32_t* ck = p.cand_key + ((int64_t)r * p.nchunks + c) * TOPK;
  int32_t* ci = p.cand_id + ((int64_t)r * p.nchunks + c) * TOPK;
  hist_topk<SpCta>(S.keys, S.hist, n, k_keep, [&](int i, int o) {
    ck[o] = S.keys[i];
    ci[o] = b0 + i;
  }, &S.ht);
  if (tid == 0) *slot_n = k_keep;
}

// Best min(512, total) of `lists` ordered lists of (key, id) candidates, emitted in list order (the
// lists are in block order end to end, so the output is ascending and ties keep the lower block).
// One CTA per row; list j of row r holds n[j] entries at keys/ids + (r * lists + j) * 512 when
// row_major, else at + (j * rows + r) * 512 (the ranks' exchanged arrays).  The row's keys are first
// packed end to end into shared memory (all of a thread's loads in flight at once), so the selection's
// passes read shared memory; only the <= 512 emitted entries look their list up again (binary search).
struct MergeArgs {
  const uint32_t* keys;
  const int32_t* ids;
  const int32_t* n;
  int lists, rows, row_major;
  uint32_t* out_key;  // nullable [rows][512]
  int32_t* out_id;    // [rows][512]
  int32_t* out_n;     // [rows]
};
constexpr int SM_THREADS = 512;
inline size_t split_merge_smem(int lists) { return (size_t)lists * TOPK * sizeof(uint32_t); }

__global__ void __launch_bounds__(SM_THREADS) k_split_merge(MergeArgs a) {
  extern __shared__ uint32_t mkeys[];  // [total] the row's keys, list after list
  __shared__ FastTopScratch fs;
  __shared__ int off[SPLIT_MAX_LISTS + 1];
  using All = Group<SM_THREADS, 0>;
  const int r = blockIdx.x;
  auto idx = [&](int j) { return a.row_major ? (int64_t)r * a.lists + j : (int64_t)j * a.rows + r; };
  if (threadIdx.x == 0) {
    int acc = 0;
    for (int j = 0; j < a.lists; ++j) {
      off[j] = acc;
      acc += min(max(__ldg(a.n + idx(j)), 0), TOPK);
    }
    off[a.lists] = acc;
  }
  __syncthreads();
  const int total = off[a.lists];
  const int k = min(TOPK, total);
  if (k == 0) {
    if (threadIdx.x == 0) a.out_n[r] = 0;
    return;
  }
  auto locate = [&](int i) {  // packed index -> (list, entry): the last list starting at or before i
    int lo = 0, hi = a.lists - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (off[mid] <= i) lo = mid; else hi = mid - 1;
    }
    return idx(lo) * TOPK + (i - off[lo]);
  };
  // one list per warp at a time, a lane's 16 loads issued before any is stored (in flight together)
  {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int j = warp; j < a.lists; j += SM_THREADS / 32) {
      const uint32_t* src = a.keys + idx(j) * TOPK;
      const int o = off[j], cnt = off[j + 1] - o;
      uint32_t kv[TOPK / 32];
#pragma unroll
      for (int u = 0; u < TOPK / 32; ++u) {
        const int e = lane + 32 * u;
        kv[u] = e < cnt ? __ldg(src + e) : 0u;
      }
#pragma unroll
      for (int u = 0; u < TOPK / 32; ++u) {
        const int e = lane + 32 * u;
        if (e < cnt) mkeys[o + e] = kv[u];
      }
    }
  }
  __syncthreads();
  fast_topk<All>([&](int i) { return mkeys[i]; }, total, k,
                 [&](int i, int o) {
                   a.out_id[(int64_t)r * TOPK + o] = __ldg(a.ids + locate(i));
                   if (a.out_key) a.out_key[(int64_t)r * TOPK + o] = mkeys[i];
                 },
                 &fs);
  if (threadIdx.x == 0) a.out_n[r] = k;
}

static cudaError_t launch_merge(const MergeArgs& a, cudaStream_t st) {
  static int attr_bytes[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  const size_t smem = split_merge_smem(a.lists);
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (attr_bytes[dev] < (int)smem) {
    const cudaError_t e = cudaFuncSetAttribute(k_split_merge, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    attr_bytes[dev] = (int)smem;
  }
  k_split_merge<<<a.rows, SM_THREADS, smem, st>>>(a);
  return cudaGetLastError();
}

// Positions of row r this rank attends to: the kept blocks it holds (4 positions each) and, if it
// holds the request's last position, the tail 4 * floor(L/4) .. L-1.  One warp per row, output in
// ascending order.
__global__ void __launch_bounds__(32) k_split_positions(SplitParams p, const int32_t* blocks, const int32_t* nblocks,
                                                        int32_t* pos, int32_t* npos) {
  const int r = blockIdx.x, lane = threadIdx.x;
  const int L = __ldg(p.seq_len + r);
  const int lo = __ldg(p.page_lo + r), cnt = __ldg(p.page_cnt + r);
  const int g0 = lo * PAGE, g1 = (lo + cnt) * PAGE;  // global positions held: [g0, g1)
  const int nb = L >> 2;
  int n = __ldg(nblocks + r);
  if (n < 0 || n > TOPK || n > nb) {
    if (lane == 0) set_error(p.err, QSA_DEVERR_SELECTION);
    n = 0;
  }
  int32_t* out = pos + (int64_t)r * MAX_SEL;
  int o = 0;
  for (int i0 = 0; i0 < n; i0 += 32) {
    const int i = i0 + lane;
    const int b = i < n ? __ldg(blocks + (int64_t)r * TOPK + i) : -1;
    const bool mine = b >= 0 && 4 * b >= g0 && 4 * b < g1;
    const unsigned m = __ballot_sync(0xffffffffu, mine);
    if (mine) {
      const int at = o + 4 * __popc(m & ((1u << lane) - 1u));
#pragma unroll
      for (int j = 0; j < 4; ++j) out[at + j] = 4 * b + j;
    }
    o += 4 * __popc(m);
  }
  const int tail0 = 4 * nb;
  if (L >= 1 && L - 1 >= g0 && L - 1 < g1) {  // this rank holds the last position, hence the tail
    if (lane < L - tail0) out[o + lane] = tail0 + lane;
    o += L - tail0;
  }
  if (lane == 0) npos[r] = o;
}

// out[r] = sum_k e^(lse_k - M) out_k[r] / sum_k e^(lse_k - M), per head (M the largest lse; ranks
// with no positions have lse = -inf and weight 0).  grid = rows, 16 x 32 threads (head, 4 dims).
__global__ void __launch_bounds__(HQ * 32) k_split_combine(const __nv_bfloat16* outs, const float* lses, int world,
                                                           int rows, __nv_bfloat16* out) {
  const int r = blockIdx.x, h = threadIdx.x >> 5, c4 = threadIdx.x & 31;
  float M = -INFINITY;
  for (int k = 0; k < world; ++k) M = fmaxf(M, __ldg(lses + ((int64_t)k * rows + r) * HQ + h));
  const float base = M == -INFINITY ? 0.f : M;
  float den = 0.f, acc[4] = {0.f, 0.f, 0.f, 0.f};
  for (int k = 0; k < world; ++k) {
    const float wk = expf(__ldg(lses + ((int64_t)k * rows + r) * HQ + h) - base);
    const uint2 v = __ldg(reinterpret_cast<const uint2*>(outs + (((int64_t)k * rows + r) * HQ + h) * D) + c4);
    den += wk;
    acc[0] += wk * bf16_bits_to_f32((uint16_t)(v.x & 0xFFFFu));
    acc[1] += wk * bf16_bits_to_f32((uint16_t)(v.x >> 16));
    acc[2] += wk * bf16_bits_to_f32((uint16_t)(v.y & 0xFFFFu));
    acc[3] += wk * bf16_bits_to_f32((uint16_t)(v.y >> 16));
  }
  const float inv = den > 0.f ? 1.f / den : 0.f;
  uint2 o;
  o.x = pack_bf16x2(acc[0] * inv, acc[1] * inv);
  o.y = pack_bf16x2(acc[2] * inv, acc[3] * inv);
  reinterpret_cast<uint2*>(out + ((int64_t)r * HQ + h) * D)[c4] = o;
}

// ---- host launchers ----
cudaError_t launch_split_score(const SplitParams& p, int rows, cudaStream_t st) {
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  const size_t smem = sizeof(SpSmem) + 128;
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    const cudaError_t e = cudaFuncSetAttribute(k_split_score, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  k_split_score<<<dim3(p.nchunks, rows), SP_THREADS, smem, st>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  MergeArgs a{p.cand_key, p.cand_id, p.cand_n, p.nchunks, rows, 1, p.out_key, p.out_id, p.out_n};
  return launch_merge(a, st);
}

cudaError_t launch_split_merge(const uint32_t* keys, const int32_t* ids, const int32_t* n, int world, int rows,
                               int32_t* blocks, int32_t* nblocks, cudaStream_t st) {
  MergeArgs a{keys, ids, n, world, rows, 0, nullptr, blocks, nblocks};
  return launch_merge(a, st);
}

cudaError_t launch_split_positions(const SplitParams& p, const int32_t* blocks, const int32_t* nblocks, int rows,
                                   int32_t* pos, int32_t* npos, cudaStream_t st) {
  k_split_positions<<<rows, 32, 0, st>>>(p, blocks, nblocks, pos, npos);
  return cudaGetLastError();
}

cudaError_t launch_split_combine(const __nv_bfloat16* outs, const float* lses, int world, int rows,
                                 __nv_bfloat16* out, cudaStream_t st) {
  k_split_combine<<<rows, HQ * 32, 0, st>>>(outs, lses, world, rows, out);
  return cudaGetLastError();
}

}  // namespace qsa
