// Streaming block scorer with a fused exact top-512 (decode and any query
// whose blocks stream from the paged compressed cache).
//
// Blog section "Qwen Sparse Attention: Retrieve Coarsely, Attend Precisely"
// (SGLang day-0 blog for Qwen3.8-Flash-Next): a query scores every visible
// compressed block and the best 512 are kept.  Score (the text's formula is
// lost; this is the stated reading): s_b = sum_h w_h * max(0, q~_h . k^_b);
// ties keep the lower block index.
//
// Design (B200): the pass is HBM-bound -- 256 bytes of compressed key per
// block against 4 dot products of 128.  Each CTA owns a chunk of one row's
// blocks.  A producer warp streams whole 64-token pages (16 compressed keys =
// 4 KiB, contiguous because the cache is page aligned) with 2-D TMA into a
// 16-deep shared-memory ring, 128-byte swizzled so that ldmatrix reads are
// conflict free.  Eight consumer warps each turn a page into 16 scores with
// eight m16n8k16 bf16 MMAs (A = 16 keys x 16 dims, B = the 4 rotated query
// heads padded to 8 columns) -- this keeps the FP32 pipes free, the tensor
// pipe is nowhere near busy.  Scores never leave the SM: they become
// order-preserving 32-bit keys in shared memory, a CTA-wide radix select keeps
// the chunk's best 512, and the last CTA of the row to finish (atomic ticket,
// no waiting) merges the chunks' candidates from L2 into the final 512.
#include "qsa_common.cuh"
#include "qsa_kernels.h"

namespace qsa {

constexpr int SC_CONS = 8;                      // consumer warps
constexpr int SC_THREADS = (SC_CONS + 1) * 32;  // + one producer warp
constexpr int SC_STAGES = 16;                   // pages in flight per CTA
constexpr int SC_PAGE_BYTES = PAGE_BLOCKS * D * 2;  // 4096

struct __align__(1024) ScoreSmem {
  uint8_t stage[SC_STAGES][SC_PAGE_BYTES];  // each page: two 16 x 128 B halves (dims 0-63, 64-127)
  uint32_t keys[SC_MAX_CHUNK];
  uint64_t full[SC_STAGES];
  uint64_t empty[SC_STAGES];
  SelectScratch sel;
  int is_last;
};

__global__ void __launch_bounds__(SC_THREADS, 2) k_score_topk(ScoreParams p, const __grid_constant__ CUtensorMap tmap) {
  extern __shared__ uint8_t smem_raw[];
  ScoreSmem& S = *reinterpret_cast<ScoreSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int row = blockIdx.y, chunk = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int req = p.row_req ? __ldg(p.row_req + row) : row;
  const int L = __ldg(p.row_len + row) + p.len_offset;
  int32_t* sel = p.sel + (int64_t)row * TOPK;
  if (req < 0 || req >= p.c.batch || L < 1 || L > p.max_len) {
    if (chunk == 0 && tid == 0) {
      set_error(p.err, (req < 0 || req >= p.c.batch) ? QSA_DEVERR_REQUEST : QSA_DEVERR_LENGTH);
      p.sel_n[row] = 0;
    }
    return;
  }
  const int nb = L >> 2;
  if (nb <= TOPK) {  // every complete block is kept
    if (chunk == 0) {
      for (int i = tid; i < nb; i += blockDim.x) sel[i] = i;
      if (tid == 0) p.sel_n[row] = nb;
    }
    return;
  }
  const int nchunks = ceil_div(nb, p.chunk);
  if (chunk >= nchunks) return;
  const int b0 = chunk * p.chunk;
  const int nvalid = min(p.chunk, nb - b0);
  const int npages = ceil_div(nvalid, PAGE_BLOCKS);
  const int page0 = b0 / PAGE_BLOCKS;

  if (tid == 0) {
    for (int s = 0; s < SC_STAGES; ++s) {
      mbar_init(&S.full[s], 1);
      mbar_init(&S.empty[s], 1);
    }
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == SC_CONS) {
    // ---------------- producer: one lane issues the page loads ----------------
    if (lane == 0) {
      prefetch_tmap(&tmap);
      const int32_t* pt = p.c.page_table + (int64_t)req * p.c.max_pages;
      for (int i = 0; i < npages; ++i) {
        const int s = i % SC_STAGES;
        if (i >= SC_STAGES) mbar_wait(&S.empty[s], ((i / SC_STAGES) - 1) & 1, p.err);
        const int lp = page0 + i;
        const int phys = lp < p.c.max_pages ? __ldg(pt + lp) : -1;
        if (phys < 0 || phys >= p.c.num_pages) {
          set_error(p.err, QSA_DEVERR_PAGE);
          mbar_arrive(&S.full[s]);  // complete the phase without data
          continue;
        }
        mbar_arrive_expect_tx(&S.full[s], SC_PAGE_BYTES);
        tma_load_2d(S.stage[s], &tmap, 0, phys * PAGE_BLOCKS, &S.full[s]);
        tma_load_2d(S.stage[s] + SC_PAGE_BYTES / 2, &tmap, 64, phys * PAGE_BLOCKS, &S.full[s]);
      }
    }
  } else {
    // ---------------- consumers: 16 scores per page on the tensor pipe --------
    const int g = lane >> 2, cq = lane & 3;
    // B operand: column n = index head n (n < 4), k = dim; padded heads are 0.
    uint32_t bq[8][2];
    const uint32_t* q32 = reinterpret_cast<const uint32_t*>(p.qrot + (int64_t)row * HI * D);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      bq[j][0] = g < HI ? __ldg(q32 + ((g * D + 16 * j + 2 * cq) >> 1)) : 0u;
      bq[j][1] = g < HI ? __ldg(q32 + ((g * D + 16 * j + 2 * cq + 8) >> 1)) : 0u;
    }
    const float wa = cq < 2 ? __ldg(p.w + (int64_t)row * HI + 2 * cq) : 0.f;
    const float wb = cq < 2 ? __ldg(p.w + (int64_t)row * HI + 2 * cq + 1) : 0.f;
    // ldmatrix lane geometry: matrix mtx = lane/8 covers rows (mtx&1)*8.., dims (mtx>>1)*8..
    const int mtx = lane >> 3;
    const int rr = (lane & 7) + ((mtx & 1) << 3);
    const uint32_t lane_off = rr * 128;
    for (int i = warp; i < npages; i += SC_CONS) {
      const int s = i % SC_STAGES;
      mbar_wait(&S.full[s], (i / SC_STAGES) & 1, p.err);
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
      const uint32_t base = smem_u32(S.stage[s]) + lane_off;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int c16 = ((j & 3) << 1) + (mtx >> 1);
        uint32_t a[4];
        ldmatrix_x4(a[0], a[1], a[2], a[3], base + (j >> 2) * (SC_PAGE_BYTES / 2) + ((c16 ^ (rr & 7)) << 4));
        mma_bf16_16816(acc, a, bq[j][0], bq[j][1]);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.empty[s]);
      // acc: rows g / g+8 (keys), columns 2cq, 2cq+1 (heads)
      float lo = wa * fmaxf(acc[0], 0.f) + wb * fmaxf(acc[1], 0.f);
      float hi = wa * fmaxf(acc[2], 0.f) + wb * fmaxf(acc[3], 0.f);
      lo += __shfl_xor_sync(0xffffffffu, lo, 1);
      hi += __shfl_xor_sync(0xffffffffu, hi, 1);
      lo += __shfl_xor_sync(0xffffffffu, lo, 2);
      hi += __shfl_xor_sync(0xffffffffu, hi, 2);
      if (cq < 2) {
        const int local = i * PAGE_BLOCKS + g + 8 * cq;
        if (local < nvalid) S.keys[local] = score_key(cq ? hi : lo);
      }
    }
  }
  __syncthreads();

  // ---------------- chunk top-512 ----------------
  SelectResult r{0u, 0u, nvalid};  // nvalid <= 512: keep all (every key matches the empty mask)
  auto skey = [&](int i) { return S.keys[i]; };
  if (nvalid > TOPK) r = radix_select(skey, nvalid, TOPK, &S.sel);
  if (nchunks == 1) {
    select_compact(skey, nvalid, r, [&](int i, int o) { sel[o] = b0 + i; }, &S.sel);
    if (tid == 0) p.sel_n[row] = TOPK;
    return;
  }
  uint32_t* ck = p.cand_key + ((int64_t)row * p.max_chunks + chunk) * TOPK;
  int32_t* ci = p.cand_id + ((int64_t)row * p.max_chunks + chunk) * TOPK;
  select_compact(
      skey, nvalid, r,
      [&](int i, int o) {
        ck[o] = S.keys[i];
        ci[o] = b0 + i;
      },
      &S.sel);
  for (int o = min(nvalid, TOPK) + tid; o < TOPK; o += blockDim.x) {  // pad: below every real key
    ck[o] = 0u;
    ci[o] = -1;
  }

  // ---------------- last CTA of the row merges ----------------
  __threadfence();
  __syncthreads();
  if (tid == 0) S.is_last = atomicAdd(p.counters + row, 1) == nchunks - 1;
  __syncthreads();
  if (!S.is_last) return;
  __threadfence();
  const uint32_t* rk = p.cand_key + (int64_t)row * p.max_chunks * TOPK;
  const int32_t* ri = p.cand_id + (int64_t)row * p.max_chunks * TOPK;
  const int n = nchunks * TOPK;
  auto gkey = [&](int i) { return __ldcg(rk + i); };
  const SelectResult m = radix_select(gkey, n, TOPK, &S.sel);
  select_compact(gkey, n, m, [&](int i, int o) { sel[o] = __ldcg(ri + i); }, &S.sel);
  if (tid == 0) {
    p.sel_n[row] = TOPK;
    p.counters[row] = 0;  // ready for the next call
  }
}

int score_chunk_for(int rows, int max_len, int num_sms) {
  const int nb = max_len / CBLK;
  int chunk = 2048;
  // prefer more CTAs when the batch is small, fewer (less merge work) when it is large
  while (chunk > SC_MIN_CHUNK && (int64_t)rows * ceil_div(nb, chunk) < 4 * num_sms) chunk >>= 1;
  while (chunk < SC_MAX_CHUNK && (int64_t)rows * ceil_div(nb, chunk) > 16 * num_sms) chunk <<= 1;
  return chunk;
}

cudaError_t launch_score_topk(const ScoreParams& p, int rows, const CUtensorMap* tmap, cudaStream_t st) {
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  const size_t smem = sizeof(ScoreSmem) + 1024;
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(k_score_topk, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  dim3 grid(p.max_chunks, rows);
  k_score_topk<<<grid, SC_THREADS, smem, st>>>(p, *tmap);
  return cudaGetLastError();
}

}  // namespace qsa
