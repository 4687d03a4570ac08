// Streaming block scorer with a fused exact top-512 (decode and any query
// whose blocks stream from the paged compressed cache).
//
// Blog section "Qwen Sparse Attention: Retrieve Coarsely, Attend Precisely"
// (SGLang day-0 blog for Qwen3.8-Flash-Next): a query scores every visible
// compressed block and the best 512 are kept.  Score (the text's formula is
// lost; this is the stated reading): s_b = sum_h w_h * max(0, q~_h . k^_b);
// ties keep the lower block index.
//
// Design (B200).  The pass is HBM-bound: 256 bytes of compressed key per block
// against 4 dot products of 128.  Work is balanced whatever the mix of context
// lengths: all pages to score (64 tokens = 16 compressed keys = 4 KiB,
// contiguous because the cache is page aligned) are laid end to end over the
// rows, each row preceded by SC_ROW_COST empty pages that stand for the fixed
// work of starting a segment, and each persistent CTA (one of 16 warps per SM)
// owns an equal contiguous range of that list.  A range crosses at most a few
// rows; its piece of one row is a "segment".
//   * Pages sit at random places in HBM, so what bounds the pass is how many
//     independent 4 KiB reads are in flight; a measured probe of this access
//     pattern peaks with many warps each holding whole pages, not with one
//     TMA producer per CTA.  So every warp reads its own pages with coalesced
//     16-byte loads straight into registers (each load instruction covers
//     eight keys x 64 contiguous bytes), U pages at a time.
//   * The loaded registers ARE the A fragments of m16n8k16 bf16 MMAs (A = 16
//     keys x 16 dims, B = the 4 rotated query heads padded to 8 columns):
//     because a dot product does not care about the order of its terms, the
//     query's B fragments are built with the same permutation of dims that
//     the loads produce, and no shuffle or shared-memory staging is needed.
//     The FP32 pipes stay free; the tensor pipe is far from busy.
//   * Scores become order-preserving 32-bit keys in shared memory, counted
//     as they are written into a log-scale histogram, so that the segment's
//     exact top-512 (hist_topk) needs one pass over the keys.  A segment that
//     is a whole row gives the answer directly; otherwise its candidates go
//     to the row's list in global memory, and the CTA that completes the
//     row's last segment (atomic page count, no waiting) merges them: it
//     orders the row's segments by block and selects the final 512 from
//     their candidates in block-ordered chunks, ascending.  Scores never
//     travel to HBM.
//   * The sparse GQA is launched as a programmatic dependent of this kernel
//     and waits per row: each row's selection is published (release flag) as
//     soon as it is final.
#include <cstdlib>

#include "qsa_common.cuh"
#include "qsa_kernels.h"

namespace qsa {

#ifndef QSA_SC_PAGES_PER_LOAD
#define QSA_SC_PAGES_PER_LOAD 1
#endif
// One CTA of 16 warps per SM: the streaming keeps 16 warps' pages in flight per SM, and the
// selection phases, which are bound by latency, run on all 16 warps instead of half of them.
#ifndef QSA_SC_CTAS_PER_SM
#define QSA_SC_CTAS_PER_SM (16 / QSA_SC_WARPS)
#endif
constexpr int SC_WARPS = QSA_SC_WARPS;
constexpr int SC_THREADS = SC_WARPS * 32;
constexpr int SC_U = QSA_SC_PAGES_PER_LOAD;  // pages a warp loads before computing
constexpr int SC_SEG_KEYS = SC_MAX_SEG_PAGES * PAGE_BLOCKS;  // 8192

using Cta = Group<SC_THREADS, 0>;

constexpr int SC_MERGE_CAP = SC_SEG_KEYS / 2;  // merge candidates held at once

// Kept small on purpose: the L1 cache shares the SM's memory with this, and the page loads in
// flight need L1 room (a larger footprint measurably slows the streaming).
struct ScoreSmem {
  uint32_t keys[SC_SEG_KEYS];           // a segment's score keys; a merge's candidate keys
                                        // [0, SC_MERGE_CAP) and block ids [SC_MERGE_CAP, 2 SC_MERGE_CAP)
  alignas(16) uint32_t hist[HT_WORDS];  // histogram of `keys` (built as they are written)
  HistTopScratch ht;
  int32_t pid[SC_MAX_SEG_PAGES];    // physical pages of the current segment (-1: invalid)
  int32_t off[SC_ROWS_SMEM + 1];    // exclusive prefix of pages per row
  int4 segs[SC_MAX_SEGS];           // merge: the row's segments (start block, cand offset, count, -)
  int vstart[SC_MAX_SEGS + 1];      // merge: prefix of the ordered segments' counts
  double cs[D / 2], sn[D / 2];      // fused front end: RoPE angles of the current row's query
  uint32_t qraw[HI * D / 2];        // fused front end: unrotated query, then rotated (bf16 pairs)
  int warp_tot[33];
  int bcast[4];
  int next_page;  // streaming: the next unclaimed page group of the segment
};
static_assert(SC_SEG_KEYS <= HT_MAX_N && SC_SEG_KEYS <= 32 * SC_THREADS, "a segment's keys fit one selection");
static_assert(2 * HT_TIE_CAP >= TOPK && SC_MERGE_CAP > TOPK, "merge survivors fit the tie storage");
static_assert(sizeof(SelectScratch) <= HT_WORDS * 4, "the radix fallback borrows the histogram");

struct Segment {
  int row, p0, np;  // row, first page within the row, pages
};

// Largest row r with off[r] <= g (off is non-decreasing; rows without pages
// have empty intervals and are never returned for g < off[rows]).
__device__ __forceinline__ int row_of_page(const int32_t* off_s, const int32_t* off_g, int rows, int g) {
  int lo = 0, hi = rows - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    const int v = off_s ? off_s[mid] : __ldg(off_g + mid);
    if (v <= g) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

// The segments of a row, in block order: its pages (page-list interval [rs, re)) cut at every range
// boundary (multiples of ppc) and every SC_MAX_SEG_PAGES pages from a range piece's start -- the
// same cuts the segment loop makes.  Calls f(j, first page in the list, pages) for segment j and
// returns the number of segments.  A partial segment's candidates go to slot j of the row's list.
template <class F>
__device__ __forceinline__ int for_each_segment(int rs, int re, int ppc, F f) {
  int j = 0;
  for (int g = rs; g < re;) {
    const int e = min(re, (g / ppc + 1) * ppc);
    for (int a = g; a < e; a += SC_MAX_SEG_PAGES, ++j) f(j, a, min(e, a + SC_MAX_SEG_PAGES) - a);
    g = e;
  }
  return j;
}

__global__ void __launch_bounds__(SC_THREADS, QSA_SC_CTAS_PER_SM) k_score_topk(ScoreParams p) {
  extern __shared__ uint8_t smem_raw[];
  ScoreSmem& S = *reinterpret_cast<ScoreSmem*>(smem_aligned<128>(smem_raw));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int rows = p.rows;
  const bool fused = p.idx_q != nullptr;  // the host sets it only when rows <= SC_ROWS_SMEM
  // Every CTA of this grid is resident (the grid is sized to residency); the sparse GQA launched
  // after it may start now on SMs this grid frees, and waits per row for the row's flag.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  auto row_of = [&](int r, int& req, int& L) {
    req = p.row_req ? __ldg(p.row_req + r) : r;
    L = __ldg(p.row_len + r) + p.len_offset;
    return req >= 0 && req < p.c.batch && L >= 1 && L <= p.max_len;
  };

  // ---- rows with at most 512 complete blocks keep them all (and append here); bad rows keep none ----
  for (int r = blockIdx.x; r < rows; r += gridDim.x) {
    int req, L;
    const bool ok = row_of(r, req, L);
    const int nb = ok ? (L >> 2) : 0;
    if (nb > TOPK) continue;
    int32_t* sel = p.sel + (int64_t)r * TOPK;
    for (int i = tid; i < nb; i += SC_THREADS) sel[i] = i;
    if (tid == 0) {
      p.sel_n[r] = nb;
      if (!ok) set_error(p.err, (req < 0 || req >= p.c.batch) ? QSA_DEVERR_REQUEST : QSA_DEVERR_LENGTH);
    }
    if (fused && p.knew && ok && warp == 0) warp_decode_append(p.c, req, L, p.knew + (int64_t)r * D, p.fr, p.err);
    if (p.row_ready) {
      __syncthreads();
      if (tid == 0) publish_ready(p.row_ready + r * READY_STRIDE);
    }
  }

  // ---- the page list ----
  const bool off_in_smem = rows <= SC_ROWS_SMEM;
  if (fused) {  // exclusive prefix of the pages each row streams
    int running = 0;
    for (int base = 0; base < rows; base += SC_THREADS) {
      const int r = base + tid;
      int pages = 0;
      if (r < rows) {
        int req, L;
        const int nb = row_of(r, req, L) ? (L >> 2) : 0;
        pages = nb > TOPK ? SC_ROW_COST + ceil_div(nb, PAGE_BLOCKS) : 0;
      }
      int tot;
      const int ex = group_exclusive_scan<Cta>(pages, S.warp_tot, &tot);
      if (r < rows) S.off[r] = running + ex;
      running += tot;
    }
    if (tid == 0) S.off[rows] = running;
  } else if (off_in_smem) {
    for (int i = tid; i <= rows; i += SC_THREADS) S.off[i] = __ldg(p.page_off + i);
  }
  __syncthreads();
  const int32_t* off_s = off_in_smem ? S.off : nullptr;
  auto off_at = [&](int r) { return off_in_smem ? S.off[r] : __ldg(p.page_off + r); };
  const int P = off_at(rows);
  if (P == 0) return;
  int ppc = ceil_div(P, gridDim.x);  // pages per range
  ppc = max(ppc, p.ppc_min);
  const int nranges = ceil_div(P, ppc);

  const int g8 = lane >> 2, cq = lane & 3;
  const uint4* cidx = reinterpret_cast<const uint4*>(p.c.cidx);
  int range = -1, g = 0, gend = 0;
  int cur_row = -1;
  uint32_t bq[8][2];
  float wa = 0.f, wb = 0.f;
  while (true) {
    // ---- next segment: ranges blockIdx.x, +gridDim.x, ..., cut at row boundaries and every 512 pages ----
    if (g >= gend) {
      range = range < 0 ? (int)blockIdx.x : range + (int)gridDim.x;
      if (range >= nranges) break;
      g = range * ppc;
      gend = min(P, g + ppc);
    }
    Segment sg;
    sg.row = row_of_page(off_s, p.page_off, rows, g);
    const int rend = off_at(sg.row + 1);
    const int rstart = off_at(sg.row) + SC_ROW_COST;  // the row's first page to stream
    if (g < rstart) {  // the row's empty pages: nothing to do
      g = min(rstart, gend);
      continue;
    }
    sg.p0 = g - rstart;
    sg.np = min(min(gend, rend), g + SC_MAX_SEG_PAGES) - g;
    const int g_seg = g;
    g += sg.np;
    if (sg.np <= 0) continue;
    const int r = sg.row;
    const int req = p.row_req ? __ldg(p.row_req + r) : r;
    const int L = __ldg(p.row_len + r) + p.len_offset;
    const bool new_row = r != cur_row;
    uint32_t qv = 0;
    if (fused && new_row) {  // the row's index query and its RoPE angles at position L - 1
      if (tid < HI * D / 2) qv = __ldg(reinterpret_cast<const uint32_t*>(p.idx_q + (int64_t)r * HI * D) + tid);
      if (tid < D / 2) sincos((double)(L - 1) * p.fr.f[tid], &S.sn[tid], &S.cs[tid]);
    }
    {  // the segment's physical pages
      const int32_t* pt = p.c.page_table + (int64_t)req * p.c.max_pages;
      for (int k = tid; k < sg.np; k += SC_THREADS) {
        const int lp = sg.p0 + k;
        int phys = lp < p.c.max_pages ? __ldg(pt + lp) : -1;
        if (phys < 0 || phys >= p.c.num_pages) {
          set_error(p.err, QSA_DEVERR_PAGE);
          phys = -1;
        }
        S.pid[k] = phys;
      }
    }
    if (new_row) {
      // B operand, permuted like the loads: column n = index head n (zero for n >= 4); for k-step
      // j = 2u + h, lane (n, c) holds dims 8(c+4u) + 4h + {0,1} (b0) and + {2,3} (b1).
      cur_row = r;
      const uint32_t* q32 = reinterpret_cast<const uint32_t*>(p.qrot + (int64_t)r * HI * D);
      if (fused) {  // rotate here: pairs (i, i + 64) of head h, FP64 angles, one bf16 rounding
        constexpr int NR = HI * D / 2;  // threads of the rotation: one pair (i, i + 64) of one head each
        if (tid < NR) S.qraw[tid] = qv;
        __syncthreads();
        const int h = tid >> 6, i = tid & 63;
        uint16_t y0 = 0, y1 = 0;
        if (tid < NR) {
          const uint16_t* q16 = reinterpret_cast<const uint16_t*>(S.qraw) + h * D;
          const double x0 = (double)bf16_bits_to_f32(q16[i]);
          const double x1 = (double)bf16_bits_to_f32(q16[i + D / 2]);
          y0 = f64_to_bf16_bits(x0 * S.cs[i] - x1 * S.sn[i]);
          y1 = f64_to_bf16_bits(x0 * S.sn[i] + x1 * S.cs[i]);
        }
        __syncthreads();
        if (tid < NR) {
          uint16_t* o16 = reinterpret_cast<uint16_t*>(S.qraw) + h * D;
          o16[i] = y0;
          o16[i + D / 2] = y1;
        }
        __syncthreads();
        q32 = S.qraw;
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int d0 = 8 * (cq + 4 * (j >> 1)) + 4 * (j & 1);
        bq[j][0] = g8 < HI ? q32[(g8 * D + d0) >> 1] : 0u;  // shared (fused) or global memory
        bq[j][1] = g8 < HI ? q32[(g8 * D + d0 + 2) >> 1] : 0u;
      }
      wa = cq < 2 ? __ldg(p.w + (int64_t)r * HI + 2 * cq) : 0.f;
      wb = cq < 2 ? __ldg(p.w + (int64_t)r * HI + 2 * cq + 1) : 0.f;
    }
    const int nb = L >> 2;
    const int b0 = sg.p0 * PAGE_BLOCKS;
    const int nvalid = min(sg.np * PAGE_BLOCKS, nb - b0);
    const int np_row = off_at(r + 1) - off_at(r) - SC_ROW_COST;
    // The row's decode append is made by the CTA owning its last page, before that page is read;
    // when it completes block nb - 1 (in the last page), that page is read with coherent loads.
    int fresh_k = -1;
    if (fused && p.knew && sg.p0 + sg.np == np_row) {
      if (warp == 0) warp_decode_append(p.c, req, L, p.knew + (int64_t)r * D, p.fr, p.err);
      if ((L & 3) == 0) fresh_k = sg.np - 1;
    }
    // A segment that is not the whole row writes its candidates to slot `ord` of the row's list:
    // its rank among the row's segments, in block order.
    const bool partial = sg.np != np_row;
    const int ncand = min(nvalid, TOPK);
    int ord = 0;
    if (partial) for_each_segment(rstart, rend, ppc, [&](int j, int a, int) { ord = a < g_seg ? j + 1 : ord; });
    ht_zero<Cta>(S.hist);
    if (tid == 0) S.next_page = SC_WARPS * SC_U;
    Cta::sync();

    // ---- stream: warp w starts with pages w*U .. w*U+U-1, then claims the next U pages from a
    // shared counter (claimed while its current pages load), so the warps end together ----
    for (int k0 = warp * SC_U; k0 < sg.np;) {
      int k_next = 0;
      if (lane == 0) k_next = atomicAdd(&S.next_page, SC_U);
      PageRegs pr[SC_U];
#pragma unroll
      for (int u = 0; u < SC_U; ++u) {
        const int k = k0 + u;
        const int phys = k < sg.np ? S.pid[k] : -1;
        if (phys >= 0) {
          if (k == fresh_k) load_page_fresh(pr[u], cidx + (int64_t)phys * (PAGE_BLOCKS * D / 8), g8, cq);
          else load_page(pr[u], cidx + (int64_t)phys * (PAGE_BLOCKS * D / 8), g8, cq);
        }
      }
#pragma unroll
      for (int u = 0; u < SC_U; ++u) {
        const int k = k0 + u;
        if (k >= sg.np) break;
        float lo, hi;
        score_page(pr[u], bq, wa, wb, lo, hi);
        if (S.pid[k] < 0) lo = hi = 0.f;  // unreadable page (flagged above)
        if (cq < 2) {
          const int local = k * PAGE_BLOCKS + g8 + 8 * cq;
          if (local < nvalid) {
            const uint32_t key = score_key(cq ? hi : lo);
            S.keys[local] = key;
            ht_count(S.hist, key);
          }
        }
      }
      k0 = __shfl_sync(0xffffffffu, k_next, 0);
    }
    Cta::sync();

    // ---- the segment's best 512 ----
    int32_t* sel = p.sel + (int64_t)r * TOPK;
    if (sg.np == np_row) {  // the whole row (nb > 512 here): this is the answer
      hist_topk<Cta>(S.keys, S.hist, nvalid, TOPK, [&](int i, int o) { sel[o] = b0 + i; }, &S.ht);
      if (tid == 0) {
        p.sel_n[r] = TOPK;
        if (p.row_ready) publish_ready(p.row_ready + r * READY_STRIDE);
      }
      continue;
    }
    const int seg_slots = min(p.seg_cap, SC_MAX_SEGS);
    if (ord >= seg_slots) {  // more segments than the workspace was sized for: drop this one, flag it
      if (tid == 0) set_error(p.err, QSA_DEVERR_SELECTION);
    } else {
      uint32_t* ck = p.cand_key + ((int64_t)r * p.seg_cap + ord) * TOPK;
      int32_t* ci = p.cand_id + ((int64_t)r * p.seg_cap + ord) * TOPK;
      auto put = [&](int i, int o) {
        ck[o] = S.keys[i];
        ci[o] = b0 + i;
      };
      if (nvalid > TOPK) {
        hist_topk<Cta>(S.keys, S.hist, nvalid, TOPK, put, &S.ht);
      } else {
        for (int i = tid; i < nvalid; i += SC_THREADS) put(i, i);
      }
    }
    __threadfence();
    Cta::sync();
    if (tid == 0) S.bcast[1] = atomicAdd(p.pages_done + r, sg.np) + sg.np == np_row;
    Cta::sync();
    if (!S.bcast[1]) continue;

    // ---- this CTA finished the row: merge its segments' candidates ----
    // The segments, their first blocks and candidate counts follow from the page list alone.
    __threadfence();
    if (tid == 0) {
      const int seg_slots = min(p.seg_cap, SC_MAX_SEGS);
      int acc = 0, ns_ = 0;
      for_each_segment(rstart, rend, ppc, [&](int j, int a, int npg) {
        if (j >= seg_slots) return;  // dropped by its writer (flagged there)
        const int sb0 = (a - rstart) * PAGE_BLOCKS;
        const int cnt = min(min(npg * PAGE_BLOCKS, nb - sb0), TOPK);
        S.segs[j] = make_int4(sb0, j * TOPK, cnt, 0);
        S.vstart[j] = acc;
        acc += cnt;
        ns_ = j + 1;
      });
      S.vstart[ns_] = acc;
      S.bcast[2] = ns_;
    }
    Cta::sync();
    const int ns = S.bcast[2];
    const uint32_t* rk = p.cand_key + (int64_t)r * p.seg_cap * TOPK;
    const int32_t* ri = p.cand_id + (int64_t)r * p.seg_cap * TOPK;
    // virtual index v (ascending block order) -> index into the row's candidate list
    auto gidx = [&](int v) {
      int lo = 0, hi = ns - 1;
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (S.vstart[mid] <= v) lo = mid;
        else hi = mid - 1;
      }
      return S.segs[lo].y + (v - S.vstart[lo]);
    };
    const int nv = S.vstart[ns];
    const int kk_sel = min(TOPK, nv);  // < 512 only when segments were dropped (flagged above)
    // Candidates are taken in block order, SC_MERGE_CAP at a time: each chunk is selected together
    // with the best 512 of the chunks before it (kept at the front of the buffer, still in block
    // order), so index order stays block order and ties keep the lower block.
    int32_t* mids = reinterpret_cast<int32_t*>(S.keys + SC_MERGE_CAP);
    unsigned long long* surv = S.ht.tie;  // survivors (key, id) of a non-final chunk
    for (int done = 0, held = 0;;) {
      const int take = min(nv - done, SC_MERGE_CAP - held);
      ht_zero<Cta>(S.hist);
      Cta::sync();
      for (int i = tid; i < held; i += SC_THREADS) ht_count(S.hist, S.keys[i]);
      // stage keys and ids, SU independent loads per thread in flight, counting keys as they arrive
      constexpr int SU = 8;
      for (int j0 = 0; j0 < take; j0 += SU * SC_THREADS) {
        uint32_t kk[SU];
        int32_t ii[SU];
#pragma unroll
        for (int u = 0; u < SU; ++u) {
          const int j = j0 + u * SC_THREADS + tid;
          if (j < take) {
            const int gi = gidx(done + j);
            kk[u] = __ldcg(rk + gi);
            ii[u] = __ldcg(ri + gi);
          }
        }
#pragma unroll
        for (int u = 0; u < SU; ++u) {
          const int j = j0 + u * SC_THREADS + tid;
          if (j < take) {
            S.keys[held + j] = kk[u];
            mids[held + j] = ii[u];
            ht_count(S.hist, kk[u]);
          }
        }
      }
      Cta::sync();
      const int n = held + take;
      done += take;
      if (done >= nv) {
        hist_topk<Cta>(S.keys, S.hist, n, kk_sel, [&](int v, int o) { sel[o] = mids[v]; }, &S.ht);
        break;
      }
      hist_topk<Cta>(S.keys, S.hist, n, kk_sel,
                     [&](int v, int o) { surv[o] = ((unsigned long long)S.keys[v] << 32) | (uint32_t)mids[v]; },
                     &S.ht);
      for (int o = tid; o < kk_sel; o += SC_THREADS) {
        const unsigned long long e = surv[o];
        S.keys[o] = (uint32_t)(e >> 32);
        mids[o] = (int32_t)(uint32_t)e;
      }
      held = kk_sel;
      Cta::sync();
    }
    if (tid == 0) {
      if (kk_sel < TOPK) set_error(p.err, QSA_DEVERR_SELECTION);
      p.sel_n[r] = kk_sel;
      p.pages_done[r] = 0;  // ready for the next call
      if (p.row_ready) publish_ready(p.row_ready + r * READY_STRIDE);
    }
    Cta::sync();
  }
}

// Persistent grid: as many CTAs as are resident at once (QSA_SC_CTAS_PER_SM per SM when the
// shared memory allows it), so that no CTA waits for a second wave.
cudaError_t launch_score_topk(const ScoreParams& p, int num_sms, cudaStream_t st) {
  static int resident[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  const size_t smem = sizeof(ScoreSmem) + 128;
  int per_sm = QSA_SC_CTAS_PER_SM;
  if (dev >= 0 && dev < 64) {
    if (resident[dev] == 0) {
      cudaError_t e = cudaFuncSetAttribute(k_score_topk, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
      int n = 0;
      e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k_score_topk, SC_THREADS, smem);
      if (e != cudaSuccess) return e;
      resident[dev] = max(1, min(n, QSA_SC_CTAS_PER_SM));
    }
    per_sm = resident[dev];
  }
  k_score_topk<<<per_sm * num_sms, SC_THREADS, smem, st>>>(p);
  return cudaGetLastError();
}

}  // namespace qsa