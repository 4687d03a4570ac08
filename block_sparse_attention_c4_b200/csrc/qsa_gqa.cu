// Sparse GQA over the raw paged K/V at the kept positions (decode, IndexShare
// draft steps, explicit position lists).
//
// Blog section "Qwen Sparse Attention: Retrieve Coarsely, Attend Precisely"
// (SGLang day-0 blog for Qwen3.8-Flash-Next): the compressed keys are only an
// index; the softmax and the value sum use the original, uncompressed K/V at
// the (at most 2051) selected positions.  Section "IndexShare MTP: Reusing the
// QSA Selection Across Draft Steps": draft query i also sees the positions
// drafted since the capture, up to its own.
//
// Design (B200): one CTA covers every query head of a row (16 heads x up to 8
// queries sharing one position list) for a contiguous range of positions
// (split-K), so each K/V row crosses HBM once.  16-position tiles of K and V
// (both KV heads, 1 KiB per position) are gathered with 16-byte cp.async
// into a 4-deep, XOR-swizzled shared-memory ring.  Warp (g, d-half, m-tile):
// S = Q_g K_g^T with m16n8k16 bf16 MMAs (rows = query heads of KV group g),
// an online softmax in the log2 domain, and O += P V_g for its 64 output
// dims.  The splits of a row form one thread-block cluster: each leaves its
// (O, m, l) partial in its own shared memory and, after a cluster barrier,
// merges one slice of the row's outputs from all of them through distributed
// shared memory.  (Without clusters -- the allocation-free entry point, or
// more splits than a cluster holds -- partials go through global memory and
// the last CTA of the row, by atomic ticket, merges them.)
#include <cooperative_groups.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include <mutex>

#include "qsa_common.cuh"
#include "qsa_kernels.h"

namespace qsa {


constexpr int GQ_TILE = 16;
constexpr int GQ_STAGES = 4;      // bf16 ring: 3 tiles of 16 KB in flight
constexpr int GQ_STAGES_F8 = 7;   // fp8 ring: 6 tiles of 8 KB in flight, the bf16 ring's bytes in flight (the
                                  // gather is bound by them) at the same 3 CTAs per SM
constexpr int GQ_ROW_BYTES = D * 2;                             // 256 B: one head of one position
constexpr int GQ_KV_BYTES = GQ_TILE * HKV * GQ_ROW_BYTES;       // 8 KiB: K (or V) of a tile
constexpr int GQ_STAGE_BYTES = 2 * GQ_KV_BYTES;                 // 16 KiB

constexpr int GQ_MAX_TILES = (QSA_MAX_SEL + QSA_MAX_DRAFT + GQ_TILE - 1) / GQ_TILE;  // per row

// The queries (both KV groups, MT*16 rows each) are staged in shared memory only until they are
// in registers; when they fit one tile's bf16 area they pass through the last ring stage (bf16 K/V)
// or the V buffers (fp8 K/V), which the pipeline first writes after every warp has read them.  Less
// shared memory leaves more L1 for the loads.
//
// FP8 K/V (E4M3, one scale for K and one for V): a tile is gathered as 512 B per position into a
// half-size ring stage (K rows with their 16-byte chunks swizzled).  Every E4M3 value is a bf16 value,
// so the conversions are exact.  K is read from the stage straight into the B fragments of Q K^T
// (4 consecutive dims per 32-bit load, the same dim order in the query's A fragments); each warp
// converts only the half of its KV group's V that it multiplies into a bf16 buffer of its own, so no
// CTA-wide pass or barrier sits on a tile's path.  The ring, then the V buffers, are one contiguous
// area that the split merge reuses.
template <int MT, bool F8>
struct GqaSmem {
  static constexpr int STAGE = F8 ? GQ_STAGE_BYTES / 2 : GQ_STAGE_BYTES;  // a tile's K and V as gathered
  static constexpr int STAGES = F8 ? GQ_STAGES_F8 : GQ_STAGES;
  static constexpr int VBUF = GQ_TILE * (GQ_ROW_BYTES / 2);  // fp8: one warp's V half, bf16 [16 pos][64 dims]
  static constexpr int CVT = F8 ? MT * 4 * VBUF : 128;
  static constexpr int QBYTES = HKV * MT * 16 * GQ_ROW_BYTES;
  static constexpr bool Q_IN_RING = QBYTES <= (F8 ? CVT : GQ_STAGE_BYTES);
  alignas(128) uint8_t kv[STAGES][STAGE];  // [K|V][group][pos][row], bf16 rows swizzled; fp8: K rows swizzled
  alignas(128) uint8_t cvt[CVT];           // fp8: the warps' V buffers (warp w at w * VBUF), rows swizzled
  alignas(128) uint8_t qsep[Q_IN_RING ? 16 : QBYTES];
  int is_last;
  alignas(16) int32_t slot[4];  // [p.tiles_per_split * 16] physical slot of each position of this CTA (-1: none)
  // split merge: the O partial (up to 32*MT heads x 128 fp32) in the ring area, (m, l) after it or in qsep
  static constexpr int AREA = STAGES * STAGE + (F8 ? CVT : 0);
  static constexpr int PO_BYTES = 32 * MT * D * 4, PML_BYTES = 32 * MT * 2 * 4;
  static constexpr bool ML_IN_RING = PO_BYTES + PML_BYTES <= AREA;
  static constexpr bool CLUSTER_FITS =
      PO_BYTES <= AREA && (ML_IN_RING || (Q_IN_RING ? 16 : QBYTES) >= PML_BYTES);
  __device__ __forceinline__ uint8_t* area() { return kv[0]; }
  __device__ __forceinline__ uint8_t* qrow(int g, int rho) {
    uint8_t* q = Q_IN_RING ? (F8 ? cvt : kv[STAGES - 1]) : qsep;
    return q + (g * MT * 16 + rho) * GQ_ROW_BYTES;
  }
};

// Eight E4M3 values -> eight bf16 values (exact), element order kept.
__device__ __forceinline__ uint32_t e4m3x2_to_bf16x2(uint16_t v) {
  const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(v), __NV_E4M3);
  const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h));
  return pack_bf16x2(f.x, f.y);
}

__device__ __forceinline__ uint4 e4m3x8_to_bf16x8(uint2 v) {
  return make_uint4(e4m3x2_to_bf16x2((uint16_t)(v.x & 0xFFFFu)), e4m3x2_to_bf16x2((uint16_t)(v.x >> 16)),
                    e4m3x2_to_bf16x2((uint16_t)(v.y & 0xFFFFu)), e4m3x2_to_bf16x2((uint16_t)(v.y >> 16)));
}

__device__ __forceinline__ uint32_t swz(int row, int chunk) { return (uint32_t)(((chunk ^ (row & 7)) << 4)); }

template <int MT, bool F8>
__global__ void __launch_bounds__(MT * 128) k_sparse_gqa(GqaParams p) {
  constexpr int THREADS = MT * 128;
  using Smem = GqaSmem<MT, F8>;
  extern __shared__ uint8_t smem_raw[];
  Smem& S = *reinterpret_cast<Smem*>(smem_aligned<128>(smem_raw));
  const int row = blockIdx.y, split = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nq = p.nq_row;
  const int req = p.row_req ? __ldg(p.row_req + row) : row;
  bool bad = req < 0 || req >= p.c.batch;
  if (bad && split == 0 && tid == 0) set_error(p.err, QSA_DEVERR_REQUEST);

  // ---- load the queries of both KV groups: row rho = query*8 + head-in-group ----
  {
    const __nv_bfloat16* qrow = p.q + (int64_t)row * nq * HQ * D;
    constexpr int CHUNKS = HKV * MT * 16 * (GQ_ROW_BYTES / 16);
    for (int c = tid; c < CHUNKS; c += THREADS) {
      const int g = c / (MT * 16 * 16);
      const int rho = (c / 16) % (MT * 16);
      const int ch = c % 16;
      const int qi = rho >> 3, h = g * GROUP + (rho & 7);
      uint4 v = make_uint4(0, 0, 0, 0);
      if (qi < nq) v = __ldg(reinterpret_cast<const uint4*>(qrow + ((int64_t)qi * HQ + h) * D) + ch);
      *reinterpret_cast<uint4*>(S.qrow(g, rho) + swz(rho, ch)) = v;
    }
  }

  // ---- launched early (programmatic dependent of the scorer): wait until this row's selection
  // is final; the queries above were loaded meanwhile ----
  if (p.row_ready) {
    if (!bad) {  // the row's page-table lines into L2 meanwhile: the slots are looked up right after
      const int L = __ldg(p.row_len + row) + p.len_offset;
      const int npg = L >= 1 && L <= p.max_len ? min(ceil_div(L, PAGE), p.c.max_pages) : 0;
      const int32_t* pt = p.c.page_table + (int64_t)req * p.c.max_pages;
      for (int i = tid * 32; i < npg; i += THREADS * 32) asm volatile("prefetch.global.L2 [%0];" ::"l"(pt + i));
    }
    if (tid == 0 && !wait_ready(p.row_ready + row * READY_STRIDE, p.err, p.wait_ns ? p.wait_ns : WAIT_LIMIT_NS))
      S.is_last = -1;
    else if (tid == 0) S.is_last = 0;
    __syncthreads();
    if (S.is_last < 0) bad = true;
  }

  // ---- the row's position list (coherent loads: the scorer may have written it just now) ----
  int nbase = 0, nsel4 = 0, tail0 = 0;
  const int32_t* sel = nullptr;
  const int32_t* list = nullptr;
  if (!bad) {
    if (p.mode == 0) {
      const int L = __ldg(p.row_len + row) + p.len_offset;
      const int nsel = __ldcg(p.sel_n + row);
      if (L < 1 || L > p.max_len || nsel < 0 || nsel > TOPK || nsel > (L >> 2)) {
        if (split == 0 && tid == 0) set_error(p.err, QSA_DEVERR_SELECTION);
        bad = true;
      } else {
        sel = p.sel + (int64_t)row * TOPK;
        nsel4 = 4 * nsel;
        tail0 = (L >> 2) << 2;
        nbase = nsel4 + (L & 3);
      }
    } else {
      const int n = __ldg(p.list_n + row);
      if (n < 0 || n > p.list_stride || n > MAX_SEL) {
        if (split == 0 && tid == 0) set_error(p.err, QSA_DEVERR_SELECTION);
        bad = true;
      } else {
        list = p.list + (int64_t)row * p.list_stride;
        nbase = n;
      }
    }
  }
  const int ext0 = (!bad && p.extra_base) ? __ldg(p.extra_base + row) : 0;
  const int ntot = bad ? 0 : nbase + (p.extra_base ? p.n_extra : 0);
  const int tiles = ceil_div(ntot, GQ_TILE);
  int tps = ceil_div(tiles, p.splits);
  if (tps > p.tiles_per_split) {  // more positions than the host bound it was sized for
    if (split == 0 && tid == 0) set_error(p.err, QSA_DEVERR_SELECTION);
    tps = p.tiles_per_split;
  }
  const int t_begin = min(tiles, split * tps), t_end = min(tiles, t_begin + tps);
  const int ntl = t_end - t_begin;

  auto position = [&](int j) -> int {
    if (j < nbase) {
      if (list) return __ldg(list + j);
      return j < nsel4 ? __ldcg(sel + (j >> 2)) * CBLK + (j & 3) : tail0 + (j - nsel4);
    }
    return ext0 + (j - nbase);
  };

  // ---- physical slots of this CTA's positions, resolved once up front ----
  if (p.mode == 0 && !p.extra_base) {
    // kept blocks: the 4 positions of a block are 4 consecutive slots of one page (a page holds 16
    // whole blocks), so one thread per block makes one selection read and one page-table read
    // (a tile of 16 positions is 4 blocks; the tail positions 4 * floor(L/4) .. L-1 follow the blocks)
    const int nsel = nsel4 >> 2;
    for (int i = tid; i < ntl * (GQ_TILE / 4); i += THREADS) {
      const int bi = t_begin * (GQ_TILE / 4) + i;  // block slot in the row's position order
      int32_t s4[4] = {-1, -1, -1, -1};
      if (bi < nsel) {
        const int64_t s0 = slot_of(p.c, req, __ldcg(sel + bi) * CBLK, p.err);
        if (s0 >= 0) {
#pragma unroll
          for (int e = 0; e < 4; ++e) s4[e] = (int32_t)(s0 + e);
        }
      } else {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int jj = 4 * bi + e;
          if (jj < ntot) s4[e] = (int32_t)slot_of(p.c, req, tail0 + (jj - nsel4), p.err);
        }
      }
      *reinterpret_cast<int4*>(S.slot + 4 * i) = make_int4(s4[0], s4[1], s4[2], s4[3]);
    }
  } else {
    for (int j = tid; j < ntl * GQ_TILE; j += THREADS) {
      const int jj = t_begin * GQ_TILE + j;
      S.slot[j] = jj < ntot ? (int32_t)slot_of(p.c, req, position(jj), p.err) : -1;
    }
  }
  __syncthreads();

  // ---- async gather of one tile into a stage ----
  auto issue_tile = [&](int t, int stage) {
    uint8_t* dst0 = S.kv[stage];
    const int32_t* tslot = S.slot + (t - t_begin) * GQ_TILE;
    if constexpr (!F8) {
      // chunk id c in [0, 1024): kv = c >> 9, pos j = (c >> 5) & 15, group = (c >> 4) & 1, 16 B chunk = c & 15
      constexpr int PER = 1024 / THREADS;  // chunks per thread
#pragma unroll
      for (int k = 0; k < PER; ++k) {
        const int c = tid + k * THREADS;
        const int kvsel = c >> 9, j = (c >> 5) & 15, g = (c >> 4) & 1, ch = c & 15;
        const int64_t sl = tslot[j];
        const __nv_bfloat16* base = kvsel ? p.c.v : p.c.k;
        const __nv_bfloat16* src = sl >= 0 ? base + sl * p.c.kv_stride + g * D + ch * 8 : base;
        uint8_t* dst = dst0 + kvsel * GQ_KV_BYTES + g * (GQ_TILE * GQ_ROW_BYTES) + j * GQ_ROW_BYTES + swz(j, ch);
        cp_async_16(dst, src, sl >= 0 ? 16 : 0);
      }
    } else {
      // chunk id c in [0, 512): kv = c >> 8, pos j = (c >> 4) & 15, group = (c >> 3) & 1, 16 B chunk = c & 7;
      // rows of 128 B, kv_stride counted in bytes
      constexpr int PER = 512 / THREADS;
#pragma unroll
      for (int k = 0; k < PER; ++k) {
        const int c = tid + k * THREADS;
        const int kvsel = c >> 8, j = (c >> 4) & 15, g = (c >> 3) & 1, ch = c & 7;
        const int64_t sl = tslot[j];
        const uint8_t* base = reinterpret_cast<const uint8_t*>(kvsel ? p.c.v : p.c.k);
        const uint8_t* src = sl >= 0 ? base + sl * p.c.kv_stride + g * D + ch * 16 : base;
        // K rows: chunk ch of position j at chunk ch ^ (j & 7), so that the fragment loads of 8 positions
        // at one dim offset hit 8 different bank groups
        uint8_t* dst = dst0 + kvsel * (GQ_KV_BYTES / 2) + g * (GQ_TILE * D) + j * D + ((kvsel ? ch : ch ^ (j & 7)) << 4);
        cp_async_16(dst, src, sl >= 0 ? 16 : 0);
      }
    }
  };

  // prologue of the pipeline
  constexpr int NST = Smem::STAGES;
#pragma unroll
  for (int k = 0; k < NST - 1; ++k) {
    if (k < ntl) issue_tile(t_begin + k, k);
    cp_async_commit();
  }
  __syncthreads();  // queries in shared memory

  // ---- warp role and its query fragments ----
  const int g = warp & 1, dh = (warp >> 1) & 1, mt = warp >> 2;
  const int gq = lane >> 2, cq = lane & 3;
  uint32_t qa[8][4];
  if constexpr (!F8) {
    const int mtx = lane >> 3;
    const int rho = mt * 16 + (lane & 7) + ((mtx & 1) << 3);
#pragma unroll
    for (int j = 0; j < 8; ++j)
      ldmatrix_x4(qa[j][0], qa[j][1], qa[j][2], qa[j][3], smem_u32(S.qrow(g, rho) + swz(rho, 2 * j + (mtx >> 1))));
  } else {
    // k-step j, lane (gq, cq): MMA k = 2cq, 2cq+1 are dims 16j + 4cq + {0, 1}, k = 2cq+8, 2cq+9 are
    // dims 16j + 4cq + {2, 3} (the order the K fragments are read in below)
    const int r0 = mt * 16 + gq, r1 = r0 + 8;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int ch = 2 * j + (cq >> 1), off = (cq & 1) * 8;
      qa[j][0] = *reinterpret_cast<const uint32_t*>(S.qrow(g, r0) + swz(r0, ch) + off);
      qa[j][1] = *reinterpret_cast<const uint32_t*>(S.qrow(g, r1) + swz(r1, ch) + off);
      qa[j][2] = *reinterpret_cast<const uint32_t*>(S.qrow(g, r0) + swz(r0, ch) + off + 4);
      qa[j][3] = *reinterpret_cast<const uint32_t*>(S.qrow(g, r1) + swz(r1, ch) + off + 4);
    }
  }
  const int qi0 = (mt * 16 + gq) >> 3, qi1 = (mt * 16 + gq + 8) >> 3;  // query of rows gq, gq+8
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  float o[8][4];
#pragma unroll
  for (int n = 0; n < 8; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;

  for (int it = 0; it < ntl; ++it) {
    cp_async_wait<NST - 2>();
    __syncthreads();
    if (it + NST - 1 < ntl) issue_tile(t_begin + it + NST - 1, (it + NST - 1) % NST);
    cp_async_commit();

    const int stage = it % NST;
    const int t = t_begin + it;
    const uint8_t* tile = S.kv[stage];
    // S = Q K^T : 16 rows x 16 positions
    float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    const uint8_t* vbase;  // this warp's V rows (bf16, rows swizzled), and the row size and chunk base
    int vrow, vch0;
    if constexpr (!F8) {
      const uint8_t* kbase = tile + g * (GQ_TILE * GQ_ROW_BYTES);
      vbase = tile + GQ_KV_BYTES + g * (GQ_TILE * GQ_ROW_BYTES);
      vrow = GQ_ROW_BYTES;
      vch0 = dh * 8;
      const int mtx = lane >> 3;
      const int pj = (lane & 7) + ((mtx >> 1) << 3);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        uint32_t b0, b1, b2, b3;
        ldmatrix_x4(b0, b1, b2, b3, smem_u32(kbase + pj * GQ_ROW_BYTES + swz(pj, 2 * j + (mtx & 1))));
        mma_bf16_16816(s[0], qa[j], b0, b1);
        mma_bf16_16816(s[1], qa[j], b2, b3);
      }
    } else {
      // this warp's half of its group's V (dims dh*64 .. +63) -> bf16 in its own buffer: lane l converts
      // the 32 values of position l/2, dims dh*64 + 32 (l&1) .. +31
      uint8_t* vb = S.cvt + warp * Smem::VBUF;
      {
        const int pos = lane >> 1, hf = lane & 1;
        const uint4* src = reinterpret_cast<const uint4*>(tile + GQ_KV_BYTES / 2 + g * (GQ_TILE * D) + pos * D +
                                                          dh * 64 + hf * 32);
        const uint4 a = src[0], b = src[1];
        uint8_t* dst = vb + pos * (GQ_ROW_BYTES / 2);
        *reinterpret_cast<uint4*>(dst + swz(pos, 4 * hf + 0)) = e4m3x8_to_bf16x8(make_uint2(a.x, a.y));
        *reinterpret_cast<uint4*>(dst + swz(pos, 4 * hf + 1)) = e4m3x8_to_bf16x8(make_uint2(a.z, a.w));
        *reinterpret_cast<uint4*>(dst + swz(pos, 4 * hf + 2)) = e4m3x8_to_bf16x8(make_uint2(b.x, b.y));
        *reinterpret_cast<uint4*>(dst + swz(pos, 4 * hf + 3)) = e4m3x8_to_bf16x8(make_uint2(b.z, b.w));
      }
      vbase = vb;
      vrow = GQ_ROW_BYTES / 2;
      vch0 = 0;
      // K fragments straight from the fp8 rows: lane (gq, cq) reads dims 16j + 4cq .. +3 of positions gq
      // and gq + 8 (chunk j of a row sits at chunk j ^ (pos & 7))
      const uint8_t* k0 = tile + g * (GQ_TILE * D) + gq * D + 4 * cq;
      const uint8_t* k1 = k0 + 8 * D;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const uint32_t w0 = *reinterpret_cast<const uint32_t*>(k0 + ((j ^ (gq & 7)) << 4));
        const uint32_t w1 = *reinterpret_cast<const uint32_t*>(k1 + ((j ^ (gq & 7)) << 4));
        mma_bf16_16816(s[0], qa[j], e4m3x2_to_bf16x2((uint16_t)(w0 & 0xFFFFu)), e4m3x2_to_bf16x2((uint16_t)(w0 >> 16)));
        mma_bf16_16816(s[1], qa[j], e4m3x2_to_bf16x2((uint16_t)(w1 & 0xFFFFu)), e4m3x2_to_bf16x2((uint16_t)(w1 >> 16)));
      }
      __syncwarp();  // the warp's V buffer is written
    }
    // mask, scale (log2 domain), online softmax
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
    for (int n = 0; n < 2; ++n)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int jj = t * GQ_TILE + 8 * n + 2 * cq + e;
        const int ex = jj - nbase;  // >= 0: a drafted position, seen by queries ex..
        const bool ok0 = jj < ntot && (ex < 0 || ex <= qi0);
        const bool ok1 = jj < ntot && (ex < 0 || ex <= qi1);
        s[n][e] = ok0 ? s[n][e] * p.scale_log2 : -INFINITY;
        s[n][2 + e] = ok1 ? s[n][2 + e] * p.scale_log2 : -INFINITY;
        mx0 = fmaxf(mx0, s[n][e]);
        mx1 = fmaxf(mx1, s[n][2 + e]);
      }
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
    const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
    const float base0 = mn0 == -INFINITY ? 0.f : mn0, base1 = mn1 == -INFINITY ? 0.f : mn1;
    const float c0 = exp2f(m0 - base0), c1 = exp2f(m1 - base1);
    m0 = mn0;
    m1 = mn1;
    float pr[2][4];
#pragma unroll
    for (int n = 0; n < 2; ++n) {
      pr[n][0] = exp2f(s[n][0] - base0);
      pr[n][1] = exp2f(s[n][1] - base0);
      pr[n][2] = exp2f(s[n][2] - base1);
      pr[n][3] = exp2f(s[n][3] - base1);
    }
    l0 = l0 * c0 + (pr[0][0] + pr[0][1] + pr[1][0] + pr[1][1]);
    l1 = l1 * c1 + (pr[0][2] + pr[0][3] + pr[1][2] + pr[1][3]);
#pragma unroll
    for (int n = 0; n < 8; ++n) {
      o[n][0] *= c0;
      o[n][1] *= c0;
      o[n][2] *= c1;
      o[n][3] *= c1;
    }
    uint32_t pa[4];
    pa[0] = pack_bf16x2(pr[0][0], pr[0][1]);
    pa[1] = pack_bf16x2(pr[0][2], pr[0][3]);
    pa[2] = pack_bf16x2(pr[1][0], pr[1][1]);
    pa[3] = pack_bf16x2(pr[1][2], pr[1][3]);
    // O += P V over this warp's 64 dims
    {
      const int mtx = lane >> 3;
      const int pj = (lane & 7) + ((mtx & 1) << 3);
#pragma unroll
      for (int pp = 0; pp < 4; ++pp) {
        const int ch = vch0 + pp * 2 + (mtx >> 1);
        uint32_t b0, b1, b2, b3;
        ldmatrix_x4_trans(b0, b1, b2, b3, smem_u32(vbase + pj * vrow + swz(pj, ch)));
        mma_bf16_16816(o[2 * pp], pa, b0, b1);
        mma_bf16_16816(o[2 * pp + 1], pa, b2, b3);
      }
    }
  }
  cp_async_wait<0>();
  if constexpr (F8) {  // the V scale, applied once to the unnormalised sums
#pragma unroll
    for (int n = 0; n < 8; ++n) {
      o[n][0] *= p.v_scale;
      o[n][1] *= p.v_scale;
      o[n][2] *= p.v_scale;
      o[n][3] *= p.v_scale;
    }
  }

  // ---- finish: full row sums, then write the result or a partial ----
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
  const int rho0 = mt * 16 + gq, rho1 = rho0 + 8;
  const int h0 = g * GROUP + (rho0 & 7), h1 = g * GROUP + (rho1 & 7);
  const int nh = nq * HQ;
  if (p.splits == 1) {
    if (p.row_ready && tid == 0) p.row_ready[row * READY_STRIDE] = 0;  // ready for the next call
    const float i0 = l0 > 0.f ? 1.f / l0 : 0.f, i1 = l1 > 0.f ? 1.f / l1 : 0.f;
    __nv_bfloat16* out = p.out + (int64_t)row * nh * D;
#pragma unroll
    for (int n = 0; n < 8; ++n) {
      const int d = dh * 64 + 8 * n + 2 * cq;
      if (qi0 < nq)
        *reinterpret_cast<uint32_t*>(out + ((int64_t)qi0 * HQ + h0) * D + d) = pack_bf16x2(o[n][0] * i0, o[n][1] * i0);
      if (qi1 < nq)
        *reinterpret_cast<uint32_t*>(out + ((int64_t)qi1 * HQ + h1) * D + d) = pack_bf16x2(o[n][2] * i1, o[n][3] * i1);
    }
    if (p.lse && dh == 0 && cq == 0) {
      constexpr float LN2 = 0.69314718055994530942f;
      if (qi0 < nq) p.lse[(int64_t)row * nh + qi0 * HQ + h0] = l0 > 0.f ? (m0 + log2f(l0)) * LN2 : -INFINITY;
      if (qi1 < nq) p.lse[(int64_t)row * nh + qi1 * HQ + h1] = l1 > 0.f ? (m1 + log2f(l1)) * LN2 : -INFINITY;
    }
    return;
  }
  if (Smem::CLUSTER_FITS && p.cluster_merge) {
    namespace cg = cooperative_groups;
    cg::cluster_group cl = cg::this_cluster();
    // own partial into the (now idle) ring: O [heads][128] fp32, then (m, l) per head
    __syncthreads();  // every warp is done with the ring
    float* po_s = reinterpret_cast<float*>(S.area());
    float* pml_s = Smem::ML_IN_RING ? po_s + 32 * MT * D : reinterpret_cast<float*>(S.qsep);
#pragma unroll
    for (int n = 0; n < 8; ++n) {
      const int d = dh * 64 + 8 * n + 2 * cq;
      if (qi0 < nq) *reinterpret_cast<float2*>(po_s + (qi0 * HQ + h0) * D + d) = make_float2(o[n][0], o[n][1]);
      if (qi1 < nq) *reinterpret_cast<float2*>(po_s + (qi1 * HQ + h1) * D + d) = make_float2(o[n][2], o[n][3]);
    }
    if (dh == 0 && cq == 0) {
      if (qi0 < nq) *reinterpret_cast<float2*>(pml_s + (qi0 * HQ + h0) * 2) = make_float2(m0, l0);
      if (qi1 < nq) *reinterpret_cast<float2*>(pml_s + (qi1 * HQ + h1) * 2) = make_float2(m1, l1);
    }
    cl.sync();
    // this CTA's slice of (head, 4 dims) items, merged from every split's shared memory
    const int ns = p.splits;  // the cluster size
    const int rank = (int)cl.block_rank();
    const int nitems = nh * (D / 4);
    const int per = ceil_div(nitems, ns);
    const int i_end = min(nitems, (rank + 1) * per);
    __nv_bfloat16* out = p.out + (int64_t)row * nh * D;
    for (int idx = rank * per + tid; idx < i_end; idx += THREADS) {
      const int hh = idx / (D / 4), c4 = idx % (D / 4);
      float2 ml[GQ_CLUSTER_MAX];
      float4 ov[GQ_CLUSTER_MAX];
#pragma unroll
      for (int s2 = 0; s2 < GQ_CLUSTER_MAX; ++s2) {
        ml[s2] = make_float2(-INFINITY, 0.f);
        ov[s2] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (s2 < ns) {
          ml[s2] = *reinterpret_cast<const float2*>(cl.map_shared_rank(pml_s, s2) + hh * 2);
          ov[s2] = *reinterpret_cast<const float4*>(cl.map_shared_rank(po_s, s2) + hh * D + c4 * 4);
        }
      }
      float M = -INFINITY;
#pragma unroll
      for (int s2 = 0; s2 < GQ_CLUSTER_MAX; ++s2) M = fmaxf(M, ml[s2].x);
      const float base = M == -INFINITY ? 0.f : M;
      float den = 0.f;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int s2 = 0; s2 < GQ_CLUSTER_MAX; ++s2) {
        const float wgt = exp2f(ml[s2].x - base);  // 0 for splits without positions
        den += wgt * ml[s2].y;
        acc.x += wgt * ov[s2].x;
        acc.y += wgt * ov[s2].y;
        acc.z += wgt * ov[s2].z;
        acc.w += wgt * ov[s2].w;
      }
      const float inv = den > 0.f ? 1.f / den : 0.f;
      uint2 pk;
      pk.x = pack_bf16x2(acc.x * inv, acc.y * inv);
      pk.y = pack_bf16x2(acc.z * inv, acc.w * inv);
      *reinterpret_cast<uint2*>(out + (int64_t)hh * D + c4 * 4) = pk;
      if (p.lse && c4 == 0) {
        constexpr float LN2 = 0.69314718055994530942f;
        p.lse[(int64_t)row * nh + hh] = den > 0.f ? (M + log2f(den)) * LN2 : -INFINITY;
      }
    }
    cl.sync();  // no CTA leaves while another still reads its shared memory
    if (rank == 0 && tid == 0 && p.row_ready) p.row_ready[row * READY_STRIDE] = 0;  // ready for the next call
    return;
  }
  float* po = p.part_o + ((int64_t)row * p.splits + split) * nh * D;
  float* pml = p.part_ml + ((int64_t)row * p.splits + split) * nh * 2;
#pragma unroll
  for (int n = 0; n < 8; ++n) {
    const int d = dh * 64 + 8 * n + 2 * cq;
    if (qi0 < nq) *reinterpret_cast<float2*>(po + ((int64_t)qi0 * HQ + h0) * D + d) = make_float2(o[n][0], o[n][1]);
    if (qi1 < nq) *reinterpret_cast<float2*>(po + ((int64_t)qi1 * HQ + h1) * D + d) = make_float2(o[n][2], o[n][3]);
  }
  if (dh == 0 && cq == 0) {
    if (qi0 < nq) *reinterpret_cast<float2*>(pml + (qi0 * HQ + h0) * 2) = make_float2(m0, l0);
    if (qi1 < nq) *reinterpret_cast<float2*>(pml + (qi1 * HQ + h1) * 2) = make_float2(m1, l1);
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) S.is_last = atomicAdd(p.counters + row, 1) == p.splits - 1;
  __syncthreads();
  if (!S.is_last) return;
  __threadfence();
  // merge.  Every load of a step is issued before any is used: (a) per head, the (m, l) of all
  // splits give normalized split weights (kept in the now idle ring); (b) per (head, 4 dims), the
  // weighted sum over splits, four splits x four items of loads in flight per thread.
  const float* pob = p.part_o + (int64_t)row * p.splits * nh * D;
  const float* pmb = p.part_ml + (int64_t)row * p.splits * nh * 2;
  __nv_bfloat16* out = p.out + (int64_t)row * nh * D;
  float* wsm = reinterpret_cast<float*>(S.area());  // [nh][GQ_MAX_SPLITS]
  const int splits = p.splits;
  for (int hh = tid; hh < nh; hh += THREADS) {
    float mv[GQ_MAX_SPLITS], lv[GQ_MAX_SPLITS];
#pragma unroll
    for (int s2 = 0; s2 < GQ_MAX_SPLITS; ++s2) {
      float2 ml = make_float2(-INFINITY, 0.f);
      if (s2 < splits) ml = __ldcg(reinterpret_cast<const float2*>(pmb + ((int64_t)s2 * nh + hh) * 2));
      mv[s2] = ml.x;
      lv[s2] = ml.y;
    }
    float M = -INFINITY;
#pragma unroll
    for (int s2 = 0; s2 < GQ_MAX_SPLITS; ++s2) M = fmaxf(M, mv[s2]);
    const float base = M == -INFINITY ? 0.f : M;
    float den = 0.f;
#pragma unroll
    for (int s2 = 0; s2 < GQ_MAX_SPLITS; ++s2) {
      mv[s2] = exp2f(mv[s2] - base);  // 0 for unused splits
      den += mv[s2] * lv[s2];
    }
    const float inv = den > 0.f ? 1.f / den : 0.f;
#pragma unroll
    for (int s2 = 0; s2 < GQ_MAX_SPLITS; ++s2) wsm[hh * GQ_MAX_SPLITS + s2] = mv[s2] * inv;
    if (p.lse) {
      constexpr float LN2 = 0.69314718055994530942f;
      p.lse[(int64_t)row * nh + hh] = den > 0.f ? (M + log2f(den)) * LN2 : -INFINITY;
    }
  }
  __syncthreads();
  constexpr int IT = 4;  // items per thread in flight
  const int nitems = nh * (D / 4);
  for (int idx0 = 0; idx0 < nitems; idx0 += IT * THREADS) {
    float4 acc[IT];
#pragma unroll
    for (int i = 0; i < IT; ++i) acc[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s0 = 0; s0 < splits; s0 += 4) {
      float4 v[IT][4];
#pragma unroll
      for (int i = 0; i < IT; ++i)
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int idx = idx0 + i * THREADS + tid, s2 = s0 + u;
          v[i][u] = make_float4(0.f, 0.f, 0.f, 0.f);
          if (idx < nitems && s2 < splits)
            v[i][u] = __ldcg(reinterpret_cast<const float4*>(pob + ((int64_t)s2 * nh + idx / (D / 4)) * D +
                                                              (idx % (D / 4)) * 4));
        }
#pragma unroll
      for (int i = 0; i < IT; ++i)
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int idx = idx0 + i * THREADS + tid, s2 = s0 + u;
          if (idx < nitems && s2 < splits) {
            const float wgt = wsm[(idx / (D / 4)) * GQ_MAX_SPLITS + s2];
            acc[i].x += wgt * v[i][u].x;
            acc[i].y += wgt * v[i][u].y;
            acc[i].z += wgt * v[i][u].z;
            acc[i].w += wgt * v[i][u].w;
          }
        }
    }
#pragma unroll
    for (int i = 0; i < IT; ++i) {
      const int idx = idx0 + i * THREADS + tid;
      if (idx < nitems) {
        uint2 pk;
        pk.x = pack_bf16x2(acc[i].x, acc[i].y);
        pk.y = pack_bf16x2(acc[i].z, acc[i].w);
        *reinterpret_cast<uint2*>(out + (int64_t)(idx / (D / 4)) * D + (idx % (D / 4)) * 4) = pk;
      }
    }
  }
  if (tid == 0) {
    p.counters[row] = 0;  // ready for the next call
    if (p.row_ready) p.row_ready[row * READY_STRIDE] = 0;
  }
}

// Workspace bound on the split count (no device needed): at most 8 resident
// CTAs per SM on at most 256 SMs.
int gqa_split_bound(int rows, int max_pos) {
  const int tiles = ceil_div(max(max_pos, 1), GQ_TILE);
  int s = ceil_div(8 * 256, rows > 0 ? rows : 1);
  s = min(s, max(1, tiles / 2));
  return max(1, min(s, GQ_MAX_SPLITS));
}

template <int MT, bool F8>
static size_t gqa_smem_bytes(int tiles_per_split) {
  return sizeof(GqaSmem<MT, F8>) + sizeof(int32_t) * (size_t)tiles_per_split * GQ_TILE + 128;
}

template <int MT, bool F8>
static int occupancy(size_t smem) {
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k_sparse_gqa<MT, F8>, MT * 128, smem) != cudaSuccess) return 1;
  return max(n, 1);
}

// Splits so that the grid is one wave of resident CTAs (rows x splits <=
// resident CTAs per SM x SMs), each split at least two tiles.
template <int MT, bool F8>
static void choose_splits(int rows, int max_pos, int num_sms, int bound, int& splits, int& tps) {
  const int tiles = ceil_div(max(max_pos, 1), GQ_TILE);
  rows = max(rows, 1);
  for (int occ_try = 8; occ_try >= 1; --occ_try) {
    int s = (occ_try * num_sms) / rows;
    s = max(1, min(s, min(max(1, tiles / 2), min(bound, GQ_MAX_SPLITS))));
    const int t = ceil_div(tiles, s);
    if (occupancy<MT, F8>(gqa_smem_bytes<MT, F8>(t)) >= occ_try || occ_try == 1) {
      splits = s;
      tps = t;
      return;
    }
  }
  splits = 1;
  tps = tiles;
}

// Clusters of `splits` CTAs, each with `smem` bytes of dynamic shared memory, that can be resident at
// once (device query, cached per device for a few (splits, smem) pairs).
#ifndef QSA_GQA_CLUSTER_SLACK
#define QSA_GQA_CLUSTER_SLACK 0  // percent of the cluster slots left free
#endif
template <int MT, bool F8>
static int active_clusters(int splits, size_t smem) {
  struct Entry {
    int splits;
    size_t smem;
    int n;
  };
  constexpr int CAP = 32;
  static Entry cache[64][CAP] = {};
  static std::mutex mu;
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64 || splits < 1 || splits > GQ_CLUSTER_MAX) return 0;
  {
    std::lock_guard<std::mutex> lk(mu);
    for (const Entry& e : cache[dev])
      if (e.splits == splits && e.smem == smem) return e.n;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(splits, 1);
  cfg.blockDim = dim3(MT * 128);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)splits;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, k_sparse_gqa<MT, F8>, &cfg) != cudaSuccess) {
    cudaGetLastError();
    n = 0;
  }
  std::lock_guard<std::mutex> lk(mu);
  for (Entry& e : cache[dev])
    if (e.splits == 0) {
      e = Entry{splits, smem, n};
      break;
    }
  return n;
}

template <int MT, bool F8>
static cudaError_t launch_mt(GqaParams p, int rows, int max_pos, int num_sms, int bound, cudaStream_t st) {
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  const size_t smem_max = gqa_smem_bytes<MT, F8>(GQ_MAX_TILES);
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    const cudaError_t e =
        cudaFuncSetAttribute(k_sparse_gqa<MT, F8>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_max);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  choose_splits<MT, F8>(rows, max_pos, num_sms, p.cluster_merge ? min(bound, GQ_CLUSTER_MAX) : bound, p.splits,
                    p.tiles_per_split);
  if (!GqaSmem<MT, F8>::CLUSTER_FITS) p.cluster_merge = 0;
  if (p.cluster_merge) {
    // every row's cluster resident at once (QSA_GQA_CLUSTER_SLACK percent of the slots spare): a
    // cluster that finds no GPC with room for all its CTAs waits a whole CTA lifetime for one
    const int tiles = ceil_div(max(max_pos, 1), GQ_TILE);
    while (p.splits >= 2 &&
           (int64_t)rows * 100 > (int64_t)active_clusters<MT, F8>(p.splits, gqa_smem_bytes<MT, F8>(p.tiles_per_split)) *
                                     (100 - QSA_GQA_CLUSTER_SLACK)) {
      --p.splits;
      p.tiles_per_split = ceil_div(tiles, p.splits);
    }
  }
  if (p.splits < 2 || p.splits > GQ_CLUSTER_MAX) p.cluster_merge = 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.splits, rows);
  cfg.blockDim = dim3(MT * 128);
  cfg.dynamicSmemBytes = gqa_smem_bytes<MT, F8>(p.tiles_per_split);
  cfg.stream = st;
  cudaLaunchAttribute attr[3];
  int na = 0;
  if (p.row_ready) {  // may start before the scorer ends; each CTA waits for its row's flag
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  if (p.cluster_merge) {  // one cluster per row: its splits
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = (unsigned)p.splits;
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = 1;
    ++na;
  }
  if (p.cluster_merge) {
    // Clusters placed for load balance: while the decode scorer's CTAs exit, a cluster otherwise often
    // waits for a GPC with room for all its CTAs (measured: the mean decode step falls from 145.3 to
    // 143.0 us at the same median, 90th percentile 162.8 -> 144.5 us).
    attr[na].id = cudaLaunchAttributeClusterSchedulingPolicyPreference;
    attr[na].val.clusterSchedulingPolicyPreference = cudaClusterSchedulingPolicyLoadBalancing;
    ++na;
  }
  cfg.attrs = na ? attr : nullptr;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, k_sparse_gqa<MT, F8>, p);
}

cudaError_t launch_gqa(const GqaParams& p, int rows, int max_pos, int num_sms, int split_bound, cudaStream_t st) {
  const int mt = ceil_div(p.nq_row * GROUP, 16);
  if (p.fp8) {
    switch (mt) {
      case 1: return launch_mt<1, true>(p, rows, max_pos, num_sms, split_bound, st);
      case 2: return launch_mt<2, true>(p, rows, max_pos, num_sms, split_bound, st);
      case 3:
      case 4: return launch_mt<4, true>(p, rows, max_pos, num_sms, split_bound, st);
      default: return cudaErrorInvalidValue;
    }
  }
  switch (mt) {
    case 1: return launch_mt<1, false>(p, rows, max_pos, num_sms, split_bound, st);
    case 2: return launch_mt<2, false>(p, rows, max_pos, num_sms, split_bound, st);
    case 3:
    case 4: return launch_mt<4, false>(p, rows, max_pos, num_sms, split_bound, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace qsa
