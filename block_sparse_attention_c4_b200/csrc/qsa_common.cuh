// Shared device helpers of the QSA c4 kernels (sm_100a): constants, bf16
// conversions, inline-PTX wrappers (mbarrier, TMA, ldmatrix, mma, cp.async),
// block scans and the CTA-wide radix select used by the top-512.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/qsa.h"

namespace qsa {

constexpr int D = QSA_HEAD_DIM;        // 128
constexpr int HI = QSA_INDEX_HEADS;    // 4
constexpr int HQ = QSA_Q_HEADS;        // 16
constexpr int HKV = QSA_KV_HEADS;      // 2
constexpr int GROUP = HQ / HKV;        // 8 query heads per KV head
constexpr int CBLK = QSA_BLOCK;        // 4 tokens per compressed block
constexpr int TOPK = QSA_TOPK;         // 512
constexpr int PAGE = QSA_PAGE_SIZE;    // 64 tokens per page
constexpr int PAGE_BLOCKS = PAGE / CBLK;  // 16 compressed entries per page
constexpr int MAX_SEL = QSA_MAX_SEL;   // 2051

// Everything a kernel needs to know about the cache, by value.
struct CacheView {
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  __nv_bfloat16* cidx;
  __nv_bfloat16* ring;
  const int32_t* page_table;
  int64_t num_pages;
  int64_t kv_stride;  // bf16 elements from one slot's K (or V) rows to the next slot's
  int32_t max_pages;
  int32_t batch;
};

// RoPE inverse frequencies theta^(-i/64), i < 64, computed on the host in FP64.
struct RopeFreqs {
  double f[D / 2];
};

__device__ __forceinline__ void set_error(int* err, int bits) {
  if (err) atomicOr(err, bits);
}

// Physical slot of logical position `pos` of request `req`, or -1 (and an
// error bit) when the page is outside the table or the pool.
__device__ __forceinline__ int64_t slot_of(const CacheView& c, int req, int pos, int* err) {
  const int lp = pos >> 6;
  if (pos < 0 || lp >= c.max_pages) {
    set_error(err, QSA_DEVERR_POSITION);
    return -1;
  }
  const int phys = __ldg(c.page_table + (int64_t)req * c.max_pages + lp);
  if (phys < 0 || phys >= c.num_pages) {
    set_error(err, QSA_DEVERR_PAGE);
    return -1;
  }
  return (int64_t)phys * PAGE + (pos & (PAGE - 1));
}

// ---------------------------------------------------------------------------
// bf16 conversions
// ---------------------------------------------------------------------------
__device__ __forceinline__ float bf16_bits_to_f32(uint16_t h) { return __uint_as_float((uint32_t)h << 16); }

// FP64 -> bf16 bits, rounding once to nearest even at the 8th significant bit
// (integer arithmetic on the FP64 encoding).  Valid in float's normal range,
// which covers every value the kernels round (unit-norm keys, rotated queries).
__device__ __forceinline__ uint16_t f64_to_bf16_bits(double x) {
  unsigned long long b = (unsigned long long)__double_as_longlong(x);
  const unsigned long long lsb = (b >> 45) & 1ull;
  b += ((1ull << 44) - 1ull) + lsb;
  b &= ~((1ull << 45) - 1ull);
  const float f = __double2float_rn(__longlong_as_double((long long)b));  // exact now
  return (uint16_t)(__float_as_uint(f) >> 16);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Order-preserving map float -> uint32 (larger float, larger key); -0 == +0.
__device__ __forceinline__ uint32_t score_key(float s) {
  uint32_t u = __float_as_uint(s);
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float key_score(uint32_t k) {
  const uint32_t u = (k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k;
  return __uint_as_float(u);
}

// ---------------------------------------------------------------------------
// Block compression (blog section "Qwen Sparse Attention: Retrieve Coarsely,
// Attend Precisely"): the mean of 4 raw index keys as an FP32 sum in token
// order times 1/4, divided by its L2 norm and rotated at the block's first
// position in FP64 (host-computed inverse frequencies), rounded once to bf16.
// ---------------------------------------------------------------------------
// One warp compresses one block.  Lane l owns dims l, l+32, l+64, l+96, i.e.
// the rotation pairs (l, l+64) and (l+32, l+96), so the rotation needs no
// exchange.  `keys4[j]` points at the raw key of token 4b+j.
__device__ __forceinline__ void warp_compress_block(const __nv_bfloat16* const keys4[4], int64_t b,
                                                    const RopeFreqs& fr, __nv_bfloat16* out) {
  const int lane = threadIdx.x & 31;
  float m[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const int d = lane + 32 * e;
    float s = __bfloat162float(keys4[0][d]);
    s = s + __bfloat162float(keys4[1][d]);
    s = s + __bfloat162float(keys4[2][d]);
    s = s + __bfloat162float(keys4[3][d]);
    m[e] = s * 0.25f;
  }
  double n2 = 0.0;
#pragma unroll
  for (int e = 0; e < 4; ++e) n2 += (double)m[e] * (double)m[e];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) n2 += __shfl_xor_sync(0xffffffffu, n2, o);
  const double nrm = sqrt(n2);
  double kh[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) kh[e] = nrm > 0.0 ? (double)m[e] / nrm : 0.0;
  const double p = (double)(CBLK * b);
  uint16_t res[4];
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    const int i = lane + 32 * e;  // pair (i, i + 64): kh[e] and kh[e + 2]
    double sn, cs;
    sincos(p * fr.f[i], &sn, &cs);
    const double x0 = kh[e], x1 = kh[e + 2];
    res[e] = f64_to_bf16_bits(x0 * cs - x1 * sn);
    res[e + 2] = f64_to_bf16_bits(x0 * sn + x1 * cs);
  }
  uint16_t* o = reinterpret_cast<uint16_t*>(out);
#pragma unroll
  for (int e = 0; e < 4; ++e) o[lane + 32 * e] = res[e];
}

__device__ __forceinline__ int64_t cidx_entry(const CacheView& c, int req, int64_t b, int* err) {
  const int64_t s = slot_of(c, req, (int)(CBLK * b), err);
  return s < 0 ? -1 : s / CBLK;
}

// Decode append of one row (one warp): the new index key of position L-1 goes to ring slot
// (L-1) mod 4, and when it completes block b = L/4 - 1 that block is compressed from ring slots
// 0..2 and the new key.
__device__ __forceinline__ void warp_decode_append(const CacheView& c, int req, int L, const __nv_bfloat16* key,
                                                   const RopeFreqs& fr, int* err) {
  const int pos = L - 1;
  __nv_bfloat16* ring = c.ring + (int64_t)req * CBLK * D;
  if ((pos & 3) == 3) {
    const __nv_bfloat16* k4[4] = {ring, ring + D, ring + 2 * D, key};
    const int64_t b = pos >> 2;
    const int64_t e = cidx_entry(c, req, b, err);
    if (e >= 0) warp_compress_block(k4, b, fr, c.cidx + e * D);
    __syncwarp();
  }
  const uint32_t* src = reinterpret_cast<const uint32_t*>(key);
  uint32_t* dst = reinterpret_cast<uint32_t*>(ring + (pos & 3) * D);
  for (int i = threadIdx.x & 31; i < D / 2; i += 32) dst[i] = src[i];
}

// ---------------------------------------------------------------------------
// Shared-memory / async-copy PTX wrappers
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// The first A-aligned byte of the dynamic shared memory `raw`, derived by pointer arithmetic so
// that the compiler still knows every access through it to be a shared-memory access (rounding
// the address as an integer would turn them all into slower generic loads, stores and atomics).
template <int A>
__device__ __forceinline__ uint8_t* smem_aligned(uint8_t* raw) {
  return raw + ((A - (smem_u32(raw) & (A - 1))) & (A - 1));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(20000u)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

// Every wait inside a kernel is bounded: it gives up after `limit_ns` of wall time (the host passes
// WAIT_LIMIT_NS unless a diagnostic asks for a shorter limit), records QSA_DEVERR_TIMEOUT and returns
// false; the caller then proceeds without the data and the kernel ends.
constexpr uint64_t WAIT_LIMIT_NS = 2000000000ull;

// Cross-kernel readiness of one row (programmatic dependent launch): the producer publishes
// after its block barrier (release, GPU scope); a consumer thread waits for it (acquire).
// Returns whether the row became ready.
__device__ __forceinline__ void publish_ready(int* flag) {
  asm volatile("fence.acq_rel.gpu;\n\tst.release.gpu.global.b32 [%0], 1;" ::"l"(flag) : "memory");
}

__device__ __forceinline__ bool wait_ready(const int* flag, int* err, uint64_t limit_ns) {
  uint64_t t0 = 0;
  for (int spin = 0;; ++spin) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(flag) : "memory");
    if (v != 0) return true;
    if (spin == 0) {
      asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t0));
    } else if ((spin & 15) == 0) {
      uint64_t t;
      asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
      if (t - t0 > limit_ns) break;
    }
    __nanosleep(256);  // few polls: many CTAs may wait at once
  }
  set_error(err, QSA_DEVERR_TIMEOUT);
  return false;
}

// Row flags sit one per 128-byte line, so that waiting CTAs do not all poll the same L2 lines.
constexpr int READY_STRIDE = 32;

// Bounded mbarrier wait (see WAIT_LIMIT_NS).
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, int* err,
                                          uint64_t limit_ns = WAIT_LIMIT_NS) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (global_timer_ns() - t0 > limit_ns) break;
  }
  set_error(err, QSA_DEVERR_TIMEOUT);
  return false;
}

// 2-D tiled TMA load into this CTA's shared memory, completing on `bar`.
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cta.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::
          "r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3, uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3,
                                                  uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// D = A(16x16, row) * B(16x8, col) + C, bf16 inputs, f32 accumulate.
__device__ __forceinline__ void mma_bf16_16816(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// 16-byte cp.async global -> shared; src_bytes = 0 writes zeros.
#ifndef QSA_CP_L2_PROMOTE
#define QSA_CP_L2_PROMOTE 0
#endif
__device__ __forceinline__ void cp_async_16(void* dst, const void* src, int src_bytes) {
#if QSA_CP_L2_PROMOTE == 256
  asm volatile("cp.async.cg.shared.global.L2::256B [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src),
               "r"(src_bytes)
               : "memory");
#elif QSA_CP_L2_PROMOTE == 128
  asm volatile("cp.async.cg.shared.global.L2::128B [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src),
               "r"(src_bytes)
               : "memory");
#else
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(src_bytes)
               : "memory");
#endif
}

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }

template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// ---------------------------------------------------------------------------
// Thread groups: the first NT threads of the block, synchronising on named
// barrier BAR (BAR == 0: the whole block with __syncthreads).  Lets a subset of
// warps (e.g. the consumer warps of a warp-specialised kernel) run the
// collective helpers below while other warps keep working.
// ---------------------------------------------------------------------------
template <int NT, int BAR>
struct Group {
  static constexpr int N = NT;
  __device__ __forceinline__ static void sync() {
    if constexpr (BAR == 0) {
      __syncthreads();
    } else {
      asm volatile("bar.sync %0, %1;" ::"n"(BAR), "n"(NT) : "memory");
    }
  }
};

// Exclusive scan over the group.  `warp_tot` needs 33 ints of shared memory.
// Returns the exclusive prefix of `v`; *total gets the group total.
template <class G>
__device__ __forceinline__ int group_exclusive_scan(int v, int* warp_tot, int* total) {
  constexpr int NW = G::N / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_tot[warp] = x;
  G::sync();
  if (warp == 0) {
    int t = lane < NW ? warp_tot[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += y;
    }
    if (lane < NW) warp_tot[lane] = t;  // inclusive warp prefix
    if (lane == 31) warp_tot[32] = t;
  }
  G::sync();
  const int before = warp > 0 ? warp_tot[warp - 1] : 0;
  const int res = before + x - v;
  *total = warp_tot[32];
  G::sync();
  return res;
}

// The same with a single barrier: every thread adds up the warp totals before its own warp.  The
// caller must pass another barrier before `warp_tot` is written again.
template <class G>
__device__ __forceinline__ int group_exclusive_scan_1b(int v, int* warp_tot, int* total) {
  constexpr int NW = G::N / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_tot[warp] = x;
  G::sync();
  int before = 0, tot = 0;
#pragma unroll
  for (int w = 0; w < NW; ++w) {
    const int t = warp_tot[w];
    before += w < warp ? t : 0;
    tot += t;
  }
  *total = tot;
  return before + x - v;
}

// ---------------------------------------------------------------------------
// Exact top-k selection on 32-bit keys over a group (larger key first, then
// lower index first).
//
// radix_select: finds the masked prefix T with
//   count(key & mask > T) < k <= count(key & mask >= T)
// and `need`, how many elements with key & mask == T are still to be taken.
// It first reduces min and max to skip the high bits every key shares, then
// walks down in digits of up to 11 bits (2048-bin histograms, warp-aggregated
// shared-memory atomics), stopping early once the threshold bin is taken whole.
// select_compact: keeps every key & mask > T and the first `need` elements
// with key & mask == T in index order, emitting them in index order.
// KeyAt: int -> uint32 accessor; any n (the loops stride over the group).
// ---------------------------------------------------------------------------
constexpr int SEL_BINS = 2048;

struct SelectScratch {
  int hist[SEL_BINS];
  int warp_tot[33];
  int digit;
  int above;
  uint32_t kmin[32];
  uint32_t kmax[32];
};

struct SelectResult {
  uint32_t thresh;
  uint32_t mask;
  int need;
};

template <class G, typename KeyAt>
__device__ SelectResult radix_select(KeyAt key_at, int n, int k, SelectScratch* sc) {
  constexpr int NT = G::N;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // common high bits of all keys
  uint32_t mn = 0xFFFFFFFFu, mx = 0u;
  for (int i = tid; i < n; i += NT) {
    const uint32_t u = key_at(i);
    mn = min(mn, u);
    mx = max(mx, u);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    mn = min(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  if (lane == 0) {
    sc->kmin[warp] = mn;
    sc->kmax[warp] = mx;
  }
  G::sync();
  mn = sc->kmin[0];
  mx = sc->kmax[0];
  for (int w = 1; w < NT / 32; ++w) {
    mn = min(mn, sc->kmin[w]);
    mx = max(mx, sc->kmax[w]);
  }
  G::sync();
  if (mn == mx) return SelectResult{mx, 0xFFFFFFFFu, k};  // all keys equal: the first k by index
  int hb = 31 - __clz(mn ^ mx);                           // highest bit that differs
  uint32_t mask = hb == 31 ? 0u : ~((2u << hb) - 1u);
  uint32_t prefix = mx & mask;
  int remaining = k;
  const int n_round = (n + NT - 1) / NT * NT;
  while (hb >= 0) {
    const int lo = max(0, hb - 10);
    const int bins = 1 << (hb - lo + 1);
    for (int i = tid; i < bins; i += NT) sc->hist[i] = 0;
    G::sync();
    for (int i = tid; i < n_round; i += NT) {
      bool valid = false;
      uint32_t dg = 0xFFFFFFFFu;
      if (i < n) {
        const uint32_t u = key_at(i);
        if ((u & mask) == prefix) {
          valid = true;
          dg = (u >> lo) & (uint32_t)(bins - 1);
        }
      }
      const unsigned peers = __match_any_sync(0xffffffffu, dg);
      if (valid && lane == __ffs(peers) - 1) atomicAdd(&sc->hist[dg], __popc(peers));
    }
    if (tid == 0) {  // defaults, in case no digit qualifies (k larger than the keys left)
      sc->digit = 0;
      sc->above = 0;
    }
    G::sync();
    // thread t owns the digits bins-1-t*per .. bins-per-t*per (descending)
    const int per = (bins + NT - 1) / NT;
    int local = 0;
    for (int j = 0; j < per; ++j) {
      const int d = bins - 1 - (tid * per + j);
      if (d >= 0) local += sc->hist[d];
    }
    int tot;
    const int ex = group_exclusive_scan<G>(local, sc->warp_tot, &tot);
    if (ex < remaining && ex + local >= remaining) {
      int c = ex;
      for (int j = 0; j < per; ++j) {
        const int d = bins - 1 - (tid * per + j);
        if (d < 0) break;
        const int h = sc->hist[d];
        if (c + h >= remaining) {
          sc->digit = d;
          sc->above = c;
          break;
        }
        c += h;
      }
    }
    G::sync();
    const uint32_t d = (uint32_t)sc->digit;
    const int above = sc->above;
    const int in_bin = sc->hist[d];
    G::sync();
    remaining -= above;
    prefix |= d << lo;
    mask |= (uint32_t)(bins - 1) << lo;
    hb = lo - 1;
    if (in_bin == remaining) break;  // the whole bin is taken: no finer digit needed
  }
  return SelectResult{prefix, mask, remaining};
}

// Emit(i, out_index) is called for each kept element, out_index in [0, k).
template <class G, typename KeyAt, typename Emit>
__device__ void select_compact(KeyAt key_at, int n, SelectResult r, Emit emit, SelectScratch* sc) {
  constexpr int NT = G::N;
  const int tid = threadIdx.x;
  int base_gt = 0, base_eq = 0;
  for (int t0 = 0; t0 < n; t0 += NT) {
    const int i = t0 + tid;
    int gt = 0, eq = 0;
    if (i < n) {
      const uint32_t km = key_at(i) & r.mask;
      gt = km > r.thresh;
      eq = km == r.thresh;
    }
    int tot;
    const int ex = group_exclusive_scan<G>(gt | (eq << 16), sc->warp_tot, &tot);
    const int eq_before = base_eq + (ex >> 16);  // equal elements before i (in index order)
    if (gt || (eq && eq_before < r.need)) emit(i, base_gt + (ex & 0xFFFF) + min(eq_before, r.need));
    base_gt += tot & 0xFFFF;
    base_eq += tot >> 16;
  }
}

// ---------------------------------------------------------------------------
// Fast exact top-k (k <= n) for keys held in shared memory, in a few light
// passes: (1) min/max, to skip the high bits every key shares; (2) one
// histogram of the next <= 11 bits, which finds the bin D holding the k-th
// key; (3) the elements of bin D are gathered and ranked among themselves by
// (key desc, index asc), which gives the exact cut (key T, index I) of the
// k-th element; (4) an order-preserving compaction (warp ballots, one barrier
// round) emits every element above the cut in index order.  Falls back to
// radix_select/select_compact when bin D holds more than FT_BIN_CAP keys
// (heavily tied keys).  Emit(i, out_index), out_index in [0, k).
// ---------------------------------------------------------------------------
constexpr int FT_BIN_CAP = 1024;

struct FastTopScratch {
  SelectScratch sel;
  uint32_t bin_key[FT_BIN_CAP];
  int bin_idx[FT_BIN_CAP];
  int bin_cnt;
  uint32_t cut_key;
  int cut_idx;
  int warp_cnt[33];
};

template <class G, typename KeyAt, typename Emit>
__device__ void fast_topk(KeyAt key_at, int n, int k, Emit emit, FastTopScratch* fs) {
  constexpr int NT = G::N, NW = NT / 32;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  SelectScratch* sc = &fs->sel;
  // (1) min / max
  uint32_t mn = 0xFFFFFFFFu, mx = 0u;
  for (int i = tid; i < n; i += NT) {
    const uint32_t u = key_at(i);
    mn = min(mn, u);
    mx = max(mx, u);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    mn = min(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  if (lane == 0) {
    sc->kmin[warp] = mn;
    sc->kmax[warp] = mx;
  }
  if (tid == 0) fs->bin_cnt = 0;
  G::sync();
  mn = sc->kmin[0];
  mx = sc->kmax[0];
#pragma unroll
  for (int w = 1; w < NW; ++w) {
    mn = min(mn, sc->kmin[w]);
    mx = max(mx, sc->kmax[w]);
  }
  // cut: elements with (key > T) or (key == T and index <= I) are kept
  uint32_t T;
  int I;
  if (mn == mx) {  // all keys equal: the first k by index
    T = mx;
    I = k - 1;
  } else {
    // (2) histogram over linear bins of the score range.  bin() is monotone
    // (IEEE subtraction, multiplication and floor are), so a larger key never
    // lands in a lower bin; scores spread over the bins far better than the
    // raw bits of their encoding do.
    const float smin = key_score(mn), smax = key_score(mx);
    const float span = smax - smin;
    if (!(span > 1e-30f) || !(span < 3.0e38f)) {  // degenerate range: exact radix refinement
      const SelectResult r = radix_select<G>(key_at, n, k, sc);
      select_compact<G>(key_at, n, r, emit, sc);
      return;
    }
    const float scale = (float)SEL_BINS / span;
    auto bin_of = [&](uint32_t u) { return min(SEL_BINS - 1, (int)((key_score(u) - smin) * scale)); };
    constexpr int bins = SEL_BINS;
    for (int i = tid; i < bins; i += NT) sc->hist[i] = 0;
    G::sync();
    for (int i = tid; i < n; i += NT) atomicAdd(&sc->hist[bin_of(key_at(i))], 1);
    if (tid == 0) {  // defaults, in case no bin qualifies
      sc->digit = 0;
      sc->above = 0;
    }
    G::sync();
    constexpr int per = (bins + NT - 1) / NT;  // thread t owns bins bins-1-t*per .. (descending)
    int local = 0;
#pragma unroll
    for (int j = 0; j < per; ++j) {
      const int d = bins - 1 - (tid * per + j);
      if (d >= 0) local += sc->hist[d];
    }
    int tot;
    const int ex = group_exclusive_scan<G>(local, sc->warp_tot, &tot);
    if (ex < k && ex + local >= k) {
      int c = ex;
      for (int j = 0; j < per; ++j) {
        const int d = bins - 1 - (tid * per + j);
        if (d < 0) break;
        const int h = sc->hist[d];
        if (c + h >= k) {
          sc->digit = d;
          sc->above = c;
          break;
        }
        c += h;
      }
    }
    G::sync();
    const int D = sc->digit;
    const int need = k - sc->above;  // elements still to take from bin D (>= 1)
    const int inbin = sc->hist[D];
    G::sync();
    if (inbin > FT_BIN_CAP) {  // heavily tied keys: exact radix refinement
      const SelectResult r = radix_select<G>(key_at, n, k, sc);
      select_compact<G>(key_at, n, r, emit, sc);
      return;
    }
    // (3) gather bin D and rank its elements
    for (int i = tid; i < n; i += NT) {
      const uint32_t u = key_at(i);
      if (bin_of(u) == D) {
        const int slot = atomicAdd(&fs->bin_cnt, 1);
        fs->bin_key[slot] = u;
        fs->bin_idx[slot] = i;
      }
    }
    G::sync();
    const int cnt = fs->bin_cnt;
    for (int j = tid; j < cnt; j += NT) {
      const uint32_t kj = fs->bin_key[j];
      const int ij = fs->bin_idx[j];
      int rank = 0;
      for (int m = 0; m < cnt; ++m) {
        const uint32_t km = fs->bin_key[m];
        rank += (km > kj) || (km == kj && fs->bin_idx[m] < ij);
      }
      if (rank == need - 1) {
        fs->cut_key = kj;
        fs->cut_idx = ij;
      }
    }
    G::sync();
    T = fs->cut_key;
    I = fs->cut_idx;
    G::sync();
  }
  // (4) order-preserving compaction: warp w owns [w*chunk, (w+1)*chunk)
  const int chunk = ((n + NW - 1) / NW + 31) & ~31;
  const int w0 = min(n, warp * chunk), w1 = min(n, w0 + chunk);
  auto kept = [&](int i) {
    const uint32_t u = key_at(i);
    return u > T || (u == T && i <= I);
  };
  int count = 0;
  for (int base = w0; base < w1; base += 32) {
    const int i = base + lane;
    count += __popc(__ballot_sync(0xffffffffu, i < w1 && kept(i)));
  }
  if (lane == 0) fs->warp_cnt[warp] = count;
  G::sync();
  int out = 0;
  for (int w = 0; w < warp; ++w) out += fs->warp_cnt[w];
  for (int base = w0; base < w1; base += 32) {
    const int i = base + lane;
    const bool kp = i < w1 && kept(i);
    const unsigned m = __ballot_sync(0xffffffffu, kp);
    if (kp) emit(i, out + __popc(m & ((1u << lane) - 1u)));
    out += __popc(m);
  }
  G::sync();
}

// ---------------------------------------------------------------------------
// Exact top-k of n <= HT_MAX_N keys in shared memory whose histogram was
// built while the keys were produced (ht_count, by the producing warps):
// bins are the top HT_BITS bits of the order-preserving key, i.e. a
// log-scale histogram of the scores (1/16 octave).  The selection then takes
// four light steps and a single pass over the keys:
//   (1) a scan of the histogram finds the bin D holding the k-th key;
//   (2) one pass writes, per 32 consecutive keys, the ballot of the keys in
//       bins above D as one word of a keep bitmap, and puts the keys of bin D
//       into the warp's own tie list (no atomics);
//   (3) the ties are ranked by (key desc, index asc); the first `need` set
//       their bits;
//   (4) a popcount prefix over the bitmap words emits the kept indices in
//       ascending order.
// Every loop loads several independent values before using any of them:
// with a few warps per SM the selection is bound by latency, not work.
// Bins hold 16-bit counts, two per word (n <= 8192 never overflows one).
// If one warp finds more ties than its list holds, the ties are gathered
// again with a shared counter; more than HT_TIE_CAP ties in all (heavily
// tied keys) fall back to radix_select / select_compact, which borrow the
// histogram's storage.  Emit(i, o): kept index i, output slot o in [0, k),
// called after the last read of `keys`; requires k <= n.
// ---------------------------------------------------------------------------
constexpr int HT_BITS = 13;
constexpr int HT_BINS = 1 << HT_BITS;  // 8192 bins
constexpr int HT_WORDS = HT_BINS / 2;  // 4096 words of two 16-bit counts
constexpr int HT_MAX_N = 16384;
constexpr int HT_TIE_CAP = 512;

struct HistTopScratch {
  int warp_tot[33];
  int D, above, tie_n;  // tie_n: shared tie counter of the regather path and of row selections
  int tie_cnt[32];  // ties found by each warp
  uint32_t bits[HT_MAX_N / 32];
  // ties of the cut bin as one comparable word: key in the high half, bitwise-inverted index in the
  // low half, so a larger value ranks first under (key desc, index asc).  The warps' lists fill
  // the first half; the second half holds them packed for ranking.
  unsigned long long tie[2 * HT_TIE_CAP];
};

__device__ __forceinline__ int ht_bin(uint32_t key) { return (int)(key >> (32 - HT_BITS)); }

// Counts one key (any thread, any order).
__device__ __forceinline__ void ht_count(uint32_t* hist, uint32_t key) {
  const int b = ht_bin(key);
  atomicAdd(hist + (b >> 1), 1u << ((b & 1) * 16));
}

template <class G>
__device__ __forceinline__ void ht_zero(uint32_t* hist) {
  for (int i = threadIdx.x; i < HT_WORDS / 4; i += G::N) reinterpret_cast<uint4*>(hist)[i] = make_uint4(0, 0, 0, 0);
}

__device__ __forceinline__ unsigned long long ht_tie_word(uint32_t key, int i) {
  return ((unsigned long long)key << 32) | (uint32_t)~i;
}

template <class G, typename Emit>
__device__ void hist_topk(const uint32_t* keys, uint32_t* hist, int n, int k, Emit emit, HistTopScratch* sc) {
  constexpr int NT = G::N, NW = NT / 32;
  constexpr int PER = HT_BINS / NT;  // bins per thread
  constexpr int WCAP = HT_TIE_CAP / NW;
  static_assert(PER % 8 == 0, "layout");  // callers keep n <= 32 * NT (one bitmap word per thread)
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // (1) thread t owns bins top-PER*t-PER+1 .. top-PER*t (descending order of ownership)
  const int lo_bin = HT_BINS - PER * (tid + 1);
  uint32_t cw[PER / 2];
#pragma unroll
  for (int q = 0; q < PER / 8; ++q) {
    const uint4 v = reinterpret_cast<const uint4*>(hist + lo_bin / 2)[q];
    cw[4 * q] = v.x;
    cw[4 * q + 1] = v.y;
    cw[4 * q + 2] = v.z;
    cw[4 * q + 3] = v.w;
  }
  int local = 0;
#pragma unroll
  for (int q = 0; q < PER / 2; ++q) local += (int)(cw[q] & 0xFFFFu) + (int)(cw[q] >> 16);
  if (tid == 0) {
    sc->D = -1;
    sc->above = 0;
    sc->tie_n = 0;
  }
  for (int i = tid; i < HT_MAX_N / 32; i += NT) sc->bits[i] = 0u;
  int tot;
  const int ex = group_exclusive_scan_1b<G>(local, sc->warp_tot, &tot);  // keys in bins above this thread's
  if (ex < k && ex + local >= k) {
    int c = ex;
#pragma unroll
    for (int q = PER - 1; q >= 0; --q) {
      const int h = (int)((cw[q >> 1] >> ((q & 1) * 16)) & 0xFFFFu);
      if (c + h >= k) {
        sc->D = lo_bin + q;
        sc->above = c;
        break;
      }
      c += h;
    }
  }
  G::sync();
  const int D = sc->D;
  const int need = k - sc->above;
  // (2) one pass: keep-bitmap words for bins above D, ties of bin D into the warp's own list.
  // Warp w takes words w, w + NW, ...; four words' keys are loaded before any of them is used.
  unsigned long long* wtie = sc->tie + warp * WCAP;
  unsigned long long* packed = sc->tie + HT_TIE_CAP;
  int nt = 0;  // warp-uniform
  const int nwords = (n + 31) >> 5;
  for (int wd0 = warp; wd0 < nwords; wd0 += 4 * NW) {
    uint32_t key[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = (wd0 + u * NW) * 32 + lane;
      key[u] = i < n ? keys[i] : 0u;
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int wd = wd0 + u * NW;
      const int i = wd * 32 + lane;
      const int b = ht_bin(key[u]);
      const unsigned def = __ballot_sync(0xffffffffu, i < n && b > D);
      const unsigned tie = __ballot_sync(0xffffffffu, i < n && b == D);
      if (lane == 0 && wd < nwords) sc->bits[wd] = def;
      if (tie & (1u << lane)) {
        const int pos = nt + __popc(tie & ((1u << lane) - 1u));
        if (pos < WCAP) wtie[pos] = ht_tie_word(key[u], i);
      }
      nt += __popc(tie);
    }
  }
  if (lane == 0) sc->tie_cnt[warp] = nt;
  G::sync();
  int m = 0, over = 0, before = 0;
#pragma unroll
  for (int w = 0; w < NW; ++w) {
    const int c = sc->tie_cnt[w];
    before += w < warp ? c : 0;
    m += c;
    over |= c > WCAP;
  }
  if (m > HT_TIE_CAP) {  // heavily tied keys: exact radix refinement (the histogram is free now)
    SelectScratch* ss = reinterpret_cast<SelectScratch*>(hist);
    auto key_at = [&](int i) { return keys[i]; };
    const SelectResult r = radix_select<G>(key_at, n, k, ss);
    select_compact<G>(key_at, n, r, emit, ss);
    return;
  }
  if (over) {  // one warp's list overflowed: gather the ties again with a shared counter
    for (int i = tid; i < n; i += NT) {
      const uint32_t key = keys[i];
      if (ht_bin(key) == D) packed[atomicAdd(&sc->tie_n, 1)] = ht_tie_word(key, i);
    }
  } else {
    for (int c = lane; c < nt; c += 32) packed[before + c] = wtie[c];
  }
  G::sync();
  // (3) exact order inside bin D: a tie is kept when fewer than `need` ties rank above it
  for (int a = tid; a < m; a += NT) {
    const unsigned long long va = packed[a];
    int rank = 0;
    int c = 0;
    for (; c + 8 <= m; c += 8) {
      unsigned long long vc[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) vc[u] = packed[c + u];
#pragma unroll
      for (int u = 0; u < 8; ++u) rank += vc[u] > va;
    }
    for (; c < m; ++c) rank += packed[c] > va;
    if (rank < need) {
      const int ia = (int)~(uint32_t)va;
      atomicOr(&sc->bits[ia >> 5], 1u << (ia & 31));
    }
  }
  G::sync();
  // (4) ordered emission
  uint32_t wbits = tid < nwords ? sc->bits[tid] : 0u;
  int o = group_exclusive_scan_1b<G>(__popc(wbits), sc->warp_tot, &tot);
  while (wbits) {
    const int bit = __ffs(wbits) - 1;
    emit(tid * 32 + bit, o++);
    wbits &= wbits - 1u;
  }
  G::sync();
}

// ---------------------------------------------------------------------------
// Scoring one page of 16 compressed keys on the tensor cores (mma.sync), used
// by the streaming scorer and by the prefill path's exact re-scoring of a row.
// ---------------------------------------------------------------------------
#ifndef QSA_SC_L2_PROMOTE
#define QSA_SC_L2_PROMOTE 0
#endif
__device__ __forceinline__ uint4 ldg_stream(const uint4* p) {
  uint4 v;
#if QSA_SC_L2_PROMOTE == 256
  asm volatile("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
#elif QSA_SC_L2_PROMOTE == 128
  asm volatile("ld.global.nc.L1::no_allocate.L2::128B.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
#else
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
#endif
  return v;
}

// One page of 16 keys: lane (g, c) holds 16-byte chunks c, c+4, c+8, c+12 of
// keys g and g+8.  Chunk u of key g, read as four bf16 pairs x, y, z, w,
// supplies the A fragment of k-steps 2u (pairs x, y) and 2u+1 (pairs z, w):
// logical k {2c, 2c+1} -> first pair, {2c+8, 2c+9} -> second pair.
struct PageRegs {
  uint4 lo[4], hi[4];  // keys g and g + 8
};

__device__ __forceinline__ void load_page(PageRegs& r, const uint4* page, int g, int c) {
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    r.lo[u] = ldg_stream(page + g * 16 + c + 4 * u);
    r.hi[u] = ldg_stream(page + (g + 8) * 16 + c + 4 * u);
  }
}

// The same with coherent loads, for the one page this kernel has just written a compressed key to.
__device__ __forceinline__ void load_page_fresh(PageRegs& r, const uint4* page, int g, int c) {
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    r.lo[u] = __ldcg(page + g * 16 + c + 4 * u);
    r.hi[u] = __ldcg(page + (g + 8) * 16 + c + 4 * u);
  }
}

__device__ __forceinline__ void score_page(const PageRegs& r, const uint32_t (&bq)[8][2], float wa, float wb,
                                           float& lo_score, float& hi_score) {
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int u = j >> 1;
    uint32_t a[4];
    a[0] = (j & 1) ? r.lo[u].z : r.lo[u].x;
    a[1] = (j & 1) ? r.hi[u].z : r.hi[u].x;
    a[2] = (j & 1) ? r.lo[u].w : r.lo[u].y;
    a[3] = (j & 1) ? r.hi[u].w : r.hi[u].y;
    mma_bf16_16816(acc, a, bq[j][0], bq[j][1]);
  }
  // acc: rows g / g+8 (keys), columns 2c, 2c+1 (heads); sum the heads over the quad
  float lo = wa * fmaxf(acc[0], 0.f) + wb * fmaxf(acc[1], 0.f);
  float hi = wa * fmaxf(acc[2], 0.f) + wb * fmaxf(acc[3], 0.f);
  lo += __shfl_xor_sync(0xffffffffu, lo, 1);
  hi += __shfl_xor_sync(0xffffffffu, hi, 1);
  lo += __shfl_xor_sync(0xffffffffu, lo, 2);
  hi += __shfl_xor_sync(0xffffffffu, hi, 2);
  lo_score = lo;
  hi_score = hi;
}

__host__ __device__ __forceinline__ int ceil_div(int a, int b) { return (a + b - 1) / b; }

}  // namespace qsa
