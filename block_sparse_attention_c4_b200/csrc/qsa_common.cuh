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
// Shared-memory / async-copy PTX wrappers
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
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

// Bounded wait: gives up after ~2 s of wall time, records QSA_DEVERR_TIMEOUT
// and returns false (the caller then proceeds without the data).
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, int* err) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (global_timer_ns() - t0 > 2000000000ull) break;
  }
  set_error(err, QSA_DEVERR_TIMEOUT);
  return false;
}

// 2-D tiled TMA load (no multicast) into shared memory, completing on `bar`.
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
__device__ __forceinline__ void cp_async_16(void* dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(src_bytes)
               : "memory");
}

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }

template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// ---------------------------------------------------------------------------
// Block-wide exclusive scan (any blockDim that is a multiple of 32, <= 1024).
// `warp_tot` needs 33 ints of shared memory.  Returns the exclusive prefix of
// `v` and writes the block total to *total.
// ---------------------------------------------------------------------------
__device__ __forceinline__ int block_exclusive_scan(int v, int* warp_tot, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_tot[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int t = lane < nwarps ? warp_tot[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += y;
    }
    if (lane < nwarps) warp_tot[lane] = t;  // inclusive warp prefix
    if (lane == 31) warp_tot[32] = t;
  }
  __syncthreads();
  const int before = warp > 0 ? warp_tot[warp - 1] : 0;
  const int res = before + x - v;
  *total = warp_tot[32];
  __syncthreads();
  return res;
}

// ---------------------------------------------------------------------------
// CTA-wide exact top-k selection on 32-bit keys (larger key first, then lower
// index first).  Step 1, radix_select: 8-bit digits from the top find the
// masked prefix T such that count(key&mask > T) < k <= count(key&mask >= T);
// `need` is how many elements with key&mask == T are still to be taken.
// Step 2, select_compact: keeps every key&mask > T and the first `need`
// elements with key&mask == T in index order, emitting them in index order.
// KeyAt: int -> uint32 accessor; n may exceed blockDim.
// ---------------------------------------------------------------------------
struct SelectScratch {
  int hist[256];
  int warp_tot[33];
  int digit;
  int above;
};

struct SelectResult {
  uint32_t thresh;
  uint32_t mask;
  int need;
};

template <typename KeyAt>
__device__ SelectResult radix_select(KeyAt key_at, int n, int k, SelectScratch* sc) {
  const int tid = threadIdx.x, nt = blockDim.x, lane = tid & 31;
  uint32_t prefix = 0, mask = 0;
  int remaining = k;
  const int n_round = (n + nt - 1) / nt * nt;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = tid; i < 256; i += nt) sc->hist[i] = 0;
    __syncthreads();
    for (int i = tid; i < n_round; i += nt) {
      bool valid = false;
      uint32_t dg = 0xFFFFFFFFu;
      if (i < n) {
        const uint32_t u = key_at(i);
        if ((u & mask) == prefix) {
          valid = true;
          dg = (u >> shift) & 255u;
        }
      }
      const unsigned peers = __match_any_sync(0xffffffffu, dg);
      if (valid && lane == __ffs(peers) - 1) atomicAdd(&sc->hist[dg], __popc(peers));
    }
    __syncthreads();
    // suffix sums over digits: thread t < 256 handles digit 255 - t
    int cnt = 0, incl = 0;
    if (tid < 256) cnt = sc->hist[255 - tid];
    {
      int tot;
      // scan only the first 256 threads' values; others contribute zero
      const int ex = block_exclusive_scan(tid < 256 ? cnt : 0, sc->warp_tot, &tot);
      incl = ex + cnt;
      // digit d = 255 - tid: count of digits > d is ex; count >= d is incl
      if (tid < 256 && ex < remaining && incl >= remaining) {
        sc->digit = 255 - tid;
        sc->above = ex;
      }
    }
    __syncthreads();
    const uint32_t d = (uint32_t)sc->digit;
    const int above = sc->above;
    const int in_bin = sc->hist[d];
    __syncthreads();
    remaining -= above;
    prefix |= d << shift;
    mask |= 255u << shift;
    if (in_bin == remaining) break;  // the whole bin is taken: no finer digit needed
  }
  return SelectResult{prefix, mask, remaining};
}

// Emit(i, out_index) is called for each kept element, out_index in [0, k).
template <typename KeyAt, typename Emit>
__device__ void select_compact(KeyAt key_at, int n, SelectResult r, Emit emit, SelectScratch* sc) {
  const int tid = threadIdx.x, nt = blockDim.x;
  int base_gt = 0, base_eq = 0;
  for (int t0 = 0; t0 < n; t0 += nt) {
    const int i = t0 + tid;
    int gt = 0, eq = 0;
    if (i < n) {
      const uint32_t km = key_at(i) & r.mask;
      gt = km > r.thresh;
      eq = km == r.thresh;
    }
    int tot;
    const int ex = block_exclusive_scan(gt | (eq << 16), sc->warp_tot, &tot);
    const int ex_gt = ex & 0xFFFF, ex_eq = ex >> 16;
    const int eq_before = base_eq + ex_eq;  // equal elements before i
    const int taken_eq_before = min(eq_before, r.need) - min(base_eq, r.need);
    if (gt || (eq && eq_before < r.need)) emit(i, base_gt + min(base_eq, r.need) + ex_gt + taken_eq_before);
    base_gt += tot & 0xFFFF;
    base_eq += tot >> 16;
  }
}

__host__ __device__ __forceinline__ int ceil_div(int a, int b) { return (a + b - 1) / b; }

}  // namespace qsa
