// Index projection of the QSA c4 indexer: from a token's hidden state to its
// 4 index query heads (128 dims each), its one shared index key (128 dims) and
// its 4 index head weights.
//
// Blog section "Qwen Sparse Attention: Retrieve Coarsely, Attend Precisely"
// (SGLang day-0 blog for Qwen3.8-Flash-Next): the indexer projects 4 query
// heads of 128 dims and one shared 128-dim key per token, and can run on a
// second CUDA stream, overlapping the layer's main Q/K/V projection.  The
// pages give neither the hidden size nor how the head weights are formed; the
// reading used here: one bias-free linear map of the hidden state,
//   [idx_q (4 x 128) | idx_k (128) | w (4)] = W x,  W: [644][hidden] bf16,
// accumulated in FP32, idx_q / idx_k rounded once to bf16, w kept in FP32.
//
// Design (B200).  A decode step projects one row per request (a few dozen
// rows): the product is skinny and bound by reading W once from HBM (644 x
// hidden x 2 bytes, 5.3 MB at hidden 4096).  Each warp computes a tile of 16
// rows x 8 features over one slice of the hidden dimension with m16n8k16 bf16
// MMAs; A (rows) and B (features) are both read with 16-byte loads and fed to
// the MMA in the same permuted order of the hidden dimension, so no shuffle
// or shared-memory staging is needed.  The warps of a CTA split the hidden
// dimension (32 warps: one 128-dim slice each at hidden 4096, so the whole
// product is one round of loads) and add their tiles in shared memory in a
// fixed order (the result does not depend on timing).
#include "qsa_common.cuh"
#include "qsa_kernels.h"

namespace qsa {

constexpr int PJ_WARPS = 32;       // hidden-dimension slices per CTA: at hidden 4096 one 128-dim load round
                                   // per warp, so every load of the CTA is in flight at once
constexpr int PJ_ROWS = 16;        // rows of a tile (MMA M)
constexpr int PJ_FEAT = 8;         // features of a tile (MMA N)
constexpr int PJ_KCHUNK = 128;     // hidden dims per load round of a warp (8 MMA k-steps)

// 16 bf16 (two 16-byte chunks c and c + 4 ... : lane (g, c) reads chunks c, c+4, c+8, c+12 of a
// 128-dim piece of its row; chunk u read as pairs x, y, z, w feeds k-steps 2u (x, y) and 2u+1 (z, w)).
__device__ __forceinline__ void pj_load(uint4 (&r)[4], const __nv_bfloat16* row, int c) {
  const uint4* p = reinterpret_cast<const uint4*>(row);
#pragma unroll
  for (int u = 0; u < 4; ++u) r[u] = __ldg(p + c + 4 * u);
}

__global__ void __launch_bounds__(PJ_WARPS * 32) k_index_proj(ProjParams p) {
  __shared__ float part[PJ_WARPS][PJ_ROWS * PJ_FEAT];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;
  const int f0 = blockIdx.x * PJ_FEAT, r0 = blockIdx.y * PJ_ROWS;
  // rows g and g + 8 of the tile (A), feature g (B); rows / features past the end read row 0 / feature 0
  // (their results are never written)
  const int ra = min(r0 + g, p.n - 1), rb = min(r0 + g + 8, p.n - 1);
  const int fb = min(f0 + g, QSA_PROJ_FEATURES - 1);
  const __nv_bfloat16* xa = p.x + (int64_t)ra * p.hidden;
  const __nv_bfloat16* xb = p.x + (int64_t)rb * p.hidden;
  const __nv_bfloat16* wf = p.w + (int64_t)fb * p.hidden;
  const int nchunk = p.hidden / PJ_KCHUNK;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  for (int k = warp; k < nchunk; k += PJ_WARPS) {
    uint4 a_lo[4], a_hi[4], b[4];
    pj_load(a_lo, xa + k * PJ_KCHUNK, c);
    pj_load(a_hi, xb + k * PJ_KCHUNK, c);
    pj_load(b, wf + k * PJ_KCHUNK, c);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int u = j >> 1;
      uint32_t a[4];
      a[0] = (j & 1) ? a_lo[u].z : a_lo[u].x;
      a[1] = (j & 1) ? a_hi[u].z : a_hi[u].x;
      a[2] = (j & 1) ? a_lo[u].w : a_lo[u].y;
      a[3] = (j & 1) ? a_hi[u].w : a_hi[u].y;
      const uint32_t b0 = (j & 1) ? b[u].z : b[u].x;
      const uint32_t b1 = (j & 1) ? b[u].w : b[u].y;
      mma_bf16_16816(acc, a, b0, b1);
    }
  }
  // acc: rows g, g + 8; features 2c, 2c + 1
  float* mine = part[warp];
  mine[g * PJ_FEAT + 2 * c] = acc[0];
  mine[g * PJ_FEAT + 2 * c + 1] = acc[1];
  mine[(g + 8) * PJ_FEAT + 2 * c] = acc[2];
  mine[(g + 8) * PJ_FEAT + 2 * c + 1] = acc[3];
  __syncthreads();
  if (threadIdx.x < PJ_ROWS * PJ_FEAT) {
    const int i = threadIdx.x, row = r0 + i / PJ_FEAT, f = f0 + i % PJ_FEAT;
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < PJ_WARPS; ++w) s += part[w][i];  // fixed order
    if (row < p.n && f < QSA_PROJ_FEATURES) {
      if (f < HI * D) {
        p.idx_q[(int64_t)row * HI * D + f] = __float2bfloat16_rn(s);
      } else if (f < HI * D + D) {
        p.idx_k[(int64_t)row * D + (f - HI * D)] = __float2bfloat16_rn(s);
      } else {
        p.wout[(int64_t)row * HI + (f - HI * D - D)] = s;
      }
    }
  }
}

cudaError_t launch_index_proj(const ProjParams& p, cudaStream_t st) {
  dim3 grid(ceil_div(QSA_PROJ_FEATURES, PJ_FEAT), ceil_div(p.n, PJ_ROWS));
  k_index_proj<<<grid, PJ_WARPS * 32, 0, st>>>(p);
  return cudaGetLastError();
}

}  // namespace qsa
