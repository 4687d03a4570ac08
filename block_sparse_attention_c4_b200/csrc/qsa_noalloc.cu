// qsa_sparse_gqa_noalloc: the sparse GQA entry point for callers that cannot
// allocate device memory or hand the library a workspace.
//
// Who needs it: a plugin loaded into a host program whose interface passes it
// only input and output buffers; code that runs while a CUDA graph is being
// captured, where a cudaMalloc would break the capture; a deployment whose
// device-memory budget is fixed at start-up.  This entry point asks for no
// workspace and calls no allocator: its split-K scratch (partial outputs,
// running maxima and sums, arrival counters) is the file-scope device array
// below, which every GPU that loads this library keeps until the process
// exits.
//
// The computation is exactly qsa_sparse_gqa's (same kernel); only where the
// scratch lives differs, and the number of splits is capped so the partials
// fit in the array.
#include <mutex>

#include "qsa_common.cuh"
#include "qsa_kernels.h"

using namespace qsa;

namespace {

// Capacity of the array: QSA_NOALLOC_ROW_SPLITS (query, split) partials of
// 16 heads x 128 dims in FP32, their (max, sum) pairs, and one arrival
// counter per query.
constexpr int ROW_SPLITS = QSA_NOALLOC_ROW_SPLITS;
constexpr size_t OFF_COUNTERS = 256;
constexpr size_t OFF_ML = OFF_COUNTERS + sizeof(int) * QSA_NOALLOC_MAX_QUERIES;
constexpr size_t OFF_O = OFF_ML + sizeof(float) * ROW_SPLITS * HQ * 2;
constexpr size_t SCRATCH_BYTES = OFF_O + sizeof(float) * (size_t)ROW_SPLITS * HQ * D;
static_assert(SCRATCH_BYTES == QSA_NOALLOC_SCRATCH_BYTES, "qsa.h states the scratch size");
static_assert(OFF_ML % 256 == 0 && OFF_O % 256 == 0, "256-byte aligned sections");

static __device__ __align__(256) uint8_t g_noalloc_scratch[SCRATCH_BYTES];

constexpr int MAX_DEVICES = 64;
std::mutex g_mu;
uint8_t* g_addr[MAX_DEVICES] = {nullptr};

// Device address of the array on the current device, looked up once per
// device (the host-side symbol is only a stand-in, never a device address).
cudaError_t scratch_address(uint8_t** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= MAX_DEVICES) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_addr[dev] = static_cast<uint8_t*>(p);
  }
  *out = g_addr[dev];
  return cudaSuccess;
}

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
  return n;
}

}  // namespace

extern "C" qsa_status qsa_sparse_gqa_noalloc(const qsa_cache* cache, const void* q, const int32_t* q_req,
                                             const int32_t* pos, const int32_t* npos, int32_t pos_stride,
                                             int32_t max_pos, int32_t nq, float scale, void* out, float* lse,
                                             void* stream) {
  // the same checks as qsa_sparse_gqa (the compressed index cache and ring are not read here)
  const qsa_status cs = check_kv_cache(cache);
  if (cs != QSA_OK) return cs;
  if (nq < 0 || pos_stride < 0 || max_pos < 0 || max_pos > pos_stride || !valid_scale(scale)) return QSA_ERR_INVALID_ARG;
  if (nq > QSA_NOALLOC_MAX_QUERIES) return QSA_ERR_UNSUPPORTED;  // beyond the array's stated capacity
  if (max_pos > QSA_MAX_SEL) return QSA_ERR_UNSUPPORTED;
  if (nq == 0) return QSA_OK;
  if (!q || !q_req || !pos || !npos || !out) return QSA_ERR_INVALID_ARG;
  if (!host_aligned(q, 16) || !host_aligned(out, 16) || (lse && !host_aligned(lse, 4))) return QSA_ERR_INVALID_ARG;

  uint8_t* base = nullptr;
  if (scratch_address(&base) != cudaSuccess) return QSA_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // the arrival counters must start at zero whatever an earlier call left
  if (cudaMemsetAsync(base + OFF_COUNTERS, 0, sizeof(int) * (size_t)nq, st) != cudaSuccess) return QSA_ERR_CUDA;

  GqaParams p{};
  p.c.k = static_cast<const __nv_bfloat16*>(cache->k);
  p.c.v = static_cast<const __nv_bfloat16*>(cache->v);
  p.c.page_table = cache->page_table;
  p.c.num_pages = cache->num_slots / QSA_PAGE_SIZE;
  p.c.kv_stride = cache->kv_stride ? cache->kv_stride : HKV * D;
  p.c.max_pages = cache->max_pages;
  p.c.batch = cache->batch;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.nq_row = 1;
  p.row_req = q_req;
  p.mode = 1;
  p.list = pos;
  p.list_n = npos;
  p.list_stride = pos_stride;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  p.part_o = reinterpret_cast<float*>(base + OFF_O);
  p.part_ml = reinterpret_cast<float*>(base + OFF_ML);
  p.counters = reinterpret_cast<int*>(base + OFF_COUNTERS);
  const int cap = ROW_SPLITS / nq > 0 ? ROW_SPLITS / nq : 1;  // partials that fit the array
  p.err = nullptr;  // no error word: positions outside the request's page-table row or the page pool are
                    // skipped silently
  return launch_gqa(p, nq, max_pos, sm_count(), cap, st) == cudaSuccess ? QSA_OK : QSA_ERR_CUDA;
}
