// lmoe_permute_noalloc: the expert-grouped permutation without a caller
// workspace. Its scratch (the per-chunk expert count table of the counting
// sort) lives in a fixed array in device memory that the library defines, so
// the call needs no allocation at all -- for callers that are handed their
// input and output buffers but may not allocate device memory themselves.
#include <mutex>

#include "lmoe_internal.h"

namespace lmoe {
namespace {

// Scratch of the counting sort: (chunks + 1) * N int32 counters, chunks =
// ceil(T*K / 8192). 128 Ki entries = 512 KiB, held by every GPU that loads
// the library until the process exits.
constexpr int64_t kStaticScratchEntries = 128 * 1024;
static __device__ __align__(256) int32_t g_permute_scratch[kStaticScratchEntries];

// Device address of the array. Host code cannot use the symbol itself as a
// device pointer, so the address is looked up with cudaGetSymbolAddress, with
// the device current, at the first call on that device. The cached address
// belongs to the context it was looked up in: it is keyed on that context's
// process-unique id (cuCtxGetId), so after cudaDeviceReset, or any teardown
// and re-creation of the device's context, the next call looks it up again
// instead of handing the kernel an address the library no longer owns.
constexpr int kMaxDevices = 64;
struct ScratchEntry {
  unsigned long long ctx_id;
  int32_t* ptr;
};
ScratchEntry g_scratch[kMaxDevices] = {};
std::mutex g_scratch_mutex;

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

// Id of the calling thread's current context (0 when none is current or the
// driver entry points are missing).
unsigned long long current_context_id() {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
  if (get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

lmoe_status static_scratch(int32_t** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return LMOE_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  ScratchEntry& e = g_scratch[dev];
  unsigned long long ctx = current_context_id();
  if (e.ptr == nullptr || ctx == 0 || e.ctx_id != ctx) {
    // the lookup also makes the device's primary context current if no
    // context was yet, so the id is read again after it
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_permute_scratch) != cudaSuccess || p == nullptr) return LMOE_ERR_CUDA;
    e.ptr = static_cast<int32_t*>(p);
    e.ctx_id = ctx ? ctx : current_context_id();   // 0 (no id available) never matches: look up every call
  }
  *out = e.ptr;
  return LMOE_OK;
}

}  // namespace
}  // namespace lmoe

extern "C" lmoe_status lmoe_permute_noalloc(const lmoe_config* cfg, const int32_t* topk_idx, int32_t* offsets,
                                            int32_t* perm_src, int32_t* inv_perm, int32_t* padded_offsets,
                                            const void* rows, int64_t row_bytes, void* permuted_rows,
                                            const uint8_t* rows_sf, uint8_t* permuted_sf, const float* topk_w,
                                            float* perm_gate, void* stream) {
  using namespace lmoe;
  if (!cfg || !topk_idx || !offsets || !perm_src || !inv_perm || !padded_offsets) return LMOE_ERR_INVALID_ARG;
  if (cfg->T < 0 || cfg->T > (int64_t(1) << 31) / 64) return LMOE_ERR_INVALID_ARG;   // as every entry point
  if (cfg->N <= 0 || cfg->K <= 0 || cfg->K > cfg->N) return LMOE_ERR_INVALID_ARG;
  if (cfg->N > 1024 || cfg->K > 32) return LMOE_ERR_UNSUPPORTED;
  if ((rows == nullptr) != (permuted_rows == nullptr)) return LMOE_ERR_INVALID_ARG;
  if (rows && (row_bytes <= 0 || row_bytes % 16 || (reinterpret_cast<uintptr_t>(rows) & 15) ||
               (reinterpret_cast<uintptr_t>(permuted_rows) & 15)))
    return LMOE_ERR_INVALID_ARG;
  if ((rows_sf == nullptr) != (permuted_sf == nullptr)) return LMOE_ERR_INVALID_ARG;
  if (rows_sf && (!rows || (row_bytes * 2) % 64)) return LMOE_ERR_INVALID_ARG;
  if ((topk_w == nullptr) != (perm_gate == nullptr)) return LMOE_ERR_INVALID_ARG;
  const int64_t slots = cfg->T * cfg->K;
  const int64_t need = static_cast<int64_t>(permute_chunks(slots, kPermSlotsPerWarpStatic) + 1) * cfg->N;
  if (need > kStaticScratchEntries) return LMOE_ERR_WORKSPACE;   // beyond the fixed scratch
  int32_t* scratch = nullptr;
  lmoe_status st = static_scratch(&scratch);
  if (st != LMOE_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // No error word: an out-of-range expert index is skipped without a report.
  st = launch_permute(topk_idx, cfg->T, cfg->K, cfg->N, offsets, perm_src, inv_perm, padded_offsets, scratch,
                      topk_w, perm_gate, nullptr, s, kPermSlotsPerWarpStatic);
  if (st != LMOE_OK) return st;
  if (rows || rows_sf) {
    st = launch_gather(topk_idx, perm_src, offsets, padded_offsets, slots, cfg->K, rows, row_bytes, permuted_rows,
                       rows_sf, permuted_sf, cfg->N, s);
  }
  return st;
}
