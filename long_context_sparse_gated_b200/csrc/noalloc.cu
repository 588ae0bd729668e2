// csa_index_topk_noalloc: the Lightning Indexer + top-k call for callers
// that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc (or any allocator) at the point where
// they run the indexer: code inside an allocator-free inference loop whose
// memory is fixed up front, plugins that are handed only their inputs and
// outputs by a host framework, or hosts whose allocator is off limits while
// they run.  csa_index_topk needs a caller-provided workspace for its scores
// and per-query histograms; this variant takes that workspace from a
// file-scope static device array instead, so the caller passes only inputs
// and outputs.
//
// The array holds kScratchBytes (16 MiB) on every GPU that loads the
// library, from module load until the process exits.  Problems whose
// workspace (csa_index_topk_workspace_bytes) exceeds it are rejected with
// CSA_ERR_WORKSPACE before anything is launched.  All calls share the one
// array: two calls whose work overlaps on the GPU (different streams, or
// different host threads on the same device) race on it; the array keeps the
// previous call's contents, and the parts that must start at zero (the
// histograms) are cleared on every call by the regular path.
#include <cuda_runtime.h>

#include <mutex>

#include "csa.h"

namespace {

constexpr size_t kScratchBytes = 16u << 20;  // 16 MiB
constexpr int kMaxDevices = 64;

// The scratch itself.  In host code this name is only a host-side stand-in
// for the symbol; its device address comes from cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_index_scratch[kScratchBytes];

// Device address of g_index_scratch per device ordinal, looked up once per
// device with that device current.
void* g_scratch_addr[kMaxDevices] = {};
std::mutex g_scratch_mu;

csa_status scratch_for_current_device(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return CSA_ERR_LAUNCH;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_index_scratch) != cudaSuccess || !p) return CSA_ERR_LAUNCH;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return CSA_OK;
}

}  // namespace

extern "C" csa_status csa_index_topk_noalloc(const csa_params* params, const void* q_idx,
                                             const uint8_t* q_idx_sf, const float* w,
                                             const void* k_idx, const uint8_t* k_idx_sf,
                                             int64_t k_cap, const int32_t* q_pos0, int32_t T,
                                             int32_t n_max, int32_t* out_idx, int32_t* err,
                                             void* stream) {
  if (!params || T < 1 || n_max < 0) return CSA_ERR_INVALID;
  if (csa_index_topk_workspace_bytes(params, T, n_max) > kScratchBytes) return CSA_ERR_WORKSPACE;
  void* scratch = nullptr;
  const csa_status s = scratch_for_current_device(&scratch);
  if (s != CSA_OK) return s;
  return csa_index_topk(params, q_idx, q_idx_sf, w, k_idx, k_idx_sf, k_cap, q_pos0, T, n_max, out_idx,
                        scratch, kScratchBytes, err, stream);
}
