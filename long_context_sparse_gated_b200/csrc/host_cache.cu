// Host-side work that does not change between calls, done once.
//
// A call of the library launches one to four kernels; what it would
// otherwise repeat on every call is driver bookkeeping: the SM count of the
// device, raising a kernel's dynamic shared-memory limit
// (cudaFuncSetAttribute) and encoding TMA tensor maps
// (cuTensorMapEncodeTiled).  The first two are cached per device and
// context (a destroyed and re-created context starts afresh); tensor maps
// are cached per host thread, keyed by every argument of the encode, so a
// call with the same buffers and shapes as a recent one reuses the encoded
// 128-byte descriptor.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstring>
#include <mutex>

#include "kernels.h"

namespace csa {

namespace {

constexpr int kMaxDevices = 64;

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);
using EncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                              const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                              CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

template <class Fn>
Fn driver_entry(const char* name) {
  void* p = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q) == cudaSuccess && q == cudaDriverEntryPointSuccess)
    return reinterpret_cast<Fn>(p);
  return nullptr;
}

struct DriverFns {
  CtxGetCurrentFn get_cur = nullptr;
  CtxGetIdFn get_id = nullptr;
  EncodeFn encode = nullptr;
};

const DriverFns& driver() {
  static DriverFns fns;
  static std::once_flag once;
  std::call_once(once, [] {
    fns.get_cur = driver_entry<CtxGetCurrentFn>("cuCtxGetCurrent");
    fns.get_id = driver_entry<CtxGetIdFn>("cuCtxGetId");
    fns.encode = driver_entry<EncodeFn>("cuTensorMapEncodeTiled");
  });
  return fns;
}

// ---- per device and context ----------------------------------------------------

struct DeviceFacts {
  unsigned long long ctx = 0;  // context the facts below belong to
  int sms = 0;
  static constexpr int kMaxKernels = 32;
  const void* kernels[kMaxKernels] = {};
  size_t smem[kMaxKernels] = {};
  int n_kernels = 0;
};
DeviceFacts g_dev[kMaxDevices];
std::mutex g_dev_mu;

// The facts of the current device, reset when its context changed.
DeviceFacts* facts(int* dev_out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  const unsigned long long ctx = current_ctx_id();
  DeviceFacts& f = g_dev[dev];
  if (f.ctx != ctx || ctx == 0) {
    f = DeviceFacts{};
    f.ctx = ctx;
  }
  if (dev_out) *dev_out = dev;
  return &f;
}

// ---- tensor maps, per host thread ----------------------------------------------

struct MapKey {
  int dt, rank, swizzle;
  const void* base;
  uint64_t dims[5], strides[4];
  uint32_t box[5];
};

struct MapEntry {
  MapKey key;
  CUtensorMap map;
  bool used;
};

constexpr int kMapSlots = 16;
thread_local MapEntry t_maps[kMapSlots];
thread_local int t_next = 0;

}  // namespace

unsigned long long current_ctx_id() {
  const DriverFns& d = driver();
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (d.get_cur && d.get_id && d.get_cur(&ctx) == CUDA_SUCCESS && ctx && d.get_id(ctx, &id) == CUDA_SUCCESS) return id;
  return 0;
}

int sm_count() {
  std::lock_guard<std::mutex> lock(g_dev_mu);
  int dev = 0;
  DeviceFacts* f = facts(&dev);
  if (!f) return 148;
  if (f->sms == 0 && cudaDeviceGetAttribute(&f->sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    f->sms = 0;
  return f->sms > 0 ? f->sms : 148;
}

cudaError_t set_max_smem(const void* kernel, size_t bytes) {
  std::lock_guard<std::mutex> lock(g_dev_mu);
  DeviceFacts* f = facts(nullptr);
  if (f) {
    for (int i = 0; i < f->n_kernels; ++i)
      if (f->kernels[i] == kernel && f->smem[i] >= bytes) return cudaSuccess;
  }
  const cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e != cudaSuccess || !f) return e;
  for (int i = 0; i < f->n_kernels; ++i)
    if (f->kernels[i] == kernel) {
      f->smem[i] = bytes;
      return e;
    }
  if (f->n_kernels < DeviceFacts::kMaxKernels) {
    f->kernels[f->n_kernels] = kernel;
    f->smem[f->n_kernels] = bytes;
    ++f->n_kernels;
  }
  return e;
}

bool tensor_maps_available() { return driver().encode != nullptr; }

bool encode_tensor_map(CUtensorMap* map, CUtensorMapDataType dt, int rank, const void* base, const uint64_t* dims,
                       const uint64_t* strides_bytes, const uint32_t* box, CUtensorMapSwizzle sw) {
  const DriverFns& d = driver();
  if (!d.encode || rank < 1 || rank > 5) return false;
  MapKey key;
  std::memset(&key, 0, sizeof(key));
  key.dt = (int)dt;
  key.rank = rank;
  key.swizzle = (int)sw;
  key.base = base;
  for (int i = 0; i < rank; ++i) {
    key.dims[i] = dims[i];
    key.box[i] = box[i];
    if (i + 1 < rank) key.strides[i] = strides_bytes[i];
  }
  for (int i = 0; i < kMapSlots; ++i)
    if (t_maps[i].used && std::memcmp(&t_maps[i].key, &key, sizeof(key)) == 0) {
      *map = t_maps[i].map;
      return true;
    }
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  const CUresult r = d.encode(map, dt, (cuuint32_t)rank, const_cast<void*>(base), (const cuuint64_t*)dims,
                              (const cuuint64_t*)strides_bytes, (const cuuint32_t*)box, estr,
                              CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return false;
  MapEntry& e = t_maps[t_next];
  t_next = (t_next + 1) % kMapSlots;
  e.key = key;
  e.map = *map;
  e.used = true;
  return true;
}

}  // namespace csa
