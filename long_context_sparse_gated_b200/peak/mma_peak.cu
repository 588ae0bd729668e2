// Dense tensor-core throughput probe for the roofline denominators of the
// benchmark (not part of the CSA/HCA library): every SM's CTA issues a long
// run of back-to-back tcgen05.mma instructions of one kind from one thread,
// M = 128, N = 256, into one TMEM accumulator, and the host times the launch.
//
//   kind 0  kind::mxf4.block_scale (E2M1 x E2M1, UE8M0 per 32), K = 64
//   kind 1  kind::f16 with BF16 operands, K = 16
//
// Operands are whatever the shared memory holds (zeros): throughput does
// not depend on the values.  The one wait (for the final commit) is bounded
// and reports a timeout in *err instead of hanging.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../csrc/sm100.cuh"

namespace {

constexpr int kN = 256;
constexpr uint32_t kCols = 512;

struct __align__(1024) PeakSmem {
  uint8_t a[128 * 64];   // A: 128 rows x 64 B (mxf4 K = 128 nibbles; bf16 K = 32)
  uint8_t b[kN * 64];    // B: 256 rows x 64 B
  uint32_t sf[128];      // scale bytes for tcgen05.cp (all 127 = 2^0)
  uint64_t bar;
  uint32_t tmem;
  int abort;
};

__global__ void __launch_bounds__(128, 1) mma_peak_kernel(int kind, int iters, int* err) {
  extern __shared__ uint8_t raw[];
  PeakSmem& S = *reinterpret_cast<PeakSmem*>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
  using namespace csa::sm100;
  for (int i = threadIdx.x; i < (int)sizeof(S.a) / 4; i += blockDim.x) reinterpret_cast<uint32_t*>(S.a)[i] = 0u;
  for (int i = threadIdx.x; i < (int)sizeof(S.b) / 4; i += blockDim.x) reinterpret_cast<uint32_t*>(S.b)[i] = 0u;
  if (threadIdx.x < 128) S.sf[threadIdx.x] = 0x7F7F7F7Fu;
  if (threadIdx.x == 0) {
    mbar_init(&S.bar, 1);
    S.abort = 0;
    fence_mbar_init();
  }
  if (threadIdx.x < 32) {
    tmem_alloc(&S.tmem, kCols);
    tmem_relinquish();
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = S.tmem;
  if (threadIdx.x == 0) {
    const uint32_t d = tmem, sfa = tmem + 256, sfb = tmem + 260;
    const uint64_t sd = smem_desc(smem_u32(S.sf), 0, 128, 0);
    tc_cp_32x128b_warpx4(sfa, sd);
    tc_cp_32x128b_warpx4(sfb, sd);
    // K-major, 64-byte rows, 64B swizzle: 8-row groups 512 B apart
    const uint64_t ad = smem_desc(smem_u32(S.a), 16, 512, 4);
    const uint64_t bd = smem_desc(smem_u32(S.b), 16, 512, 4);
    if (kind == 0) {
      const uint32_t id = idesc_mxf4(128, kN, 0, 0);
      for (int i = 0; i < iters; ++i) mma_mxf4(d, ad, bd, id, sfa, sfb, i > 0);
    } else {
      const uint32_t id = idesc_bf16(128, kN, 0, 0);
      for (int i = 0; i < iters; ++i) mma_f16(d, ad, bd, id, i > 0);
    }
    tc_commit(&S.bar);
    volatile int* ab = &S.abort;
    if (!mbar_wait(&S.bar, 0, ab)) atomicOr(err, 4);
  }
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x < 32) {
    tc_fence_after();
    tmem_dealloc(tmem, kCols);
  }
}

}  // namespace

// Runs the probe on every SM and returns the dense tensor throughput in
// TFLOP/s (2*M*N*K flops per MMA), or a negative value on a CUDA error or a
// timed-out wait.  kind: 0 = MXFP4 (kind::mxf4), 1 = BF16 (kind::f16).
extern "C" double csa_peak_mma_tflops(int kind, int iters, int reps) {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1.0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1.0;
  // enough shared memory that one CTA (one TMEM allocation) fits per SM
  const size_t smem = 120 * 1024;
  static_assert(sizeof(PeakSmem) + 1024 <= 120 * 1024, "probe shared memory");
  if (cudaFuncSetAttribute(mma_peak_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return -1.0;
  int* err = nullptr;
  if (cudaMalloc(&err, sizeof(int)) != cudaSuccess) return -1.0;
  cudaMemset(err, 0, sizeof(int));
  cudaEvent_t e0, e1;
  cudaEventCreate(&e0);
  cudaEventCreate(&e1);
  mma_peak_kernel<<<sms, 128, smem>>>(kind, iters, err);  // warm-up
  float best = 1e30f;
  for (int r = 0; r < reps; ++r) {
    cudaEventRecord(e0);
    mma_peak_kernel<<<sms, 128, smem>>>(kind, iters, err);
    cudaEventRecord(e1);
    cudaEventSynchronize(e1);
    float ms = 0.f;
    cudaEventElapsedTime(&ms, e0, e1);
    if (ms < best) best = ms;
  }
  int h_err = 0;
  cudaError_t ce = cudaMemcpy(&h_err, err, sizeof(int), cudaMemcpyDeviceToHost);
  cudaFree(err);
  cudaEventDestroy(e0);
  cudaEventDestroy(e1);
  if (ce != cudaSuccess || cudaGetLastError() != cudaSuccess || h_err) return -1.0;
  const double k = kind == 0 ? 64.0 : 16.0;
  const double flops = (double)sms * iters * 2.0 * 128.0 * kN * k;
  return flops / (best * 1e-3) / 1e12;
}
