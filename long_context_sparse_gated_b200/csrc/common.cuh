// Device helpers shared by the CSA/HCA kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp4.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "csa.h"

namespace csa {

constexpr float kE4M3Max = 448.0f;

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t v) {
  return __uint_as_float((v & 0xFFFFu) << 16);
}

__device__ __forceinline__ uint16_t f32_to_bf16_bits(float f) {
  __nv_bfloat16 h = __float2bfloat16_rn(f);
  return *reinterpret_cast<uint16_t*>(&h);
}

__device__ __forceinline__ float e4m3_to_f32(uint32_t code) {
  __half_raw h = __nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(code & 0xFF), __NV_E4M3);
  return __half2float(__half(h));
}

// round to nearest even, saturating to +-448
__device__ __forceinline__ uint32_t f32_to_e4m3_sat(float f) {
  return static_cast<uint32_t>(__nv_cvt_float_to_fp8(f, __NV_SATFINITE, __NV_E4M3));
}

// E2M1 nibble -> float, assembled from the bit fields (OCP MX: bias 1, one
// mantissa bit, exponent field 0 is the subnormal 0 / 0.5).
__device__ __forceinline__ float e2m1_to_f32(uint32_t n) {
  uint32_t e = (n >> 1) & 3u, mt = n & 1u, s = (n >> 3) & 1u;
  uint32_t bits = e ? (((e + 126u) << 23) | (mt << 22)) : (mt ? (126u << 23) : 0u);
  return __uint_as_float(bits | (s << 31));
}

// UE8M0 scale byte -> 2^(E-127); 0xFF -> NaN
__device__ __forceinline__ float ue8m0_to_f32(uint32_t e) {
  e &= 0xFFu;
  if (e == 0xFFu) return __uint_as_float(0x7FC00000u);
  if (e == 0u) return __uint_as_float(0x00400000u);
  return __uint_as_float(e << 23);
}

// Programmatic dependent launch.  Kernels launched with launch_pdl() may
// start while the previous kernel on the stream is finishing; pdl_wait()
// blocks until that kernel has completed and its memory is visible, so every
// kernel calls it before reading any global input.  pdl_trigger() lets the
// next kernel's CTAs be scheduled early (they still wait in pdl_wait()).
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ void raise_err(int32_t* err, int32_t bits) {
  if (err) atomicOr(err, bits);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Block-wide reductions; `red` holds >= 32 floats.  All threads must call.
__device__ __forceinline__ float block_sum(float v, float* red) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = (blockDim.x + 31) >> 5;
  v = warp_sum(v);
  __syncthreads();
  if (lane == 0) red[wid] = v;
  __syncthreads();
  float r = (lane < nw) ? red[lane] : 0.f;
  r = warp_sum(r);
  return r;
}

__device__ __forceinline__ float block_max(float v, float* red) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = (blockDim.x + 31) >> 5;
  v = warp_max(v);
  __syncthreads();
  if (lane == 0) red[wid] = v;
  __syncthreads();
  float r = (lane < nw) ? red[lane] : -INFINITY;
  r = warp_max(r);
  return r;
}

// Order-preserving 32-bit key of an fp32 score: a larger score gives a
// larger key, and -0 and +0 give the same key.
__device__ __forceinline__ uint32_t score_key(float f) {
  uint32_t u = __float_as_uint(f);
  if ((u & 0x7FFFFFFFu) == 0) u = 0;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Warp-aggregated increment of hist[bin] for the lanes with `active` set.
// Every lane of the warp must call it.
__device__ __forceinline__ void hist_add(uint32_t* hist, uint32_t bin, bool active) {
  const unsigned act = __ballot_sync(0xffffffffu, active);
  if (!active) return;
  const unsigned peers = __match_any_sync(act, bin);
  const int leader = __ffs(peers) - 1;
  if ((int)(threadIdx.x & 31) == leader) atomicAdd(&hist[bin], (uint32_t)__popc(peers));
}

// Four consecutive values from f32 or BF16 storage (element offset `off`,
// a multiple of 4).
template <bool kF32>
__device__ __forceinline__ void load4(const void* base, int64_t off, float v[4]) {
  if (kF32) {
    float4 x = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(base) + off);
    v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w;
  } else {
    uint2 x = *reinterpret_cast<const uint2*>(reinterpret_cast<const uint16_t*>(base) + off);
    v[0] = bf16_bits_to_f32(x.x); v[1] = bf16_bits_to_f32(x.x >> 16);
    v[2] = bf16_bits_to_f32(x.y); v[3] = bf16_bits_to_f32(x.y >> 16);
  }
}

// OCP MX v1.0 conversion (section 6.3) of one 32-value block held as 4
// values by each of 8 consecutive lanes (`mask` = those lanes): the shared
// exponent is X = floor(log2 amax) - 2 (E2M1's largest exponent is 2),
// clamped to [-127, 127] (an all-zero block takes -127), and each value
// becomes the E2M1 code of v * 2^-X, rounded to nearest even and
// saturated.  Returns this lane's two packed bytes (value 0 in the low
// nibble of the low byte) and sets *sbyte = X + 127 (the UE8M0 scale).
__device__ __forceinline__ uint32_t mxfp4_encode_quad(const float v[4], unsigned mask, uint32_t* sbyte) {
  float am = fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3])));
  am = fmaxf(am, __shfl_xor_sync(mask, am, 1));
  am = fmaxf(am, __shfl_xor_sync(mask, am, 2));
  am = fmaxf(am, __shfl_xor_sync(mask, am, 4));
  // floor(log2 am) from the exponent field; a subnormal (or zero) amax
  // gives an exponent below -127 after the -2, i.e. the clamp
  const int e = (int)((__float_as_uint(am) >> 23) & 0xFFu);
  int X = e ? e - 127 - 2 : -127;
  X = max(-127, min(125, X));
  const float inv = __uint_as_float((uint32_t)(127 - X) << 23);  // 2^-X, X in [-127, 125]
  const uint32_t b0 = __nv_cvt_float2_to_fp4x2(make_float2(v[0] * inv, v[1] * inv), __NV_E2M1, cudaRoundNearest);
  const uint32_t b1 = __nv_cvt_float2_to_fp4x2(make_float2(v[2] * inv, v[3] * inv), __NV_E2M1, cudaRoundNearest);
  *sbyte = (uint32_t)(X + 127);
  return (b0 & 0xFFu) | ((b1 & 0xFFu) << 8);
}

// Order-preserving 16-bit key of a BF16 score (its bit pattern), -0 == +0.
__device__ __forceinline__ uint32_t score_key16(uint32_t bits) {
  bits &= 0xFFFFu;
  if ((bits & 0x7FFFu) == 0) bits = 0;
  return (bits & 0x8000u) ? (~bits & 0xFFFFu) : (bits | 0x8000u);
}

// Bins of the per-query score histogram: the top 12 bits of the key (of
// the 32-bit key of an fp32 score, or of the 16-bit key of a BF16 score).
constexpr int kScoreHistBins = 4096;
__device__ __forceinline__ uint32_t score_bin(float f) { return score_key(f) >> 20; }
__device__ __forceinline__ uint32_t score_bin16(uint32_t bits) { return score_key16(bits) >> 4; }

// RoPE angle of pair j (of r/2) at position pos, in double precision so that
// positions up to 2^20 and beyond keep a small absolute angle error.
__device__ __forceinline__ void rope_cos_sin(double pos, int j, int r, double theta, float* c, float* s) {
  double freq = pow(theta, -2.0 * (double)j / (double)r);
  double sn, cs;
  sincos(pos * freq, &sn, &cs);
  *c = (float)cs;
  *s = (float)sn;
}

}  // namespace csa
