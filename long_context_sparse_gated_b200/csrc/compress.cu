// Gated two-stream token compressor (CSA m=4, HCA m=128) with RMSNorm,
// partial RoPE and the mixed FP8/BF16 pack, one CTA per (entry, sequence).
//
// kwkr.cn notes 3.1 (two KV streams merged with softmax-normalised gate
// weights, adjacent blocks overlap), 3.2 (HCA: 128 tokens per entry);
// Qiaomu blog 混合注意力机制 (entries normalised, RoPE on part of the dims);
// WeChat 未来科技 1.1 (RoPE on the last 64 dims; RoPE dims BF16, others FP8).
//
// Thread layout: the d dims are split into d/4 quads; G = blockDim/(d/4)
// thread groups each sum a strided subset of the 2m token rows, then the
// groups' partial sums are reduced in shared memory.  Every stream row is
// read once with 8-byte (bf16) or 16-byte (f32) coalesced loads.
#include "common.cuh"
#include "kernels.h"

namespace csa {

// Output of the compressor: f32 rows, the mixed FP8/BF16 KV rows, or MXFP4
// index-key rows (the indexer's keys come from the same operator).
enum { kOutF32 = 0, kOutFp8 = 1, kOutMxfp4 = 2 };

template <bool kF32, int kOut>
__global__ void __launch_bounds__(1024) compress_kernel(
    const csa_params p, const void* __restrict__ a, const void* __restrict__ b,
    const float* __restrict__ gate, int64_t S, const int32_t* __restrict__ tok_base,
    const int32_t* __restrict__ e_begin, const int32_t* __restrict__ e_end,
    const float* __restrict__ norm_w, uint8_t* __restrict__ rows, float* __restrict__ scale,
    int64_t cap, int32_t* __restrict__ out_pos, int32_t* __restrict__ err, int64_t ring, int T_new) {
  extern __shared__ float smem[];
  const int m = p.m, d = p.d, r = p.r;
  const int quads = d >> 2;
  const int G = blockDim.x / quads;  // token groups
  float* w = smem;                    // [2m] gate weights
  float* part = smem + 2 * m;         // [G][d] partial sums
  __shared__ float red[32];

  pdl_wait();
  pdl_trigger();
  const int bs = blockIdx.y;
  // Linear buffers: entries [e_begin, e_end), token p at row p - tok_base.
  // Ring buffers (ring > 0, the decode state): e_begin holds the position
  // of the first of T_new appended tokens; the entries they complete are
  // [pos0/m, (pos0+T_new)/m), and token p sits at row p mod ring.
  const int64_t eb = ring ? (int64_t)e_begin[bs] / m : (int64_t)e_begin[bs];
  const int64_t ee = ring ? ((int64_t)e_begin[bs] + T_new) / m : (int64_t)e_end[bs];
  const int64_t e = eb + blockIdx.x;
  if (e >= ee) return;
  const int64_t base = ring ? 0 : tok_base[bs];
  const int nb = e > 0 ? m : 0;
  const int64_t ia0 = ring ? ((int64_t)m * e) % ring : (int64_t)m * e - base;
  const int64_t ib0 = ring ? (e > 0 ? ((int64_t)m * (e - 1)) % ring : 0) : (int64_t)m * (e - 1) - base;
  if (e >= cap || (!ring && (ia0 < 0 || ia0 + m > S || (nb && ib0 < 0)))) {
    if (threadIdx.x == 0) raise_err(err, CSA_DEV_ERR_RANGE);
    return;
  }
  const int n = m + nb;
  const int64_t row0 = (int64_t)bs * S;
  const int q = threadIdx.x % quads, g = threadIdx.x / quads;
  const int d0 = q * 4;

  // Latency overlap: the first kPre rows of this thread's token group and
  // (for the RoPE dims) the rotation of position m*e are fetched / computed
  // before the gate softmax, which they do not depend on.
  constexpr int kPre = 4;
  float pre[kPre][4];
#pragma unroll
  for (int k = 0; k < kPre; ++k) {
    const int i = g + k * G;
    if (g < G && i < n) {
      if (i < m)
        load4<kF32>(a, (row0 + ia0 + i) * d + d0, pre[k]);
      else
        load4<kF32>(b, (row0 + ib0 + (i - m)) * d + d0, pre[k]);
    }
  }
  float rc[2] = {1.f, 1.f}, rs_[2] = {0.f, 0.f};
  if (threadIdx.x < quads && d0 >= d - r) {
#pragma unroll
    for (int pr = 0; pr < 2; ++pr) rope_cos_sin((double)(m * e), (d0 + 2 * pr - (d - r)) >> 1, r, (double)p.rope_theta,
                                                &rc[pr], &rs_[pr]);
  }

  // 1. softmax over the union of both streams' logits
  float lmax = -INFINITY;
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const float gl = i < m ? gate[(row0 + ia0 + i) * 2 + 0] : gate[(row0 + ib0 + (i - m)) * 2 + 1];
    w[i] = gl;
    lmax = fmaxf(lmax, gl);
  }
  const float gmax = block_max(lmax, red);
  float lsum = 0.f;
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    float ex = expf(w[i] - gmax);
    w[i] = ex;
    lsum += ex;
  }
  const float inv = 1.f / block_sum(lsum, red);  // block_sum syncs: w[] is visible

  // 2. weighted merge: group g sums rows i = g, g+G, ...
  float x[4] = {0.f, 0.f, 0.f, 0.f};
  if (g < G) {
#pragma unroll
    for (int k = 0; k < kPre; ++k) {
      const int i = g + k * G;
      if (i < n) {
        const float wi = w[i] * inv;
        x[0] = fmaf(wi, pre[k][0], x[0]); x[1] = fmaf(wi, pre[k][1], x[1]);
        x[2] = fmaf(wi, pre[k][2], x[2]); x[3] = fmaf(wi, pre[k][3], x[3]);
      }
    }
#pragma unroll 4
    for (int i = g + kPre * G; i < n; i += G) {
      float v[4];
      if (i < m)
        load4<kF32>(a, (row0 + ia0 + i) * d + d0, v);
      else
        load4<kF32>(b, (row0 + ib0 + (i - m)) * d + d0, v);
      const float wi = w[i] * inv;
      x[0] = fmaf(wi, v[0], x[0]); x[1] = fmaf(wi, v[1], x[1]);
      x[2] = fmaf(wi, v[2], x[2]); x[3] = fmaf(wi, v[3], x[3]);
    }
    *reinterpret_cast<float4*>(part + g * d + d0) = make_float4(x[0], x[1], x[2], x[3]);
  }
  __syncthreads();
  const bool owner = threadIdx.x < quads;  // group 0 finishes the entry
  float y[4] = {0.f, 0.f, 0.f, 0.f};
  if (owner) {
    for (int gg = 0; gg < G; ++gg) {
      float4 t = *reinterpret_cast<const float4*>(part + gg * d + d0);
      y[0] += t.x; y[1] += t.y; y[2] += t.z; y[3] += t.w;
    }
  }
  // 3. RMSNorm
  float ss = owner ? (y[0] * y[0] + y[1] * y[1] + y[2] * y[2] + y[3] * y[3]) : 0.f;
  const float tot = block_sum(ss, red);
  const float rsq = 1.f / sqrtf(tot / (float)d + p.eps);
  if (!owner) return;  // no block-wide barrier below this point except via red in FP8 path
#pragma unroll
  for (int k = 0; k < 4; ++k) y[k] *= rsq * (norm_w ? norm_w[d0 + k] : 1.f);
  // 4. RoPE on the last r dims, pairs (d-r+2j, d-r+2j+1), angle (m*e)*theta^(-2j/r)
  if (d0 >= d - r) {
#pragma unroll
    for (int pr = 0; pr < 2; ++pr) {
      const float c = rc[pr], s = rs_[pr];
      const float x0 = y[2 * pr], x1 = y[2 * pr + 1];
      y[2 * pr] = x0 * c - x1 * s;
      y[2 * pr + 1] = x0 * s + x1 * c;
    }
  }
  const int64_t slot = (int64_t)bs * cap + e;
  if (out_pos && threadIdx.x == 0) out_pos[slot] = (int32_t)(m * e);
  if (kOut == kOutMxfp4) {
    // OCP MX conversion per 32 dims: eight consecutive owner lanes hold a
    // block; 2 packed bytes per lane, one scale byte per block
    const unsigned mask = 0xFFu << (threadIdx.x & 24);
    uint32_t sb;
    const uint32_t bytes = mxfp4_encode_quad(y, mask, &sb);
    reinterpret_cast<uint16_t*>(rows + slot * (d / 2))[q] = (uint16_t)bytes;
    if ((q & 7) == 0) reinterpret_cast<uint8_t*>(scale)[slot * (d / 32) + (q >> 3)] = (uint8_t)sb;
    return;
  }
  if (kOut == kOutF32) {
    *reinterpret_cast<float4*>(reinterpret_cast<float*>(rows) + slot * d + d0) =
        make_float4(y[0], y[1], y[2], y[3]);
    return;
  }
  // 5. pack: E4M3 codes of x/scale (scale = amax/448 over the non-RoPE
  //    dims) and BF16 RoPE dims.  Only the `quads` owner threads (a whole
  //    number of warps when quads % 32 == 0) take part from here on.
  float am = 0.f;
  if (d0 < d - r) am = fmaxf(fmaxf(fabsf(y[0]), fabsf(y[1])), fmaxf(fabsf(y[2]), fabsf(y[3])));
  am = warp_max(am);
  __shared__ float wmax[32];
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  if (lane == 0) wmax[wid] = am;
  asm volatile("bar.sync 1, %0;" ::"r"(quads));  // named barrier over the owners
  float amax = 0.f;
  for (int i = 0; i < (quads + 31) / 32; ++i) amax = fmaxf(amax, wmax[i]);
  const float sc = amax > 0.f ? amax / kE4M3Max : 1.f;
  const int64_t rb = (int64_t)(d + r);
  uint8_t* row = rows + slot * rb;
  if (d0 < d - r) {
    uint32_t c = f32_to_e4m3_sat(y[0] / sc) | (f32_to_e4m3_sat(y[1] / sc) << 8) |
                 (f32_to_e4m3_sat(y[2] / sc) << 16) | (f32_to_e4m3_sat(y[3] / sc) << 24);
    *reinterpret_cast<uint32_t*>(row + d0) = c;
  } else {
    uint2 v;
    v.x = (uint32_t)f32_to_bf16_bits(y[0]) | ((uint32_t)f32_to_bf16_bits(y[1]) << 16);
    v.y = (uint32_t)f32_to_bf16_bits(y[2]) | ((uint32_t)f32_to_bf16_bits(y[3]) << 16);
    *reinterpret_cast<uint2*>(row + (d - r) + 2 * (d0 - (d - r))) = v;
  }
  if (threadIdx.x == 0) scale[slot] = sc;
}

cudaError_t launch_compress(const csa_params& p, const void* a, const void* b, const float* gate,
                            int64_t S, const int32_t* tok_base, const int32_t* e_begin,
                            const int32_t* e_end, int32_t max_entries, const float* norm_w,
                            const csa_kv& out, int32_t* out_pos, int32_t* err, cudaStream_t st) {
  const int quads = p.d / 4;
  // more token groups for long blocks (HCA): more loads in flight per entry
  int threads = p.m >= 64 ? 1024 : 256;
  if (threads < quads) threads = quads;
  const int G = threads / quads;
  const size_t smem = (size_t)(2 * p.m + G * p.d) * sizeof(float);
  dim3 grid(max_entries, p.B);
  const bool f32 = p.act_fmt == CSA_ACT_F32, kv32 = p.kv_fmt == CSA_KV_F32;
  auto* rows = reinterpret_cast<uint8_t*>(out.rows);
  auto kfn = f32 ? (kv32 ? compress_kernel<true, kOutF32> : compress_kernel<true, kOutFp8>)
                 : (kv32 ? compress_kernel<false, kOutF32> : compress_kernel<false, kOutFp8>);
  cudaError_t e = launch_pdl(kfn, grid, dim3(threads), smem, st, p, a, b, gate, S, tok_base, e_begin, e_end, norm_w,
                             rows, out.scale, out.cap, out_pos, err, (int64_t)0, 0);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// The entries completed by T_new tokens appended at pos0[b], read from the
// stream rings (token p at row p mod ring).
cudaError_t launch_compress_ring(const csa_params& p, const void* a, const void* b, const float* gate, int64_t ring,
                                 const int32_t* pos0, int T_new, const csa_kv& out, int32_t* out_pos, int32_t* err,
                                 cudaStream_t st) {
  const int quads = p.d / 4;
  int threads = p.m >= 64 ? 1024 : 256;
  if (threads < quads) threads = quads;
  const int G = threads / quads;
  const size_t smem = (size_t)(2 * p.m + G * p.d) * sizeof(float);
  const int max_entries = (T_new + p.m - 1) / p.m;  // block ends among T_new consecutive tokens
  dim3 grid(max_entries, p.B);
  const bool f32 = p.act_fmt == CSA_ACT_F32, kv32 = p.kv_fmt == CSA_KV_F32;
  auto kfn = f32 ? (kv32 ? compress_kernel<true, kOutF32> : compress_kernel<true, kOutFp8>)
                 : (kv32 ? compress_kernel<false, kOutF32> : compress_kernel<false, kOutFp8>);
  cudaError_t e = launch_pdl(kfn, grid, dim3(threads), smem, st, p, a, b, gate, ring, (const int32_t*)nullptr, pos0,
                             (const int32_t*)nullptr, (const float*)nullptr, reinterpret_cast<uint8_t*>(out.rows),
                             out.scale, out.cap, out_pos, err, ring, T_new);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// Index keys: the compressor over the idx_dim-dim indexer streams with RoPE
// on their last rope_dims dims, written as MXFP4 rows (idx_dim/2 bytes) and
// UE8M0 scales (idx_dim/32 bytes) per entry.
cudaError_t launch_index_compress(const csa_params& p, int rope_dims, const void* a, const void* b,
                                  const float* gate, int64_t S, const int32_t* tok_base, const int32_t* e_begin,
                                  const int32_t* e_end, int32_t max_entries, const float* norm_w, void* k_idx,
                                  uint8_t* k_idx_sf, int64_t k_cap, int32_t* err, cudaStream_t st) {
  csa_params q = p;
  q.d = p.idx_dim;
  q.r = rope_dims;
  const int quads = q.d / 4;
  const int threads = 256;
  const int G = threads / quads;
  const size_t smem = (size_t)(2 * q.m + G * q.d) * sizeof(float);
  dim3 grid(max_entries, p.B);
  auto kfn = p.act_fmt == CSA_ACT_F32 ? compress_kernel<true, kOutMxfp4> : compress_kernel<false, kOutMxfp4>;
  cudaError_t e = launch_pdl(kfn, grid, dim3(threads), smem, st, q, a, b, gate, S, tok_base, e_begin, e_end, norm_w,
                             reinterpret_cast<uint8_t*>(k_idx), reinterpret_cast<float*>(k_idx_sf), k_cap,
                             (int32_t*)nullptr, err, (int64_t)0, 0);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// Index queries (or any rows of idx_dim values) to MXFP4 by the OCP MX
// conversion: one thread per 4 values, eight threads per 32-value block.
template <bool kF32>
__global__ void __launch_bounds__(256) index_quantize_kernel(const void* __restrict__ x, int64_t n_quads,
                                                             uint8_t* __restrict__ out, uint8_t* __restrict__ out_sf) {
  pdl_wait();
  pdl_trigger();
  const int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (g - (threadIdx.x & 7) >= n_quads) return;  // whole 8-lane groups leave together
  float v[4];
  load4<kF32>(x, g * 4, v);
  uint32_t sb;
  const uint32_t bytes = mxfp4_encode_quad(v, 0xFFu << (threadIdx.x & 24), &sb);
  reinterpret_cast<uint16_t*>(out)[g] = (uint16_t)bytes;
  if ((threadIdx.x & 7) == 0) out_sf[g >> 3] = (uint8_t)sb;
}

cudaError_t launch_index_quantize(const csa_params& p, const void* x, int64_t n_rows, void* out, uint8_t* out_sf,
                                  cudaStream_t st) {
  const int64_t n_quads = n_rows * (p.idx_dim / 4);
  if (n_quads == 0) return cudaSuccess;
  const int64_t blocks = (n_quads + 255) / 256;
  auto kfn = p.act_fmt == CSA_ACT_F32 ? index_quantize_kernel<true> : index_quantize_kernel<false>;
  cudaError_t e = launch_pdl(kfn, dim3((unsigned)blocks), dim3(256), 0, st, x, n_quads, reinterpret_cast<uint8_t*>(out),
                             out_sf);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace csa
