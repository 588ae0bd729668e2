// Decode-time state of CSA/HCA sequences: the sliding window's raw tokens
// and the compressor's pending tokens, appended per step, with periodic
// checkpoints (kwkr.cn notes 4.4: a state cache beside the classical KV
// cache; periodic checkpointing every 1024 tokens).
//
//   state_append_kernel   one CTA per appended token: packs the token's KV
//                         vector into its window-ring row (the cache's row
//                         layout), and copies its two stream rows and gate
//                         logits into the stream rings
//   (compress_kernel in ring mode then emits the entries these tokens
//    complete)
//   state_ckpt_kernel     one CTA per (row, sequence): copies the window rows
//                         of positions P-W .. P-1 and the stream rows of
//                         P-m .. P-1 into checkpoint slot (P/every - 1) mod n,
//                         for the last multiple P of `every` the append
//                         crossed
//   state_restore_kernel  the reverse copy, for a sequence resuming at P
#include "common.cuh"
#include "kernels.h"

namespace csa {

namespace {

// Token row p of sequence b of a ring of `cap` rows.
__device__ __forceinline__ int64_t ring_row(int bs, int64_t cap, int64_t p) { return (int64_t)bs * cap + p % cap; }

// One appended token per CTA (d/4 threads, each 4 dims): window row, stream
// rows, gate logits.
template <bool kF32, bool kKvF32>
__global__ void __launch_bounds__(128) state_append_kernel(const csa_params p, const void* __restrict__ kv_new,
                                                           const void* __restrict__ a_new,
                                                           const void* __restrict__ b_new,
                                                           const float* __restrict__ gate_new,
                                                           const int32_t* __restrict__ pos0, int T,
                                                           uint8_t* __restrict__ win_rows, float* __restrict__ win_scale,
                                                           int64_t win_cap, void* __restrict__ a_ring,
                                                           void* __restrict__ b_ring, float* __restrict__ gate_ring,
                                                           int64_t s_cap) {
  __shared__ float red[32];
  pdl_wait();
  pdl_trigger();
  const int tq = blockIdx.x, bs = blockIdx.y;
  const int d = p.d, r = p.r;
  const int d0 = 4 * threadIdx.x;
  const int64_t pos = (int64_t)pos0[bs] + tq;
  const int64_t src = ((int64_t)bs * T + tq) * d + d0;
  // stream rows and gate logits: plain copies into the rings
  const int64_t srow = ring_row(bs, s_cap, pos);
  if (kF32) {
    reinterpret_cast<float4*>(reinterpret_cast<float*>(a_ring) + srow * d + d0)[0] =
        reinterpret_cast<const float4*>(reinterpret_cast<const float*>(a_new) + src)[0];
    reinterpret_cast<float4*>(reinterpret_cast<float*>(b_ring) + srow * d + d0)[0] =
        reinterpret_cast<const float4*>(reinterpret_cast<const float*>(b_new) + src)[0];
  } else {
    reinterpret_cast<uint2*>(reinterpret_cast<uint16_t*>(a_ring) + srow * d + d0)[0] =
        reinterpret_cast<const uint2*>(reinterpret_cast<const uint16_t*>(a_new) + src)[0];
    reinterpret_cast<uint2*>(reinterpret_cast<uint16_t*>(b_ring) + srow * d + d0)[0] =
        reinterpret_cast<const uint2*>(reinterpret_cast<const uint16_t*>(b_new) + src)[0];
  }
  if (threadIdx.x == 0) {
    const float2 g = reinterpret_cast<const float2*>(gate_new)[(int64_t)bs * T + tq];
    reinterpret_cast<float2*>(gate_ring)[srow] = g;
  }
  // window row: the token's KV vector in the cache's row layout
  float y[4];
  load4<kF32>(kv_new, src, y);
  const int64_t wrow = ring_row(bs, win_cap, pos);
  if (kKvF32) {
    reinterpret_cast<float4*>(reinterpret_cast<float*>(win_rows) + wrow * d + d0)[0] = make_float4(y[0], y[1], y[2], y[3]);
    return;
  }
  // scale = amax/448 over the non-RoPE dims (1 if they are all zero); codes
  // E4M3 round-to-nearest-even, saturating, of x/scale; RoPE dims BF16
  float am = 0.f;
  if (d0 < d - r) am = fmaxf(fmaxf(fabsf(y[0]), fabsf(y[1])), fmaxf(fabsf(y[2]), fabsf(y[3])));
  const float amax = block_max(am, red);
  const float sc = amax > 0.f ? amax / kE4M3Max : 1.f;
  uint8_t* row = win_rows + wrow * (int64_t)(d + r);
  if (d0 < d - r) {
    const uint32_t c = f32_to_e4m3_sat(y[0] / sc) | (f32_to_e4m3_sat(y[1] / sc) << 8) |
                       (f32_to_e4m3_sat(y[2] / sc) << 16) | (f32_to_e4m3_sat(y[3] / sc) << 24);
    *reinterpret_cast<uint32_t*>(row + d0) = c;
  } else {
    uint2 v;
    v.x = (uint32_t)f32_to_bf16_bits(y[0]) | ((uint32_t)f32_to_bf16_bits(y[1]) << 16);
    v.y = (uint32_t)f32_to_bf16_bits(y[2]) | ((uint32_t)f32_to_bf16_bits(y[3]) << 16);
    *reinterpret_cast<uint2*>(row + (d - r) + 2 * (d0 - (d - r))) = v;
  }
  if (threadIdx.x == 0) win_scale[wrow] = sc;
}

// Copies between the rings and a checkpoint slot.  grid (W + m, B); CTA j < W
// moves the window row of position P - W + j, CTA W + i the stream rows of
// position P - m + i.  to_ckpt: rings -> slot (after an append; P = the
// last multiple of `every` in (pos0, pos0 + T], none -> nothing); else slot
// -> rings (restore at P = pos[b]).  Window positions below 0 are stored as
// zero rows and not restored.
template <bool kF32, bool kKvF32>
__global__ void __launch_bounds__(128) state_ckpt_kernel(const csa_params p, const int32_t* __restrict__ pos0, int T,
                                                         bool to_ckpt, uint8_t* __restrict__ win_rows,
                                                         float* __restrict__ win_scale, int64_t win_cap,
                                                         void* __restrict__ a_ring, void* __restrict__ b_ring,
                                                         float* __restrict__ gate_ring, int64_t s_cap,
                                                         csa_ckpt ck, int32_t* __restrict__ err) {
  pdl_wait();
  pdl_trigger();
  const int j = blockIdx.x, bs = blockIdx.y;
  const int W = p.window, m = p.m, d = p.d, r = p.r;
  int64_t P;
  if (to_ckpt) {
    const int64_t hi = (int64_t)pos0[bs] + T;
    P = hi / ck.every * ck.every;
    if (P <= pos0[bs]) return;  // no multiple of `every` crossed
  } else {
    P = pos0[bs];
    if (P <= 0 || P % ck.every) {
      if (j == 0 && threadIdx.x == 0) raise_err(err, CSA_DEV_ERR_RANGE);
      return;
    }
  }
  const int64_t slot = (P / ck.every - 1) % ck.n_slots;
  const int64_t cslot = (int64_t)bs * ck.n_slots + slot;
  const int rb = kKvF32 ? 4 * d : d + r;
  if (j < W) {
    const int64_t pos = P - W + j;
    uint8_t* crow = reinterpret_cast<uint8_t*>(ck.win_rows) + (cslot * W + j) * (int64_t)rb;
    if (pos < 0) {
      if (to_ckpt) {
        for (int x = threadIdx.x; x < rb / 16; x += blockDim.x) reinterpret_cast<uint4*>(crow)[x] = make_uint4(0, 0, 0, 0);
        if (!kKvF32 && threadIdx.x == 0) ck.win_scale[cslot * W + j] = 0.f;
      }
      return;
    }
    uint8_t* wrow = win_rows + ring_row(bs, win_cap, pos) * (int64_t)rb;
    const uint4* from = reinterpret_cast<const uint4*>(to_ckpt ? wrow : crow);
    uint4* to = reinterpret_cast<uint4*>(to_ckpt ? crow : wrow);
    for (int x = threadIdx.x; x < rb / 16; x += blockDim.x) to[x] = from[x];
    if (!kKvF32 && threadIdx.x == 0) {
      float* ws = win_scale + ring_row(bs, win_cap, pos);
      float* cs = ck.win_scale + cslot * W + j;
      if (to_ckpt) *cs = *ws;
      else *ws = *cs;
    }
    return;
  }
  const int i = j - W;
  const int64_t pos = P - m + i;  // >= 0: P is a positive multiple of m
  const int64_t srow = ring_row(bs, s_cap, pos);
  const int64_t crow = cslot * m + i;
  const int eb = kF32 ? 4 : 2;  // bytes per stream element
  uint8_t* ar = reinterpret_cast<uint8_t*>(a_ring) + srow * d * eb;
  uint8_t* br = reinterpret_cast<uint8_t*>(b_ring) + srow * d * eb;
  uint8_t* ac = reinterpret_cast<uint8_t*>(ck.a) + crow * d * eb;
  uint8_t* bc = reinterpret_cast<uint8_t*>(ck.b) + crow * d * eb;
  for (int x = threadIdx.x; x < d * eb / 16; x += blockDim.x) {
    if (to_ckpt) {
      reinterpret_cast<uint4*>(ac)[x] = reinterpret_cast<const uint4*>(ar)[x];
      reinterpret_cast<uint4*>(bc)[x] = reinterpret_cast<const uint4*>(br)[x];
    } else {
      reinterpret_cast<uint4*>(ar)[x] = reinterpret_cast<const uint4*>(ac)[x];
      reinterpret_cast<uint4*>(br)[x] = reinterpret_cast<const uint4*>(bc)[x];
    }
  }
  if (threadIdx.x == 0) {
    float2* gr = reinterpret_cast<float2*>(gate_ring) + srow;
    float2* gc = reinterpret_cast<float2*>(ck.gate) + crow;
    if (to_ckpt) *gc = *gr;
    else *gr = *gc;
  }
}

template <bool kF32, bool kKvF32>
cudaError_t launch_ckpt_t(const csa_params& p, const int32_t* pos, int T, bool to_ckpt, const csa_state& s,
                          const csa_ckpt& ck, int32_t* err, cudaStream_t st) {
  return launch_pdl(state_ckpt_kernel<kF32, kKvF32>, dim3(p.window + p.m, p.B), dim3(128), 0, st, p, pos, T, to_ckpt,
                    reinterpret_cast<uint8_t*>(s.win.rows), s.win.scale, s.win.cap, s.a, s.b, s.gate, s.s_cap, ck, err);
}

cudaError_t launch_ckpt(const csa_params& p, const int32_t* pos, int T, bool to_ckpt, const csa_state& s,
                        const csa_ckpt& ck, int32_t* err, cudaStream_t st) {
  const bool f32 = p.act_fmt == CSA_ACT_F32, kv32 = p.kv_fmt == CSA_KV_F32;
  if (f32) return kv32 ? launch_ckpt_t<true, true>(p, pos, T, to_ckpt, s, ck, err, st)
                       : launch_ckpt_t<true, false>(p, pos, T, to_ckpt, s, ck, err, st);
  return kv32 ? launch_ckpt_t<false, true>(p, pos, T, to_ckpt, s, ck, err, st)
              : launch_ckpt_t<false, false>(p, pos, T, to_ckpt, s, ck, err, st);
}

}  // namespace

cudaError_t launch_state_append(const csa_params& p, const void* kv_new, const void* a_new, const void* b_new,
                                const float* gate_new, const int32_t* pos0, int T, const csa_state& s,
                                const csa_kv& cache, int32_t* cache_pos, const csa_ckpt* ck, int32_t* err,
                                cudaStream_t st) {
  const bool f32 = p.act_fmt == CSA_ACT_F32, kv32 = p.kv_fmt == CSA_KV_F32;
  auto kfn = f32 ? (kv32 ? state_append_kernel<true, true> : state_append_kernel<true, false>)
                 : (kv32 ? state_append_kernel<false, true> : state_append_kernel<false, false>);
  cudaError_t e = launch_pdl(kfn, dim3(T, p.B), dim3(p.d / 4), 0, st, p, kv_new, a_new, b_new, gate_new, pos0, T,
                             reinterpret_cast<uint8_t*>(s.win.rows), s.win.scale, s.win.cap, s.a, s.b, s.gate, s.s_cap);
  if (e != cudaSuccess) return e;
  e = launch_compress_ring(p, s.a, s.b, s.gate, s.s_cap, pos0, T, cache, cache_pos, err, st);
  if (e != cudaSuccess) return e;
  if (ck) {
    e = launch_ckpt(p, pos0, T, true, s, *ck, err, st);
    if (e != cudaSuccess) return e;
  }
  return cudaGetLastError();
}

cudaError_t launch_state_restore(const csa_params& p, const int32_t* pos, const csa_ckpt& ck, const csa_state& s,
                                 int32_t* err, cudaStream_t st) {
  cudaError_t e = launch_ckpt(p, pos, 0, false, s, ck, err, st);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace csa
