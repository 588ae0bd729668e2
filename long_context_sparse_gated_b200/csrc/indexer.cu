// Lightning Indexer scores and exact top-k selection.
//
// Qiaomu blog 混合注意力机制 (a low-cost query per index head scores every
// compressed entry, top-k entries are kept); FP4量化感知训练 and kwkr.cn notes
// 3.4 / 4.4 (the indexer QK runs in FP4); PACMAN notes 3.1 (top-k 512 for
// V4-Flash, 1024 for V4-Pro).
//
//   I(t, s) = sum_h w_h * max(0, q_h . k_s),   s < n_t = floor((t+1)/m)
//
// index_scores_simt: CUDA-core reference path, one thread per entry, the
// query's heads decoded once per CTA into shared memory.  Summation order:
// per head over dims 0..c-1, then over heads 0..H-1, in fp32.
//
// topk_radix: one CTA per query; 4 passes of an 8-bit radix select on an
// order-preserving 32-bit key of the fp32 score find the k-th largest
// score; a final pass in index order keeps every entry above it plus the
// lowest-index entries equal to it, which yields the unique
// (score desc, index asc) top-k directly in ascending index order.
#include "common.cuh"
#include "kernels.h"

namespace csa {

template <int kHMax, int kC, bool kMx>
__global__ void __launch_bounds__(256) index_scores_simt(
    const csa_params p, const void* __restrict__ q_idx, const uint8_t* __restrict__ q_sf,
    const float* __restrict__ w, const void* __restrict__ k_idx, const uint8_t* __restrict__ k_sf,
    int64_t k_cap, const int32_t* __restrict__ q_pos0, int T, float* __restrict__ scores,
    int n_max, int32_t* __restrict__ err) {
  __shared__ float qs[kHMax * kC];
  __shared__ float ws[kHMax];
  const int H = p.n_idx_heads;
  const int qi = blockIdx.x;
  const int bs = qi / T, tq = qi % T;
  const int64_t t = (int64_t)q_pos0[bs] + tq;
  int64_t n_t = (t + 1) / p.m;
  if (n_t > n_max || n_t > k_cap) {
    if (threadIdx.x == 0 && blockIdx.y == 0) raise_err(err, CSA_DEV_ERR_RANGE);
    n_t = (int64_t)n_max < k_cap ? (int64_t)n_max : k_cap;
  }
  const int s0 = blockIdx.y * blockDim.x;
  if (s0 >= n_t) return;
  // decode the query's heads
  for (int i = threadIdx.x; i < H * kC; i += blockDim.x) {
    const int h = i / kC, c = i % kC;
    float v;
    if (kMx) {
      const uint8_t* qb = reinterpret_cast<const uint8_t*>(q_idx) + ((int64_t)qi * H + h) * (kC / 2);
      const uint32_t byte = qb[c >> 1];
      v = e2m1_to_f32((c & 1) ? (byte >> 4) : byte) *
          ue8m0_to_f32(q_sf[((int64_t)qi * H + h) * (kC / 32) + c / 32]);
    } else {
      v = reinterpret_cast<const float*>(q_idx)[((int64_t)qi * H + h) * kC + c];
    }
    qs[i] = v;
  }
  for (int h = threadIdx.x; h < H; h += blockDim.x) ws[h] = w[(int64_t)qi * H + h];
  __syncthreads();
  const int64_t s = s0 + threadIdx.x;
  if (s >= n_t) return;
  float acc[kHMax];
#pragma unroll
  for (int h = 0; h < kHMax; ++h) acc[h] = 0.f;
#pragma unroll 1
  for (int blk = 0; blk < kC / 32; ++blk) {
    float kv[32];
    if (kMx) {
      const uint8_t* kb = reinterpret_cast<const uint8_t*>(k_idx) + ((int64_t)bs * k_cap + s) * (kC / 2) + blk * 16;
      const float sc = ue8m0_to_f32(k_sf[((int64_t)bs * k_cap + s) * (kC / 32) + blk]);
      const uint4 raw = *reinterpret_cast<const uint4*>(kb);
      const uint32_t wd[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
      for (int i = 0; i < 32; ++i) kv[i] = e2m1_to_f32(wd[i >> 3] >> (4 * (i & 7))) * sc;
    } else {
      const float* kf = reinterpret_cast<const float*>(k_idx) + ((int64_t)bs * k_cap + s) * kC + blk * 32;
#pragma unroll
      for (int i = 0; i < 32; i += 4) {
        const float4 v = *reinterpret_cast<const float4*>(kf + i);
        kv[i] = v.x; kv[i + 1] = v.y; kv[i + 2] = v.z; kv[i + 3] = v.w;
      }
    }
#pragma unroll
    for (int h = 0; h < kHMax; ++h) {
      if (h < H) {
        const float* qh = qs + h * kC + blk * 32;
        float a = acc[h];
#pragma unroll
        for (int i = 0; i < 32; ++i) a = fmaf(qh[i], kv[i], a);
        acc[h] = a;
      }
    }
  }
  float score = 0.f;
#pragma unroll
  for (int h = 0; h < kHMax; ++h)
    if (h < H) score = fmaf(ws[h], fmaxf(acc[h], 0.f), score);
  scores[(int64_t)qi * n_max + s] = score;
}

// order-preserving key: larger score -> larger key; -0 and +0 map together
__device__ __forceinline__ uint32_t score_key(float f) {
  uint32_t u = __float_as_uint(f);
  if ((u & 0x7FFFFFFFu) == 0) u = 0;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// exclusive block scan of 0/1 flags for blockDim.x == 1024; returns the
// exclusive prefix and writes the block total to *total.
__device__ __forceinline__ int block_excl_scan(int flag, int* wsum, int* total) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const unsigned bal = __ballot_sync(0xffffffffu, flag);
  const int in_warp = __popc(bal & ((1u << lane) - 1u));
  if (lane == 0) wsum[wid] = __popc(bal);
  __syncthreads();
  if (wid == 0) {
    int v = wsum[lane];
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int n = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += n;
    }
    wsum[32 + lane] = incl - v;
    if (lane == 31) wsum[64] = incl;
  }
  __syncthreads();
  const int r = wsum[32 + wid] + in_warp;
  *total = wsum[64];
  __syncthreads();
  return r;
}

__global__ void __launch_bounds__(1024) topk_radix(const float* __restrict__ scores, int n_max,
                                                   const int32_t* __restrict__ q_pos0, int T, int m,
                                                   int k, int64_t k_cap, int32_t* __restrict__ out_idx) {
  __shared__ uint32_t hist[256];
  __shared__ int wsum[65];
  __shared__ uint32_t sh_sel[2];
  const int qi = blockIdx.x;
  const int bs = qi / T, tq = qi % T;
  const int64_t t = (int64_t)q_pos0[bs] + tq;
  int64_t n_t64 = (t + 1) / m;
  if (n_t64 > n_max) n_t64 = n_max;
  if (n_t64 > k_cap) n_t64 = k_cap;
  const int n_t = (int)n_t64;
  const float* sc = scores + (int64_t)qi * n_max;
  int32_t* out = out_idx + (int64_t)qi * k;
  if (n_t <= k) {
    for (int i = threadIdx.x; i < k; i += blockDim.x) out[i] = i < n_t ? i : -1;
    return;
  }
  uint32_t prefix = 0, mask = 0;
  int remaining = k;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = threadIdx.x; i < 256; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    for (int s = threadIdx.x; s < n_t; s += blockDim.x) {
      const uint32_t key = score_key(sc[s]);
      if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (threadIdx.x < 32) {
      // lane l covers bins 255-8l .. 248-8l (descending)
      const int lane = threadIdx.x;
      uint32_t c[8];
      uint32_t tot = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) { c[i] = hist[255 - 8 * lane - i]; tot += c[i]; }
      uint32_t incl = tot;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        uint32_t n = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += n;
      }
      const uint32_t before = incl - tot;  // count in higher bins
      if (before < (uint32_t)remaining && incl >= (uint32_t)remaining) {
        uint32_t acc = before;
        for (int i = 0; i < 8; ++i) {
          if (acc + c[i] >= (uint32_t)remaining) {
            sh_sel[0] = 255 - 8 * lane - i;
            sh_sel[1] = acc;
            break;
          }
          acc += c[i];
        }
      }
    }
    __syncthreads();
    const uint32_t bin = sh_sel[0];
    remaining -= (int)sh_sel[1];
    prefix |= bin << shift;
    mask |= 255u << shift;
    __syncthreads();
  }
  // prefix = key of the k-th largest score; `remaining` entries equal to it
  // are taken, the lowest indices first.
  const uint32_t thr = prefix;
  const int need_eq = remaining;
  int eq_base = 0, sel_base = 0;
  for (int s0 = 0; s0 < n_t; s0 += blockDim.x) {
    const int s = s0 + threadIdx.x;
    uint32_t key = 0;
    if (s < n_t) key = score_key(sc[s]);
    const int gt = (s < n_t) && key > thr;
    const int eq = (s < n_t) && key == thr;
    int eq_tot, sel_tot;
    const int eq_rank = eq_base + block_excl_scan(eq, wsum, &eq_tot);
    const int sel = gt || (eq && eq_rank < need_eq);
    const int pos = sel_base + block_excl_scan(sel, wsum, &sel_tot);
    if (sel) out[pos] = s;
    eq_base += eq_tot;
    sel_base += sel_tot;
  }
}

cudaError_t launch_index_scores(const csa_params& p, const void* q_idx, const uint8_t* q_sf,
                                const float* w, const void* k_idx, const uint8_t* k_sf,
                                int64_t k_cap, const int32_t* q_pos0, int T, float* scores,
                                int n_max, int32_t* err, cudaStream_t st) {
  dim3 grid(p.B * T, (n_max + 255) / 256);
  const bool mx = p.idx_fmt == CSA_IDX_MXFP4;
  if (p.n_idx_heads <= 8 && p.idx_dim == 64) {
    if (mx) index_scores_simt<8, 64, true><<<grid, 256, 0, st>>>(p, q_idx, q_sf, w, k_idx, k_sf, k_cap, q_pos0, T, scores, n_max, err);
    else index_scores_simt<8, 64, false><<<grid, 256, 0, st>>>(p, q_idx, q_sf, w, k_idx, k_sf, k_cap, q_pos0, T, scores, n_max, err);
  } else if (p.n_idx_heads <= 8 && p.idx_dim == 128) {
    if (mx) index_scores_simt<8, 128, true><<<grid, 256, 0, st>>>(p, q_idx, q_sf, w, k_idx, k_sf, k_cap, q_pos0, T, scores, n_max, err);
    else index_scores_simt<8, 128, false><<<grid, 256, 0, st>>>(p, q_idx, q_sf, w, k_idx, k_sf, k_cap, q_pos0, T, scores, n_max, err);
  } else if (p.idx_dim == 64) {
    if (mx) index_scores_simt<64, 64, true><<<grid, 256, 0, st>>>(p, q_idx, q_sf, w, k_idx, k_sf, k_cap, q_pos0, T, scores, n_max, err);
    else index_scores_simt<64, 64, false><<<grid, 256, 0, st>>>(p, q_idx, q_sf, w, k_idx, k_sf, k_cap, q_pos0, T, scores, n_max, err);
  } else {
    if (mx) index_scores_simt<64, 128, true><<<grid, 256, 0, st>>>(p, q_idx, q_sf, w, k_idx, k_sf, k_cap, q_pos0, T, scores, n_max, err);
    else index_scores_simt<64, 128, false><<<grid, 256, 0, st>>>(p, q_idx, q_sf, w, k_idx, k_sf, k_cap, q_pos0, T, scores, n_max, err);
  }
  return cudaGetLastError();
}

cudaError_t launch_topk(const csa_params& p, const float* scores, int n_max, const int32_t* q_pos0,
                        int T, int64_t k_cap, int32_t* out_idx, cudaStream_t st) {
  topk_radix<<<p.B * T, 1024, 0, st>>>(scores, n_max, q_pos0, T, p.m, p.topk, k_cap, out_idx);
  return cudaGetLastError();
}

}  // namespace csa
