// Lightning Indexer scores, CUDA-core path.
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
// Selection lives in topk.cu.
#include "common.cuh"
#include "kernels.h"

namespace csa {

template <int kHMax, int kC, bool kMx>
__global__ void __launch_bounds__(256) index_scores_simt(
    const csa_params p, const void* __restrict__ q_idx, const uint8_t* __restrict__ q_sf,
    const float* __restrict__ w, const void* __restrict__ k_idx, const uint8_t* __restrict__ k_sf,
    int64_t k_cap, const int32_t* __restrict__ q_pos0, int T, void* __restrict__ scores,
    int ld, int n_max, int32_t* __restrict__ err) {
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
  if (p.score_fmt == CSA_SCORE_BF16)
    reinterpret_cast<uint16_t*>(scores)[(int64_t)qi * ld + s] = f32_to_bf16_bits(score);
  else
    reinterpret_cast<float*>(scores)[(int64_t)qi * ld + s] = score;
}

cudaError_t launch_index_scores(const csa_params& p, const void* q_idx, const uint8_t* q_sf,
                                const float* w, const void* k_idx, const uint8_t* k_sf,
                                int64_t k_cap, const int32_t* q_pos0, int T, void* scores,
                                int ld, int n_max, int32_t* err, cudaStream_t st) {
  dim3 grid(p.B * T, (n_max + 255) / 256);
  const bool mx = p.idx_fmt == CSA_IDX_MXFP4;
  if (p.n_idx_heads <= 8 && p.idx_dim == 64) {
    if (mx) index_scores_simt<8, 64, true><<<grid, 256, 0, st>>>(p, q_idx, q_sf, w, k_idx, k_sf, k_cap, q_pos0, T, scores, ld, n_max, err);
    else index_scores_simt<8, 64, false><<<grid, 256, 0, st>>>(p, q_idx, q_sf, w, k_idx, k_sf, k_cap, q_pos0, T, scores, ld, n_max, err);
  } else if (p.n_idx_heads <= 8 && p.idx_dim == 128) {
    if (mx) index_scores_simt<8, 128, true><<<grid, 256, 0, st>>>(p, q_idx, q_sf, w, k_idx, k_sf, k_cap, q_pos0, T, scores, ld, n_max, err);
    else index_scores_simt<8, 128, false><<<grid, 256, 0, st>>>(p, q_idx, q_sf, w, k_idx, k_sf, k_cap, q_pos0, T, scores, ld, n_max, err);
  } else if (p.idx_dim == 64) {
    if (mx) index_scores_simt<64, 64, true><<<grid, 256, 0, st>>>(p, q_idx, q_sf, w, k_idx, k_sf, k_cap, q_pos0, T, scores, ld, n_max, err);
    else index_scores_simt<64, 64, false><<<grid, 256, 0, st>>>(p, q_idx, q_sf, w, k_idx, k_sf, k_cap, q_pos0, T, scores, ld, n_max, err);
  } else {
    if (mx) index_scores_simt<64, 128, true><<<grid, 256, 0, st>>>(p, q_idx, q_sf, w, k_idx, k_sf, k_cap, q_pos0, T, scores, ld, n_max, err);
    else index_scores_simt<64, 128, false><<<grid, 256, 0, st>>>(p, q_idx, q_sf, w, k_idx, k_sf, k_cap, q_pos0, T, scores, ld, n_max, err);
  }
  return cudaGetLastError();
}

}  // namespace csa
