// Sparse (CSA) and dense (HCA) MQA on the 5th-generation tensor cores.
//
// WeChat 未来科技 1.1 (MQA over the selected entries; sink logit; inverse RoPE
// on the output's RoPE dims; RoPE dims BF16, the rest FP8); kwkr.cn notes
// 3.3 (128-token window and sink join the core attention); fengweifeng.com
// notes 2. (an entry serves as both key and value).
//
// One CTA = one query, one group of 64 heads, one split of its candidate
// slots (entries, then window tokens), in 128-row tiles:
//
//   gather    8 warps load the tile's 128 rows (16-byte loads of the
//             576-byte FP8/BF16 rows), convert them to FP16 and store them
//             as a 128-row x 512-dim K-major tile (128-byte swizzle).  E4M3
//             codes are exact in FP16; the RoPE dims are stored divided by
//             the row scale s_j, so that  s_j * (V'_j . q) = v_j . q  and one
//             accumulator holds a whole logit.  FP16 (10-bit mantissa) keeps
//             the rounding of P' and of the scaled RoPE dims 8x below BF16's.
//   S^T       tcgen05.mma kind::f16 (FP16 A/B, FP32 accumulate):
//             S^T[j, h] = sum_c V'[j, c] Q[h, c]
//             (M = 128 rows, N = 64 heads, K = 512) into TMEM
//   softmax   per row thread: z = tau * s_j * S^T; per-head tile maxima and
//             sums by warp-transposed shuffles; the running max is raised
//             lazily (only when a tile exceeds it by > 8), so O is rarely
//             rescaled; P'^T[h, j] = exp(z - m_h) * s_j in FP16 to smem
//   O^T       tcgen05.mma: O^T[c, h] += sum_j V'[j, c] P'[h, j]
//             (A = V'^T, the same tile read MN-major; M = 128 dims x 4
//             blocks, N = 64 heads, K = 128 rows) into TMEM
//   epilogue  normalise with the sink term, inverse RoPE, BF16 store -- or,
//             with several splits, write the partial O/l (FP16) and (m, l)
//             that attn_merge_f16 combines in split order.
//
// 8 warps (two per TMEM lane quadrant) gather, run the softmax and the
// epilogue; thread 0 also issues the query TMA and the MMAs between block
// barriers.  Every wait is bounded (CSA_DEV_ERR_TIMEOUT).
#include <cuda.h>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace csa {

namespace {

constexpr int kRows = 128;     // rows per tile (MMA M of S^T)
constexpr int kHg = 64;        // heads per CTA (MMA N)
constexpr int kD = 512;
constexpr int kR = 64;
constexpr int kNope = kD - kR;             // 448
constexpr int kRowBytes = kNope + 2 * kR;  // 576
constexpr int kChunks = kRowBytes / 16;    // 36 16-byte chunks per stored row
constexpr int kThreads = 256;             // 8 warps: two per TMEM lane quadrant
constexpr float kLazy = 8.0f;  // raise the running max only past +8 (e^8 < 3000)
constexpr uint32_t kTmemCols = 512;        // S^T: 64, O^T: 4 x 64

struct __align__(1024) AttnSmem {
  uint8_t v[8][kRows * 128];  // 8 K-chunks of 64 dims: [128 rows][128 B], 128B swizzle
  uint8_t q[8][kHg * 128];    // 8 K-chunks: [64 heads][128 B]
  uint8_t p[2][kHg * 128];    // P'^T: 2 K-chunks of 64 rows: [64 heads][128 B]
  float scale[kRows];
  float inv_scale[kRows];
  int64_t rowoff[kRows];      // byte offset of the row, -1 when the slot is empty
  int src[kRows];             // 1 cache, 2 window
  float red[8][64];
  float mh[kHg], lh[kHg], alpha[kHg];
  uint64_t bar_q, bar_s, bar_o;
  uint32_t tmem_base;
  int abort;
  int rescale;
};

__device__ __forceinline__ uint32_t sw128(int row, int chunk16) {
  return (uint32_t)(row * 128 + ((chunk16 ^ (row & 7)) << 4));
}

// 16 E4M3 codes -> 16 FP16 (exact), as two 16-byte words
__device__ __forceinline__ void e4m3x16_to_f16(const uint4& in, uint4& lo, uint4& hi) {
  const uint32_t w[4] = {in.x, in.y, in.z, in.w};
  uint32_t o[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const __nv_fp8x2_storage_t pr = (__nv_fp8x2_storage_t)((w[i] >> (16 * k)) & 0xFFFFu);
      const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(pr, __NV_E4M3);
      o[2 * i + k] = (uint32_t)h.x | ((uint32_t)h.y << 16);
    }
  }
  lo = make_uint4(o[0], o[1], o[2], o[3]);
  hi = make_uint4(o[4], o[5], o[6], o[7]);
}

// 8 BF16 values times s -> 8 FP16 (round to nearest)
__device__ __forceinline__ uint4 bf16x8_scale_to_f16(const uint4& in, float s) {
  const uint32_t w[4] = {in.x, in.y, in.z, in.w};
  uint32_t o[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const __half2 r = __floats2half2_rn(bf16_bits_to_f32(w[i]) * s, bf16_bits_to_f32(w[i] >> 16) * s);
    o[i] = *reinterpret_cast<const uint32_t*>(&r);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// 8 BF16 -> 8 FP16 (round to nearest; queries are RMS-normalised, far
// inside the FP16 range)
__device__ __forceinline__ uint4 bf16x8_to_f16(const uint4& in) {
  return bf16x8_scale_to_f16(in, 1.0f);
}

// max / sum over the 32 lanes of a warp for each of 32 values: afterwards
// lane l holds the reduction of value index l.
template <bool kMax>
__device__ __forceinline__ float warp_transpose_reduce32(float (&v)[32]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int s = 16; s >= 1; s >>= 1) {
    const bool up = lane & s;
#pragma unroll
    for (int i = 0; i < s; ++i) {
      const float keep = up ? v[i + s] : v[i];
      const float send = up ? v[i] : v[i + s];
      const float recv = __shfl_xor_sync(0xffffffffu, send, s);
      v[i] = kMax ? fmaxf(keep, recv) : keep + recv;
    }
  }
  return v[0];
}

template <bool kDense>
__global__ void __launch_bounds__(kThreads, 1) attn_tc(
    const __grid_constant__ CUtensorMap tm_q, const uint8_t* __restrict__ cache_rows,
    const float* __restrict__ cache_scale, int64_t cache_cap, const uint8_t* __restrict__ win_rows,
    const float* __restrict__ win_scale, int64_t win_cap, const int32_t* __restrict__ idx, int topk,
    const int32_t* __restrict__ q_pos0, int T, int m, int W, int n_sel, int n_heads, float tau,
    float theta, const float* __restrict__ sink, int rows_per_split, int n_splits, uint16_t* __restrict__ out,
    __half* __restrict__ ws_o, float* __restrict__ ws_ml, int32_t* __restrict__ err) {
  extern __shared__ uint8_t smem_raw[];
  AttnSmem& S = *reinterpret_cast<AttnSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int wt = threadIdx.x;                // 0..255
  const int quad = warp & 3;                 // TMEM lane quadrant of this warp
  const int half = warp >> 2;                // head half: 32*half .. +31
  const int j = quad * 32 + lane;            // tile row of this thread
  const int qi = blockIdx.x, split = blockIdx.y, hg = blockIdx.z;
  const int bs = qi / T, tq = qi % T;
  const int h0 = hg * kHg;
  const int total = n_sel + W;
  const int sb = split * rows_per_split;
  const int se = min(total, sb + rows_per_split);
  const int n_tiles = (se - sb + kRows - 1) / kRows;
  volatile int* abort = &S.abort;
  const bool issuer = threadIdx.x == 0;

  if (issuer) {
    sm100::mbar_init(&S.bar_q, 1);
    sm100::mbar_init(&S.bar_s, 1);
    sm100::mbar_init(&S.bar_o, 1);
    S.abort = 0;
    sm100::fence_mbar_init();
  }
  if (threadIdx.x < kHg) {
    S.mh[threadIdx.x] = -INFINITY;
    S.lh[threadIdx.x] = 0.f;
  }
  if (warp == 0) {
    sm100::tmem_alloc(&S.tmem_base, kTmemCols);
    sm100::tmem_relinquish();
  }
  sm100::tc_fence_before();
  __syncthreads();
  sm100::tc_fence_after();
  pdl_wait();  // inputs may come from the previous kernel on the stream
  const int64_t t = (int64_t)q_pos0[bs] + tq;
  const int64_t n_t = (t + 1) / m;
  const uint32_t tmem = S.tmem_base;
  const uint32_t s_col = tmem;         // S^T: 64 columns
  const uint32_t o_col = tmem + 64;    // O^T block b: columns 64 + 64 b
  if (issuer) {
    sm100::prefetch_tmap(&tm_q);
    sm100::mbar_arrive_expect_tx(&S.bar_q, 8 * kHg * 128);
    for (int c = 0; c < 8; ++c) sm100::tma_load_2d(S.q[c], &tm_q, &S.bar_q, 64 * c, qi * n_heads + h0);
  }
  const uint32_t idS = sm100::idesc_f16(kRows, kHg, 0, 0);
  const uint32_t idO = sm100::idesc_f16(128, kHg, 1, 0);

  // Control flow is uniform across the CTA (every __syncthreads is reached
  // by all threads); a failed bounded wait only raises the abort flag,
  // after which every later wait returns at once and no MMA is issued.
  for (int i = 0; i < n_tiles; ++i) {
    const int tb = sb + i * kRows;
    if (i > 0) sm100::mbar_wait(&S.bar_o, (i - 1) & 1, abort);  // V' and P' buffers free
    if (wt == 0) S.rescale = 0;
    // -- resolve the tile's rows
    if (wt < kRows) {
      const int slot = tb + wt;
      int src = 0;
      int64_t row = 0;
      if (slot < se) {
        if (slot < n_sel) {
          if (kDense) {
            if (slot < n_t && slot < cache_cap) { src = 1; row = slot; }
          } else {
            const int e = idx[(int64_t)qi * topk + slot];
            if (e >= 0 && e < n_t && e < cache_cap) { src = 1; row = e; }
            else if (e != -1) raise_err(err, CSA_DEV_ERR_INDEX);
          }
        } else {
          const int64_t pos = t - W + 1 + (slot - n_sel);
          if (pos >= 0) { src = 2; row = pos % win_cap; }
        }
      }
      float sc = 1.f;
      int64_t off = -1;
      if (src == 1) { off = ((int64_t)bs * cache_cap + row); sc = cache_scale[off]; }
      if (src == 2) { off = ((int64_t)bs * win_cap + row); sc = win_scale[off]; }
      if (!(sc > 0.f) || !(sc < INFINITY)) {  // scales are positive and finite by construction
        if (src) raise_err(err, CSA_DEV_ERR_RANGE);
        src = 0;
        off = -1;
        sc = 1.f;
      }
      S.src[wt] = src;
      S.rowoff[wt] = off < 0 ? -1 : off * kRowBytes;
      S.scale[wt] = sc;
      S.inv_scale[wt] = 1.f / sc;
    }
    __syncthreads();
    // -- gather + convert: 128 rows x 36 chunks of 16 B, 18 per thread in
    //    two batches of 9 loads in flight
#pragma unroll
    for (int bt = 0; bt < 2; ++bt) {
      uint4 raw[9];
#pragma unroll
      for (int k = 0; k < 9; ++k) {
        const int u = wt + kThreads * (9 * bt + k);
        const int r = u / kChunks, c = u % kChunks;
        const int64_t off = S.rowoff[r];
        const uint8_t* base = S.src[r] == 2 ? win_rows : cache_rows;
        raw[k] = off >= 0 ? __ldg(reinterpret_cast<const uint4*>(base + off) + c) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int k = 0; k < 9; ++k) {
        const int u = wt + kThreads * (9 * bt + k);
        const int r = u / kChunks, c = u % kChunks;
        if (c < kNope / 16) {
          // dims 16c .. 16c+15 -> K-chunk (16c)/64, 16-byte slots 2(c%4), 2(c%4)+1
          uint4 lo, hi;
          e4m3x16_to_f16(raw[k], lo, hi);
          uint8_t* ch = S.v[c >> 2];
          *reinterpret_cast<uint4*>(ch + sw128(r, 2 * (c & 3))) = lo;
          *reinterpret_cast<uint4*>(ch + sw128(r, 2 * (c & 3) + 1)) = hi;
        } else {
          // RoPE dims 448 + 8(c-28) .. : chunk 7, slot (c-28)
          const uint4 v = bf16x8_scale_to_f16(raw[k], S.inv_scale[r]);
          *reinterpret_cast<uint4*>(S.v[7] + sw128(r, c - kNope / 16)) = v;
        }
      }
    }
    if (i == 0) {
      // queries: BF16 (TMA) -> FP16 in place, same swizzled positions
      sm100::mbar_wait(&S.bar_q, 0, abort);
      uint4* qv = reinterpret_cast<uint4*>(&S.q[0][0]);
      for (int e = wt; e < 8 * kHg * 128 / 16; e += kThreads) qv[e] = bf16x8_to_f16(qv[e]);
    }
    sm100::fence_proxy_async_smem();
    __syncthreads();
    // -- S^T = V' Q^T over K = 512 (32 steps of 16)
    if (issuer) {
      const bool ok = !*abort;
      sm100::tc_fence_after();
      if (ok && !*abort) {
#pragma unroll 1
        for (int kk = 0; kk < 32; ++kk) {
          const int c = kk >> 2, o = (kk & 3) * 32;
          const uint64_t a = sm100::smem_desc(sm100::smem_u32(S.v[c]) + o, 16, 1024, 2);
          const uint64_t b = sm100::smem_desc(sm100::smem_u32(S.q[c]) + o, 16, 1024, 2);
          sm100::mma_f16(s_col, a, b, idS, kk > 0);
        }
        sm100::tc_commit(&S.bar_s);
      }
    }
    sm100::mbar_wait(&S.bar_s, i & 1, abort);
    sm100::tc_fence_after();
    // -- logits of this thread's row for its 32 heads
    float z[32];
    {
      uint32_t a[16], b[16];
      const uint32_t ta = s_col + ((uint32_t)(quad * 32) << 16) + 32 * half;
      sm100::tmem_ld_x16(ta, a);
      sm100::tmem_ld_x16(ta + 16, b);
      sm100::tmem_ld_wait();
      const bool valid = S.src[j] != 0;
      const float f = tau * S.scale[j];
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        z[c] = valid ? f * __uint_as_float(a[c]) : -INFINITY;
        z[16 + c] = valid ? f * __uint_as_float(b[c]) : -INFINITY;
      }
    }
    // per-head tile maxima
    {
      float v[32];
#pragma unroll
      for (int c = 0; c < 32; ++c) v[c] = z[c];
      S.red[warp][lane] = warp_transpose_reduce32<true>(v);  // head 32*half + lane, this warp's rows
    }
    __syncthreads();
    if (wt < kHg) {
      const int h = wt, hh = h >> 5, hl = h & 31;
      float tmax = -INFINITY;
      for (int q4 = 0; q4 < 4; ++q4) tmax = fmaxf(tmax, S.red[hh * 4 + q4][hl]);
      const float mo = S.mh[h];
      float al = 1.f;
      int resc = 0;
      if (i == 0) {
        S.mh[h] = tmax;
      } else if (tmax > mo + kLazy) {
        al = (mo == -INFINITY) ? 0.f : expf(mo - tmax);
        S.mh[h] = tmax;
        S.lh[h] *= al;
        resc = 1;
      }
      S.alpha[h] = al;
      const unsigned any = __ballot_sync(0xffffffffu, resc);
      if (lane == 0 && any) S.rescale = 1;
    }
    __syncthreads();
    // rare: rescale the O^T columns of heads whose running max moved
    if (i > 0 && S.rescale) {
#pragma unroll 1
      for (int blk = 0; blk < 4; ++blk) {
#pragma unroll
        for (int g = 0; g < 2; ++g) {
          uint32_t r16[16];
          const uint32_t ta = o_col + 64 * blk + ((uint32_t)(quad * 32) << 16) + 32 * half + 16 * g;
          sm100::tmem_ld_x16(ta, r16);
          sm100::tmem_ld_wait();
#pragma unroll
          for (int c = 0; c < 16; ++c)
            r16[c] = __float_as_uint(__uint_as_float(r16[c]) * S.alpha[32 * half + 16 * g + c]);
          sm100::tmem_st_x16(ta, r16);
        }
      }
      sm100::tmem_st_wait();
    }
    // probabilities, P'^T stores and per-head sums
    {
      const float sj = S.scale[j];
      float v[32];
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        const int h = 32 * half + c;
        const float mh = S.mh[h];
        const float pr = (mh == -INFINITY || z[c] == -INFINITY) ? 0.f : expf(z[c] - mh);
        v[c] = pr;
        // P'^T[h][j]: K-major, K-chunk j/64, row h, 16-byte slot ((j%64)/8)
        const __half pb = __float2half_rn(pr * sj);
        uint8_t* dst = S.p[j >> 6] + sw128(h, (j & 63) >> 3) + 2 * (j & 7);
        *reinterpret_cast<__half*>(dst) = pb;
      }
      S.red[warp][lane] = warp_transpose_reduce32<false>(v);
    }
    sm100::tc_fence_before();
    sm100::fence_proxy_async_smem();
    __syncthreads();
    if (wt < kHg) {
      const int h = wt, hh = h >> 5, hl = h & 31;
      float ts = 0.f;
      for (int q4 = 0; q4 < 4; ++q4) ts += S.red[hh * 4 + q4][hl];
      S.lh[h] += ts;
    }
    // -- O^T[blk] += V'^T[blk] P'^T over K = 128 rows (8 steps of 16)
    if (issuer) {
      sm100::tc_fence_after();
      if (!*abort) {
#pragma unroll 1
        for (int blk = 0; blk < 4; ++blk) {
#pragma unroll 1
          for (int kk = 0; kk < 8; ++kk) {
            const uint64_t a = sm100::smem_desc(sm100::smem_u32(S.v[2 * blk]) + kk * 2048, 16384, 1024, 2);
            const uint64_t b = sm100::smem_desc(sm100::smem_u32(S.p[kk >> 2]) + (kk & 3) * 32, 16, 1024, 2);
            sm100::mma_f16(o_col + 64 * blk, a, b, idO, (i > 0 || kk > 0) ? 1u : 0u);
          }
        }
        sm100::tc_commit(&S.bar_o);
      }
    }
  }

  pdl_trigger();
  // -- epilogue
  if (n_tiles > 0) sm100::mbar_wait(&S.bar_o, (n_tiles - 1) & 1, abort);
  sm100::tc_fence_after();
  __syncthreads();  // lh final; abort flag now uniform
  const bool ok = !S.abort;
  const bool single = n_splits == 1;
  if (ok && n_tiles > 0) {
    // single split: normalise with the sink term here; several splits: the
    // partial normalised by its own sum, as FP16, plus (max, sum)
    float f[32];
#pragma unroll
    for (int c = 0; c < 32; ++c) {
      const int h = 32 * half + c;
      const float mh = S.mh[h], lh = S.lh[h];
      if (single) {
        const float sg = sink[h0 + h];
        const float ms = fmaxf(sg, mh);
        const float den = expf(sg - ms) + (mh == -INFINITY ? 0.f : lh * expf(mh - ms));
        f[c] = (mh == -INFINITY || !(den > 0.f)) ? 0.f : expf(mh - ms) / den;
      } else {
        f[c] = lh > 0.f ? 1.f / lh : 0.f;
      }
    }
#pragma unroll 1
    for (int blk = 0; blk < 4; ++blk) {
      const int c_dim = 128 * blk + quad * 32 + lane;
      float cs = 1.f, sn = 0.f;
      if (single && c_dim >= kNope) rope_cos_sin(-(double)t, (c_dim - kNope) >> 1, kR, (double)theta, &cs, &sn);
      const bool odd = lane & 1;
#pragma unroll
      for (int g = 0; g < 2; ++g) {
        uint32_t r16[16];
        sm100::tmem_ld_x16(o_col + 64 * blk + ((uint32_t)(quad * 32) << 16) + 32 * half + 16 * g, r16);
        sm100::tmem_ld_wait();
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const int hl = 16 * g + c;
          const int h = 32 * half + hl;
          float y = __uint_as_float(r16[c]) * f[hl];
          if (single) {
            const float pv = __shfl_xor_sync(0xffffffffu, y, 1);
            if (c_dim >= kNope) y = odd ? (pv * sn + y * cs) : (y * cs - pv * sn);
            out[((int64_t)qi * n_heads + h0 + h) * kD + c_dim] = f32_to_bf16_bits(y);
          } else {
            ws_o[(((int64_t)qi * n_splits + split) * n_heads + h0 + h) * kD + c_dim] = __float2half_rn(y);
          }
        }
      }
    }
    if (!single && wt < kHg) {
      const int64_t base = ((int64_t)qi * n_splits + split) * n_heads + h0 + wt;
      ws_ml[base * 2 + 0] = S.mh[wt];
      ws_ml[base * 2 + 1] = S.lh[wt];
    }
  }

  sm100::tc_fence_before();
  __syncthreads();
  if (S.abort && threadIdx.x == 0) raise_err(err, CSA_DEV_ERR_TIMEOUT);
  if (warp == 0) {
    sm100::tc_fence_after();
    sm100::tmem_dealloc(tmem, kTmemCols);
  }
}

// Combine the FP16 split partials (each O_s / l_s) of one query: for head h,
// M = max(sink, m_s), w_s = l_s e^(m_s - M) / (e^(sink - M) + sum l_s
// e^(m_s - M)), o = sum_s w_s (O_s / l_s) in split order, then the inverse
// RoPE and a BF16 store.  grid (queries, n_heads / 8), 256 threads: warp =
// head, lane = 16 dims.
__global__ void __launch_bounds__(256) attn_merge_f16(const __half* __restrict__ ws_o, const float* __restrict__ ws_ml,
                                                      int n_splits, int n_heads, const float* __restrict__ sink,
                                                      const int32_t* __restrict__ q_pos0, int T, float theta,
                                                      uint16_t* __restrict__ out) {
  pdl_wait();
  const int qi = blockIdx.x;
  const int h = blockIdx.y * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  const int bs = qi / T, tq = qi % T;
  const int64_t t = (int64_t)q_pos0[bs] + tq;
  const float sg = sink[h];
  float M = sg;
  for (int sp = 0; sp < n_splits; ++sp) M = fmaxf(M, ws_ml[(((int64_t)qi * n_splits + sp) * n_heads + h) * 2]);
  float den = expf(sg - M);
  for (int sp = 0; sp < n_splits; ++sp) {
    const int64_t b2 = (((int64_t)qi * n_splits + sp) * n_heads + h) * 2;
    const float ms = ws_ml[b2];
    if (ms != -INFINITY) den += ws_ml[b2 + 1] * expf(ms - M);
  }
  const float inv = den > 0.f ? 1.f / den : 0.f;
  const int c0 = 16 * lane;
  float acc[16];
#pragma unroll
  for (int e = 0; e < 16; ++e) acc[e] = 0.f;
  for (int sp = 0; sp < n_splits; ++sp) {
    const int64_t b2 = (((int64_t)qi * n_splits + sp) * n_heads + h) * 2;
    const float ms = ws_ml[b2];
    if (ms == -INFINITY) continue;
    const float a = ws_ml[b2 + 1] * expf(ms - M) * inv;
    const uint4* src = reinterpret_cast<const uint4*>(ws_o + (((int64_t)qi * n_splits + sp) * n_heads + h) * kD + c0);
    const uint4 v0 = src[0], v1 = src[1];
    const __half2* h0 = reinterpret_cast<const __half2*>(&v0);
    const __half2* h1 = reinterpret_cast<const __half2*>(&v1);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f0 = __half22float2(h0[e]), f1 = __half22float2(h1[e]);
      acc[2 * e] = fmaf(a, f0.x, acc[2 * e]);
      acc[2 * e + 1] = fmaf(a, f0.y, acc[2 * e + 1]);
      acc[8 + 2 * e] = fmaf(a, f1.x, acc[8 + 2 * e]);
      acc[8 + 2 * e + 1] = fmaf(a, f1.y, acc[8 + 2 * e + 1]);
    }
  }
  if (c0 >= kNope) {
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      float cs, sn;
      rope_cos_sin(-(double)t, (c0 - kNope) / 2 + e, kR, (double)theta, &cs, &sn);
      const float x = acc[2 * e], y = acc[2 * e + 1];
      acc[2 * e] = x * cs - y * sn;
      acc[2 * e + 1] = x * sn + y * cs;
    }
  }
  uint32_t o[8];
#pragma unroll
  for (int e = 0; e < 8; ++e)
    o[e] = (uint32_t)f32_to_bf16_bits(acc[2 * e]) | ((uint32_t)f32_to_bf16_bits(acc[2 * e + 1]) << 16);
  uint4* dst = reinterpret_cast<uint4*>(out + ((int64_t)qi * n_heads + h) * kD + c0);
  dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
  dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
}

using EncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                              const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                              CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeFn encode_fn() {
  static EncodeFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeFn>(p);
  }
  return fn;
}

}  // namespace

bool attn_tc_supported(const csa_params& p) {
  return p.kv_fmt == CSA_KV_FP8_BF16 && p.act_fmt == CSA_ACT_BF16 && p.d == kD && p.r == kR &&
         p.n_heads % kHg == 0 && encode_fn() != nullptr;
}

int attn_tc_rows_per_split(int total_slots, int T, bool dense) {
  const int tiles = (total_slots + kRows - 1) / kRows;
  if (T > 4) return tiles * kRows;           // prefill: one split per query
  return (dense ? 8 : 1) * kRows;            // decode: fixed split sizes
}

size_t attn_tc_smem_bytes() { return sizeof(AttnSmem) + 1024; }

cudaError_t launch_attn_tc(const csa_params& p, const void* q, const csa_kv& cache, const int32_t* idx,
                           const csa_kv& win, const float* sink, const int32_t* q_pos0, int T, int n_sel,
                           bool dense, void* out, float* ws, int32_t* err, cudaStream_t st) {
  const int nq = p.B * T;
  CUtensorMap tq;
  {
    cuuint64_t dims[2] = {(cuuint64_t)kD, (cuuint64_t)nq * p.n_heads};
    cuuint64_t str[1] = {(cuuint64_t)kD * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)kHg};
    cuuint32_t es[2] = {1, 1};
    if (encode_fn()(&tq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(q), dims, str, box, es,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  const int total = n_sel + p.window;
  const int rps = attn_tc_rows_per_split(total, T, dense);
  const int n_splits = (total + rps - 1) / rps;
  const int nhg = p.n_heads / kHg;
  // workspace: FP16 partials O/l, then (max, sum) per (query, split, head)
  const size_t n_part = (size_t)nq * n_splits * p.n_heads;
  __half* ws_o = reinterpret_cast<__half*>(ws);
  float* ws_ml = ws ? reinterpret_cast<float*>(reinterpret_cast<char*>(ws) + ((n_part * p.d * 2 + 15) & ~(size_t)15))
                    : nullptr;
  const size_t smem = attn_tc_smem_bytes();
  auto kfn = dense ? attn_tc<true> : attn_tc<false>;
  cudaError_t e = cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(nq, n_splits, nhg);
  e = launch_pdl(kfn, grid, dim3(kThreads), smem, st, tq, reinterpret_cast<const uint8_t*>(cache.rows), cache.scale,
                 cache.cap, reinterpret_cast<const uint8_t*>(win.rows), win.scale, win.cap, idx, p.topk, q_pos0, T,
                 p.m, p.window, n_sel, p.n_heads, p.softmax_scale, p.rope_theta, sink, rps, n_splits,
                 reinterpret_cast<uint16_t*>(out), ws_o, ws_ml, err);
  if (e != cudaSuccess || n_splits == 1) return e;
  return launch_pdl(attn_merge_f16, dim3(nq, p.n_heads / 8), dim3(256), 0, st, (const __half*)ws_o,
                    (const float*)ws_ml, n_splits, p.n_heads, sink, q_pos0, T, p.rope_theta,
                    reinterpret_cast<uint16_t*>(out));
}

size_t attn_tc_workspace_bytes(const csa_params& p, int T, int n_sel, bool dense) {
  const int total = n_sel + p.window;
  const int rps = attn_tc_rows_per_split(total, T, dense);
  const int n_splits = (total + rps - 1) / rps;
  if (n_splits == 1) return 0;
  const size_t n_part = (size_t)p.B * T * n_splits * p.n_heads;
  return ((n_part * p.d * 2 + 15) & ~(size_t)15) + n_part * 2 * sizeof(float);
}

}  // namespace csa
