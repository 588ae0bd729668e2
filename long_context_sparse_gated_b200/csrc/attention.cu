// Sparse (CSA) and dense (HCA) MQA with sliding window, attention sink and
// inverse RoPE -- CUDA-core reference path.
//
// WeChat 未来科技 1.1 (MQA; a learnable sink logit lets a head push its total
// attention towards 0; inverse RoPE on the core-attention output's RoPE
// dims); kwkr.cn notes 3.3 (window of the 128 most recent raw tokens joins
// the core attention; the sink is an extra denominator term);
// fengweifeng.com notes 2. (the KV entry serves as both key and value).
//
// A query's candidate slots are [0, n_sel) for entries (CSA: idx list,
// HCA: entry = slot) followed by W window slots.  Slots are cut into
// fixed-size splits (size chosen from T, never from B, so a query's bits do
// not depend on the batch it is in); one CTA handles one (query, split,
// head group), runs an online softmax over 32-row tiles and either writes
// the final output (single split) or an unnormalised partial (O, max,
// sum) that attn_merge combines in split order.
#include "common.cuh"
#include "kernels.h"

namespace csa {

constexpr int kTileRows = 32;
constexpr int kHeadGroup = 32;

struct Rows {
  const uint8_t* rows;
  const float* scale;
  int64_t cap;
};

template <bool kKvF32>
__device__ __forceinline__ float load_elem(const Rows& R, int64_t row, int c, int d, int r) {
  if (kKvF32) return reinterpret_cast<const float*>(R.rows)[row * d + c];
  const uint8_t* rp = R.rows + row * (int64_t)(d + r);
  if (c < d - r) return e4m3_to_f32(rp[c]) * R.scale[row];
  const uint16_t* rb = reinterpret_cast<const uint16_t*>(rp + (d - r));
  return bf16_bits_to_f32(rb[c - (d - r)]);
}

template <bool kKvF32, bool kActF32, bool kDense>
__global__ void __launch_bounds__(256) attn_split_simt(
    const csa_params p, const void* __restrict__ q, Rows cache, const int32_t* __restrict__ idx,
    Rows win, const float* __restrict__ sink, const int32_t* __restrict__ q_pos0, int T, int n_sel,
    int rows_per_split, int n_splits, void* __restrict__ out, float* __restrict__ ws_o,
    float* __restrict__ ws_ml, int32_t* __restrict__ err) {
  extern __shared__ float sm[];
  const int d = p.d, r = p.r, W = p.window;
  const int nth = blockDim.x;  // == d/2
  const int qi = blockIdx.x, split = blockIdx.y, hg = blockIdx.z;
  const int bs = qi / T, tq = qi % T;
  const int64_t t = (int64_t)q_pos0[bs] + tq;
  const int64_t n_t = (t + 1) / p.m;
  const int h0 = hg * kHeadGroup;
  const int nh = min(kHeadGroup, p.n_heads - h0);
  // this query's own slots (CSA: the k selected entries; HCA: its n_t
  // visible ones), then its window; a query with one split is finalised
  // here, one with several writes partials for attn_merge
  const int own_sel = kDense ? (int)min((int64_t)n_sel, n_t) : n_sel;
  const int total = own_sel + W;
  const int own_splits = (total + rows_per_split - 1) / rows_per_split;
  if (split >= own_splits) return;
  const int sb = split * rows_per_split;
  const int se = min(total, sb + rows_per_split);

  const int ldv = d + 1, ldq = d + 4, lds = kTileRows + 1;
  float* Vs = sm;                              // [R][d+1]
  float* Qs = Vs + kTileRows * ldv;            // [HG][d+4]
  float* Ss = Qs + kHeadGroup * ldq;           // [HG][R+1]
  float* Mh = Ss + kHeadGroup * lds;           // [HG]
  float* Lh = Mh + kHeadGroup;                 // [HG]
  float* Ah = Lh + kHeadGroup;                 // [HG]
  int* rsrc = reinterpret_cast<int*>(Ah + kHeadGroup);          // [R] 0 none, 1 cache, 2 window
  int64_t* rrow = reinterpret_cast<int64_t*>(rsrc + kTileRows); // [R]

  // queries of this head group, as float
  for (int i = threadIdx.x; i < nh * d; i += nth) {
    const int h = i / d, c = i % d;
    const int64_t off = ((int64_t)qi * p.n_heads + h0 + h) * d + c;
    Qs[h * ldq + c] = kActF32 ? reinterpret_cast<const float*>(q)[off]
                              : bf16_bits_to_f32(reinterpret_cast<const uint16_t*>(q)[off]);
  }
  if (threadIdx.x < kHeadGroup) {
    Mh[threadIdx.x] = -INFINITY;
    Lh[threadIdx.x] = 0.f;
  }
  const int c0 = threadIdx.x, c1 = threadIdx.x + nth;
  float o0[kHeadGroup], o1[kHeadGroup];
#pragma unroll
  for (int h = 0; h < kHeadGroup; ++h) o0[h] = o1[h] = 0.f;

  for (int tb = sb; tb < se; tb += kTileRows) {
    if (threadIdx.x < kTileRows) {
      const int slot = tb + threadIdx.x;
      int src = 0;
      int64_t row = 0;
      if (slot < se) {
        if (slot < own_sel) {
          if (kDense) {
            if (slot < n_t && slot < cache.cap) { src = 1; row = slot; }
          } else {
            const int e = idx[(int64_t)qi * p.topk + slot];
            if (e >= 0 && e < n_t && e < cache.cap) {
              src = 1; row = e;
            } else if (e != -1) {
              raise_err(err, CSA_DEV_ERR_INDEX);
            }
          }
        } else {
          const int64_t pos = t - W + 1 + (slot - own_sel);
          if (pos >= 0) { src = 2; row = pos % win.cap; }
        }
      }
      rsrc[threadIdx.x] = src;
      rrow[threadIdx.x] = (int64_t)bs * (src == 2 ? win.cap : cache.cap) + row;
    }
    __syncthreads();
    for (int i = threadIdx.x; i < kTileRows * d; i += nth) {
      const int j = i / d, c = i % d;
      const int src = rsrc[j];
      float v = 0.f;
      if (src == 1) v = load_elem<kKvF32>(cache, rrow[j], c, d, r);
      else if (src == 2) v = load_elem<kKvF32>(win, rrow[j], c, d, r);
      Vs[j * ldv + c] = v;
    }
    __syncthreads();
    for (int pr = threadIdx.x; pr < nh * kTileRows; pr += nth) {
      const int h = pr / kTileRows, j = pr % kTileRows;
      float z = -INFINITY;
      if (rsrc[j]) {
        const float* qh = Qs + h * ldq;
        const float* vj = Vs + j * ldv;
        float acc = 0.f;
        for (int c = 0; c < d; ++c) acc = fmaf(qh[c], vj[c], acc);
        z = p.softmax_scale * acc;
      }
      Ss[h * lds + j] = z;
    }
    __syncthreads();
    if (threadIdx.x < nh) {
      const int h = threadIdx.x;
      float mx = Mh[h];
      for (int j = 0; j < kTileRows; ++j) mx = fmaxf(mx, Ss[h * lds + j]);
      float alpha, sum = 0.f;
      if (mx == -INFINITY) {
        alpha = 1.f;
        for (int j = 0; j < kTileRows; ++j) Ss[h * lds + j] = 0.f;
      } else {
        alpha = expf(Mh[h] - mx);
        for (int j = 0; j < kTileRows; ++j) {
          const float e = expf(Ss[h * lds + j] - mx);
          Ss[h * lds + j] = e;
          sum += e;
        }
      }
      Lh[h] = Lh[h] * alpha + sum;
      Mh[h] = mx;
      Ah[h] = alpha;
    }
    __syncthreads();
#pragma unroll
    for (int h = 0; h < kHeadGroup; ++h) {
      if (h < nh) { o0[h] *= Ah[h]; o1[h] *= Ah[h]; }
    }
    for (int j = 0; j < kTileRows; ++j) {
      const float v0 = Vs[j * ldv + c0], v1 = Vs[j * ldv + c1];
#pragma unroll
      for (int h = 0; h < kHeadGroup; ++h) {
        if (h < nh) {
          const float pj = Ss[h * lds + j];
          o0[h] = fmaf(pj, v0, o0[h]);
          o1[h] = fmaf(pj, v1, o1[h]);
        }
      }
    }
    __syncthreads();
  }

  if (own_splits > 1) {
    const int64_t base = ((int64_t)qi * n_splits + split) * p.n_heads + h0;
#pragma unroll
    for (int h = 0; h < kHeadGroup; ++h) {
      if (h < nh) {
        ws_o[(base + h) * d + c0] = o0[h];
        ws_o[(base + h) * d + c1] = o1[h];
      }
    }
    if (threadIdx.x < nh) {
      ws_ml[(base + threadIdx.x) * 2 + 0] = Mh[threadIdx.x];
      ws_ml[(base + threadIdx.x) * 2 + 1] = Lh[threadIdx.x];
    }
    return;
  }
  // single split: finalise here (sink, normalisation, inverse RoPE)
  // rotation of dim c (in pair j) needs the partner dim c^1, owned by lane^1
  float cs0 = 1.f, sn0 = 0.f, cs1 = 1.f, sn1 = 0.f;
  if (c0 >= d - r) rope_cos_sin(-(double)t, (c0 - (d - r)) >> 1, r, (double)p.rope_theta, &cs0, &sn0);
  if (c1 >= d - r) rope_cos_sin(-(double)t, (c1 - (d - r)) >> 1, r, (double)p.rope_theta, &cs1, &sn1);
  const bool odd = threadIdx.x & 1;
#pragma unroll
  for (int h = 0; h < kHeadGroup; ++h) {
    if (h < nh) {
      const float sg = sink[h0 + h];
      const float M = Mh[h];
      const float Ms = fmaxf(sg, M);
      const float den = expf(sg - Ms) + (M == -INFINITY ? 0.f : Lh[h] * expf(M - Ms));
      const float f = (den > 0.f && M != -INFINITY) ? expf(M - Ms) / den : 0.f;
      float y0 = o0[h] * f, y1 = o1[h] * f;
      const float p0 = __shfl_xor_sync(0xffffffffu, y0, 1), p1 = __shfl_xor_sync(0xffffffffu, y1, 1);
      // pair (x, y) -> (x c - y s, x s + y c) with angle -t*freq (c, s of -t)
      if (c0 >= d - r) y0 = odd ? (p0 * sn0 + y0 * cs0) : (y0 * cs0 - p0 * sn0);
      if (c1 >= d - r) y1 = odd ? (p1 * sn1 + y1 * cs1) : (y1 * cs1 - p1 * sn1);
      const int64_t off = ((int64_t)qi * p.n_heads + h0 + h) * d;
      if (kActF32) {
        reinterpret_cast<float*>(out)[off + c0] = y0;
        reinterpret_cast<float*>(out)[off + c1] = y1;
      } else {
        reinterpret_cast<uint16_t*>(out)[off + c0] = f32_to_bf16_bits(y0);
        reinterpret_cast<uint16_t*>(out)[off + c1] = f32_to_bf16_bits(y1);
      }
    }
  }
}

// Combine the splits of one (query, head) in split order, add the sink,
// normalise and apply the inverse RoPE.  grid (queries, n_h), d/2 threads.
template <bool kActF32>
__global__ void __launch_bounds__(256) attn_merge(const csa_params p, const float* __restrict__ ws_o,
                                                  const float* __restrict__ ws_ml, int n_splits,
                                                  const float* __restrict__ sink,
                                                  const int32_t* __restrict__ q_pos0, int T, int n_sel,
                                                  int dense, int rows_per_split, void* __restrict__ out) {
  const int d = p.d, r = p.r, nth = blockDim.x;
  const int qi = blockIdx.x, h = blockIdx.y;
  const int bs = qi / T, tq = qi % T;
  const int64_t t = (int64_t)q_pos0[bs] + tq;
  // the query's own split count; n_splits is only the workspace stride
  const int own_sel = dense ? (int)min((int64_t)n_sel, (t + 1) / p.m) : n_sel;
  const int own_splits = (own_sel + p.window + rows_per_split - 1) / rows_per_split;
  if (own_splits <= 1) return;  // finalised by the split kernel
  const float sg = sink[h];
  float Ms = sg;
  for (int s = 0; s < own_splits; ++s)
    Ms = fmaxf(Ms, ws_ml[(((int64_t)qi * n_splits + s) * p.n_heads + h) * 2]);
  float den = (Ms == -INFINITY) ? 0.f : expf(sg - Ms);
  const int c0 = threadIdx.x, c1 = threadIdx.x + nth;
  float y0 = 0.f, y1 = 0.f;
  for (int s = 0; s < own_splits; ++s) {
    const int64_t base = ((int64_t)qi * n_splits + s) * p.n_heads + h;
    const float M = ws_ml[base * 2], L = ws_ml[base * 2 + 1];
    if (M == -INFINITY) continue;
    const float f = expf(M - Ms);
    den += L * f;
    y0 = fmaf(ws_o[base * d + c0], f, y0);
    y1 = fmaf(ws_o[base * d + c1], f, y1);
  }
  const float inv = den > 0.f ? 1.f / den : 0.f;
  y0 *= inv;
  y1 *= inv;
  float cs0 = 1.f, sn0 = 0.f, cs1 = 1.f, sn1 = 0.f;
  if (c0 >= d - r) rope_cos_sin(-(double)t, (c0 - (d - r)) >> 1, r, (double)p.rope_theta, &cs0, &sn0);
  if (c1 >= d - r) rope_cos_sin(-(double)t, (c1 - (d - r)) >> 1, r, (double)p.rope_theta, &cs1, &sn1);
  const bool odd = threadIdx.x & 1;
  const float p0 = __shfl_xor_sync(0xffffffffu, y0, 1), p1 = __shfl_xor_sync(0xffffffffu, y1, 1);
  if (c0 >= d - r) y0 = odd ? (p0 * sn0 + y0 * cs0) : (y0 * cs0 - p0 * sn0);
  if (c1 >= d - r) y1 = odd ? (p1 * sn1 + y1 * cs1) : (y1 * cs1 - p1 * sn1);
  const int64_t off = ((int64_t)qi * p.n_heads + h) * d;
  if (kActF32) {
    reinterpret_cast<float*>(out)[off + c0] = y0;
    reinterpret_cast<float*>(out)[off + c1] = y1;
  } else {
    reinterpret_cast<uint16_t*>(out)[off + c0] = f32_to_bf16_bits(y0);
    reinterpret_cast<uint16_t*>(out)[off + c1] = f32_to_bf16_bits(y1);
  }
}

size_t attn_smem_bytes(int d) {
  return (size_t)(kTileRows * (d + 1) + kHeadGroup * (d + 4) + kHeadGroup * (kTileRows + 1) + 3 * kHeadGroup) *
             sizeof(float) +
         kTileRows * (sizeof(int) + sizeof(int64_t));
}

int attn_rows_per_split(int total_slots, int T) {
  // decode-sized batches of queries split their slots; prefill does not
  if (T <= 4) return 128;
  return ((total_slots + kTileRows - 1) / kTileRows) * kTileRows;
}

template <bool kKvF32, bool kActF32, bool kDense>
static cudaError_t launch_attn_t(const csa_params& p, const void* q, const csa_kv& cache,
                                 const int32_t* idx, const csa_kv& win, const float* sink,
                                 const int32_t* q_pos0, int T, int n_sel, void* out, float* ws,
                                 int32_t* err, cudaStream_t st) {
  const int total = n_sel + p.window;
  const int rps = attn_rows_per_split(total, T);
  const int n_splits = (total + rps - 1) / rps;
  const int nhg = (p.n_heads + kHeadGroup - 1) / kHeadGroup;
  const size_t smem = attn_smem_bytes(p.d);
  auto kfn = attn_split_simt<kKvF32, kActF32, kDense>;
  cudaError_t e = set_max_smem(reinterpret_cast<const void*>(kfn), smem);
  if (e != cudaSuccess) return e;
  Rows rc{reinterpret_cast<const uint8_t*>(cache.rows), cache.scale, cache.cap};
  Rows rw{reinterpret_cast<const uint8_t*>(win.rows), win.scale, win.cap};
  float* ws_o = ws;
  float* ws_ml = ws ? ws + (size_t)p.B * T * n_splits * p.n_heads * p.d : nullptr;
  dim3 grid(p.B * T, n_splits, nhg);
  kfn<<<grid, p.d / 2, smem, st>>>(p, q, rc, idx, rw, sink, q_pos0, T, n_sel, rps, n_splits, out, ws_o, ws_ml, err);
  e = cudaGetLastError();
  if (e != cudaSuccess || n_splits == 1) return e;
  return launch_attn_merge(p, ws_o, ws_ml, n_splits, sink, q_pos0, T, n_sel, kDense, rps, out, st);
}

cudaError_t launch_attn_merge(const csa_params& p, const float* ws_o, const float* ws_ml, int n_splits,
                              const float* sink, const int32_t* q_pos0, int T, int n_sel, bool dense,
                              int rows_per_split, void* out, cudaStream_t st) {
  if (p.act_fmt == CSA_ACT_F32)
    attn_merge<true><<<dim3(p.B * T, p.n_heads), p.d / 2, 0, st>>>(p, ws_o, ws_ml, n_splits, sink, q_pos0, T, n_sel,
                                                                   dense ? 1 : 0, rows_per_split, out);
  else
    attn_merge<false><<<dim3(p.B * T, p.n_heads), p.d / 2, 0, st>>>(p, ws_o, ws_ml, n_splits, sink, q_pos0, T, n_sel,
                                                                    dense ? 1 : 0, rows_per_split, out);
  return cudaGetLastError();
}

// The tensor-core kernel serves the FP8/BF16 layout at d = 512 with whole
// 64-head groups; every other shape and format runs on CUDA cores.
static bool use_tc(const csa_params& p) { return attn_tc_supported(p); }

static size_t attn_simt_workspace_bytes(const csa_params& p, int T, int n_sel) {
  const int total = n_sel + p.window;
  const int rps = attn_rows_per_split(total, T);
  const int n_splits = (total + rps - 1) / rps;
  if (n_splits == 1) return 0;
  return (size_t)p.B * T * n_splits * p.n_heads * (p.d + 2) * sizeof(float);
}

size_t attn_workspace_bytes(const csa_params& p, int T, int n_sel, bool dense) {
  if (use_tc(p)) return attn_tc_workspace_bytes(p, T, n_sel, dense);
  return attn_simt_workspace_bytes(p, T, n_sel);
}

cudaError_t launch_attn(const csa_params& p, const void* q, const csa_kv& cache, const int32_t* idx,
                        const csa_kv& win, const float* sink, const int32_t* q_pos0, int T,
                        int n_sel, bool dense, void* out, float* ws, int32_t* err,
                        cudaStream_t st) {
  if (use_tc(p)) return launch_attn_tc(p, q, cache, idx, win, sink, q_pos0, T, n_sel, dense, out, ws, err, st);
  const bool kv32 = p.kv_fmt == CSA_KV_F32, a32 = p.act_fmt == CSA_ACT_F32;
#define CSA_ATTN_CASE(K, A, D) \
  if (kv32 == K && a32 == A && dense == D) \
    return launch_attn_t<K, A, D>(p, q, cache, idx, win, sink, q_pos0, T, n_sel, out, ws, err, st);
  CSA_ATTN_CASE(true, true, true)
  CSA_ATTN_CASE(true, true, false)
  CSA_ATTN_CASE(true, false, true)
  CSA_ATTN_CASE(true, false, false)
  CSA_ATTN_CASE(false, true, true)
  CSA_ATTN_CASE(false, true, false)
  CSA_ATTN_CASE(false, false, true)
  CSA_ATTN_CASE(false, false, false)
#undef CSA_ATTN_CASE
  return cudaErrorInvalidValue;
}

}  // namespace csa
