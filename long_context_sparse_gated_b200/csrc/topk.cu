// Exact top-k selection of the Lightning Indexer scores.
//
// Qiaomu blog 混合注意力机制 and PACMAN notes 3.1: the selector keeps the
// index_topk (512 for V4-Flash, 1024 for V4-Pro) highest-scoring compressed
// entries of each query; ties go to the lower entry index, and the output
// lists the entries in ascending order, padded with -1.
//
// Scores become order-preserving 32-bit keys (larger score -> larger key,
// -0 == +0).  One CTA (1024 threads) per query:
//
//   1. threshold bin (histogram mode): the scoring kernel has counted every
//      key's top 12 bits into a 4096-bin per-query histogram; a reverse scan
//      finds the bin b* that holds the k-th largest key.  Without a
//      histogram every entry is a candidate.
//   2. one ordered pass over the scores copies every candidate (bin >= b*)
//      into shared memory as (index, key), in ascending index order; each
//      thread owns a contiguous run of 32 entries and one block-wide scan
//      places the runs.
//   3. an 8-bit radix select over the candidates' keys (4 passes, warp-
//      aggregated shared-memory histograms) finds the k-th largest key thr
//      and how many entries equal to thr are taken (the lowest indices).
//   4. an ordered compaction of the candidates writes the k entries,
//      already ascending.
// When the candidates do not fit in shared memory (heavy ties across a
// huge range), the CTA falls back to the same radix select read from global
// memory, then the same ordered compaction over all entries.
#include "common.cuh"
#include "kernels.h"

namespace csa {

namespace {

constexpr int kThreads = 1024;
constexpr int kPerThread = 32;
constexpr int kChunk = kThreads * kPerThread;  // 32768 entries per ordered pass
constexpr int kCap = 12288;                     // shared-memory candidates

// exclusive scan of one int per thread over the 1024-thread block; returns
// the prefix and writes the total to *total.  `tmp` holds >= 33 ints.
__device__ __forceinline__ int block_scan_excl(int v, int* tmp, int* total) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += n;
  }
  if (lane == 31) tmp[wid] = incl;
  __syncthreads();
  if (wid == 0) {
    const int w = tmp[lane];
    int wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += n;
    }
    tmp[lane] = wi - w;
    if (lane == 31) tmp[32] = wi;
  }
  __syncthreads();
  const int r = tmp[wid] + incl - v;
  *total = tmp[32];
  __syncthreads();
  return r;
}

// Radix select over n keys held by `get(i)`: the key of the k-th largest
// (1 <= k <= n) and how many keys equal to it are among the top k.
template <class Get>
__device__ void radix_select(int n, int k, Get get, uint32_t* hist, uint32_t* sel, uint32_t* thr_out,
                             int* need_out) {
  uint32_t prefix = 0, mask = 0;
  int remaining = k;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = threadIdx.x; i < 256; i += kThreads) hist[i] = 0;
    __syncthreads();
    for (int i0 = 0; i0 < n; i0 += kThreads) {
      const int i = i0 + threadIdx.x;
      uint32_t key = 0;
      bool act = false;
      if (i < n) {
        key = get(i);
        act = (key & mask) == prefix;
      }
      hist_add(hist, (key >> shift) & 255u, act);
    }
    __syncthreads();
    if (threadIdx.x < 32) {
      const int lane = threadIdx.x;
      uint32_t c[8], tot = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) { c[i] = hist[255 - 8 * lane - i]; tot += c[i]; }
      uint32_t incl = tot;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      const uint32_t before = incl - tot;
      if (before < (uint32_t)remaining && incl >= (uint32_t)remaining) {
        uint32_t acc = before;
        for (int i = 0; i < 8; ++i) {
          if (acc + c[i] >= (uint32_t)remaining) {
            sel[0] = 255 - 8 * lane - i;
            sel[1] = acc;
            break;
          }
          acc += c[i];
        }
      }
    }
    __syncthreads();
    prefix |= sel[0] << shift;
    mask |= 255u << shift;
    remaining -= (int)sel[1];
    __syncthreads();
  }
  *thr_out = prefix;
  *need_out = remaining;
}

struct TopkSmem {
  int cidx[kCap];
  uint32_t ckey[kCap];
  uint32_t hist[4096];
  int tmp[40];
  uint32_t sel[2];
  int bstar, cgt, ncand;
};

__global__ void __launch_bounds__(kThreads, 1) topk_select(const float* __restrict__ scores, int ld, int n_max,
                                                            const uint32_t* __restrict__ ghist,
                                                            const int32_t* __restrict__ q_pos0, int T, int m,
                                                            int k, int32_t* __restrict__ out_idx) {
  extern __shared__ uint8_t smem_raw[];
  TopkSmem& S = *reinterpret_cast<TopkSmem*>(smem_raw);
  const int qi = blockIdx.x;
  const int bs = qi / T, tq = qi % T;
  const int64_t t = (int64_t)q_pos0[bs] + tq;
  int64_t n64 = (t + 1) / m;
  if (n64 > n_max) n64 = n_max;
  const int n_t = (int)n64;
  const float* sc = scores + (int64_t)qi * ld;
  int32_t* out = out_idx + (int64_t)qi * k;
  if (n_t <= k) {
    for (int i = threadIdx.x; i < k; i += kThreads) out[i] = i < n_t ? i : -1;
    return;
  }
  // 1. threshold bin from the histogram (bins >= bstar are candidates)
  int bstar = 0, cand_total = n_t;
  if (ghist) {
    const uint32_t* h = ghist + (int64_t)qi * 4096;
    // thread t owns bins 4095-4t .. 4092-4t (descending)
    uint32_t c[4], tot = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) { c[i] = h[4095 - 4 * threadIdx.x - i]; tot += c[i]; }
    int total;
    const int above = block_scan_excl((int)tot, S.tmp, &total);  // count in higher bins
    if (above < k && above + (int)tot >= k) {
      int acc = above;
      for (int i = 0; i < 4; ++i) {
        if (acc + (int)c[i] >= k) {
          S.bstar = 4095 - 4 * threadIdx.x - i;
          S.ncand = acc + (int)c[i];
          break;
        }
        acc += (int)c[i];
      }
    }
    __syncthreads();
    bstar = S.bstar;
    cand_total = S.ncand;
  }
  const bool fits = cand_total <= kCap;
  if (fits) {
    // 2. ordered candidate collection
    int base_out = 0;
    for (int base = 0; base < n_t; base += kChunk) {
      const int s0 = base + threadIdx.x * kPerThread;
      uint32_t keys[kPerThread];
      int cnt = 0;
#pragma unroll
      for (int i = 0; i < kPerThread; i += 4) {
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (s0 + i < n_t) v = *reinterpret_cast<const float4*>(sc + s0 + i);
        const float f[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const uint32_t key = score_key(f[e]);
          const bool ok = (s0 + i + e < n_t) && (int)(key >> 20) >= bstar;
          keys[i + e] = ok ? key : 0u;
          cnt += ok;
        }
      }
      // keys[] == 0 marks a non-candidate: a real key is never 0 except for
      // -NaN bit patterns, which scores never take
      int total;
      int pos = base_out + block_scan_excl(cnt, S.tmp, &total);
#pragma unroll
      for (int i = 0; i < kPerThread; ++i) {
        if (keys[i]) {
          S.cidx[pos] = s0 + i;
          S.ckey[pos] = keys[i];
          ++pos;
        }
      }
      base_out += total;
    }
    __syncthreads();
    const int nc = base_out;
    // 3. exact k-th largest among the candidates
    uint32_t thr;
    int need;
    radix_select(nc, k, [&](int i) { return S.ckey[i]; }, S.hist, S.sel, &thr, &need);
    // 4. ordered compaction
    int eq_base = 0, sel_base = 0;
    for (int i0 = 0; i0 < nc; i0 += kThreads) {
      const int i = i0 + threadIdx.x;
      const uint32_t key = i < nc ? S.ckey[i] : 0u;
      const int eq = (i < nc) && key == thr;
      int tot_eq, tot_sel;
      const int r_eq = eq_base + block_scan_excl(eq, S.tmp, &tot_eq);
      const int sel = (i < nc) && (key > thr || (eq && r_eq < need));
      const int pos = sel_base + block_scan_excl(sel, S.tmp, &tot_sel);
      if (sel) out[pos] = S.cidx[i];
      eq_base += tot_eq;
      sel_base += tot_sel;
    }
    return;
  }
  // fallback: radix select straight from global memory
  uint32_t thr;
  int need;
  radix_select(n_t, k, [&](int i) { return score_key(sc[i]); }, S.hist, S.sel, &thr, &need);
  int eq_base = 0, sel_base = 0;
  for (int i0 = 0; i0 < n_t; i0 += kThreads) {
    const int i = i0 + threadIdx.x;
    const uint32_t key = i < n_t ? score_key(sc[i]) : 0u;
    const int eq = (i < n_t) && key == thr;
    int tot_eq, tot_sel;
    const int r_eq = eq_base + block_scan_excl(eq, S.tmp, &tot_eq);
    const int sel = (i < n_t) && (key > thr || (eq && r_eq < need));
    const int pos = sel_base + block_scan_excl(sel, S.tmp, &tot_sel);
    if (sel) out[pos] = i;
    eq_base += tot_eq;
    sel_base += tot_sel;
  }
}

}  // namespace

size_t topk_hist_bytes(int queries) { return (size_t)queries * 4096 * sizeof(uint32_t); }

bool topk_use_hist(int queries) { return queries <= 4096; }

int topk_scores_ld(int n_max) { return (n_max + 31) & ~31; }

cudaError_t launch_topk_select(const csa_params& p, const float* scores, int ld, int n_max,
                               const uint32_t* hist, const int32_t* q_pos0, int T, int32_t* out_idx,
                               cudaStream_t st) {
  const size_t smem = sizeof(TopkSmem);
  cudaError_t e = cudaFuncSetAttribute(topk_select, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  topk_select<<<p.B * T, kThreads, smem, st>>>(scores, ld, n_max, hist, q_pos0, T, p.m, p.topk, out_idx);
  return cudaGetLastError();
}

}  // namespace csa
