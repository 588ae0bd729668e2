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
//   3. an 8-bit radix select over the candidates' keys (warp-aggregated
//      shared-memory histograms; 3 passes over the low 20 bits when the
//      histogram fixed the top 12, else 4) finds the k-th largest key thr
//      and how many entries equal to thr are taken (the lowest indices).
//   4. an ordered compaction of the candidates (one contiguous run per
//      thread, two block scans) writes the k entries, already ascending.
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

// exclusive scan of one uint64 per thread (four 16-bit counters packed, no
// carries between them) over the 1024-thread block.  `tmp` holds >= 33
// uint64.
__device__ __forceinline__ uint64_t block_scan_excl64(uint64_t v, uint64_t* tmp, uint64_t* total) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  uint64_t incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint64_t n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += n;
  }
  if (lane == 31) tmp[wid] = incl;
  __syncthreads();
  if (wid == 0) {
    const uint64_t w = tmp[lane];
    uint64_t wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint64_t n = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += n;
    }
    tmp[lane] = wi - w;
    if (lane == 31) tmp[32] = wi;
  }
  __syncthreads();
  const uint64_t r = tmp[wid] + incl - v;
  *total = tmp[32];
  __syncthreads();
  return r;
}

// Radix select over n keys held by `get(i)` whose bits above `top_bit` all
// equal those of `prefix0` (mask0 marks the known bits): the key of the
// k-th largest (1 <= k <= n) and how many keys equal to it are among the
// top k.  Passes take 8 bits, the last one the remainder.
template <class Get>
__device__ void radix_select(int n, int k, Get get, uint32_t prefix0, uint32_t mask0, int top_bit,
                             uint32_t* hist, uint32_t* sel, uint32_t* thr_out, int* need_out) {
  uint32_t prefix = prefix0, mask = mask0;
  int remaining = k;
  for (int hi = top_bit; hi >= 0; hi -= 8) {
    const int width = hi >= 7 ? 8 : hi + 1;
    const int shift = hi + 1 - width;
    const uint32_t dmask = (1u << width) - 1u;
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
      hist_add(hist, (key >> shift) & dmask, act);
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
    mask |= dmask << shift;
    remaining -= (int)sel[1];
  }
  *thr_out = prefix;
  *need_out = remaining;
}

struct TopkSmem;

// The bin b* holding the k-th largest key, the count of entries in higher
// bins (all selected) and of entries in bins >= b* (the candidates), from a
// 4096-bin histogram of the keys' top 12 bits.  All threads must call.
template <class Sm>
__device__ void threshold_bin(const uint32_t* h, int k, Sm& S, int* bstar, int* cgt, int* ncand) {
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
        S.cgt = acc;
        S.ncand = acc + (int)c[i];
        break;
      }
      acc += (int)c[i];
    }
  }
  __syncthreads();
  *bstar = S.bstar;
  *cgt = S.cgt;
  *ncand = S.ncand;
  __syncthreads();
}

// Ordered collection of one 32768-entry chunk [base, base+32768) of a score
// row: every entry whose key's top 12 bits are >= bstar is appended, in
// index order, as (index, key) to cidx/ckey.  Loads are coalesced: load i
// (of 8) of thread t covers entries base + 4t + 4096 i .. +3; each thread's
// 8 candidate counts are packed into two uint64 (four 16-bit fields each),
// so two block scans give every load its position.  Returns the count.
template <class Sm>
__device__ int collect_chunk(const float* sc, int n_t, int base, int bstar, Sm& S, int* cidx, uint32_t* ckey) {
  uint32_t keys[8][4];
  uint64_t c01 = 0, c23 = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int s0 = base + 4 * threadIdx.x + 4096 * i;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (s0 < n_t) v = *reinterpret_cast<const float4*>(sc + s0);
    const float f[4] = {v.x, v.y, v.z, v.w};
    uint64_t cnt = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const uint32_t key = score_key(f[e]);
      const bool ok = (s0 + e < n_t) && (int)(key >> 20) >= bstar;
      keys[i][e] = ok ? key : 0u;  // 0 marks a non-candidate (only -NaN maps to 0)
      cnt += ok;
    }
    if (i < 4) c01 |= cnt << (16 * i);
    else c23 |= cnt << (16 * (i - 4));
  }
  uint64_t t01, t23;
  const uint64_t p01 = block_scan_excl64(c01, S.tmp64, &t01);
  const uint64_t p23 = block_scan_excl64(c23, S.tmp64, &t23);
  int lbase = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint64_t pf = i < 4 ? p01 : p23, tf = i < 4 ? t01 : t23;
    const int sh = 16 * (i & 3);
    int pos = lbase + (int)((pf >> sh) & 0xFFFFu);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if (keys[i][e]) {
        cidx[pos] = base + 4 * threadIdx.x + 4096 * i + e;
        ckey[pos] = keys[i][e];
        ++pos;
      }
    }
    lbase += (int)((tf >> sh) & 0xFFFFu);
  }
  return lbase;
}

struct TopkSmem {
  int cidx[kCap];
  uint32_t ckey[kCap];
  uint32_t hist[4096];
  int tmp[40];
  uint64_t tmp64[40];
  uint32_t sel[2];
  int bstar, cgt, ncand;
};

__global__ void __launch_bounds__(kThreads, 1) topk_select(const float* __restrict__ scores, int ld, int n_max,
                                                            const uint32_t* __restrict__ ghist,
                                                            const int32_t* __restrict__ q_pos0, int T, int m,
                                                            int k, int32_t* __restrict__ out_idx,
                                                            const int* __restrict__ cidx_g,
                                                            const uint32_t* __restrict__ ckey_g,
                                                            const int* __restrict__ ccount, int n_chunks) {
  extern __shared__ uint8_t smem_raw[];
  TopkSmem& S = *reinterpret_cast<TopkSmem*>(smem_raw);
  pdl_wait();
  pdl_trigger();
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
  int bstar = 0, cgt = 0, cand_total = n_t;
  if (ghist) threshold_bin(ghist + (int64_t)qi * 4096, k, S, &bstar, &cgt, &cand_total);
  bool fits = cand_total <= kCap;
  if (fits && ccount && ccount[(int64_t)qi * n_chunks] < 0) fits = false;
  if (fits) {
    // 2. ordered candidate collection (or the chunk lists a collect pass
    //    already wrote, concatenated in chunk order)
    int base_out = 0;
    if (ccount) {
      for (int c = 0; c < n_chunks; ++c) {
        const int cnt = ccount[(int64_t)qi * n_chunks + c];
        const int64_t off = ((int64_t)qi * n_chunks + c) * kCap;
        for (int i = threadIdx.x; i < cnt; i += kThreads) {
          S.cidx[base_out + i] = cidx_g[off + i];
          S.ckey[base_out + i] = ckey_g[off + i];
        }
        base_out += cnt;
      }
    } else {
      for (int base = 0; base < n_t; base += kChunk)
        base_out += collect_chunk(sc, n_t, base, bstar, S, S.cidx + base_out, S.ckey + base_out);
    }
    __syncthreads();
    const int nc = base_out;
    // 3. exact k-th largest: with a histogram the top 12 bits of the k-th
    //    key are bstar, so only bits 19..0 remain (3 passes); without one,
    //    all 32 bits (4 passes)
    uint32_t thr;
    int need;
    if (ghist)
      radix_select(nc, k - cgt, [&](int i) { return S.ckey[i]; }, (uint32_t)bstar << 20, 0xFFF00000u, 19, S.hist,
                   S.sel, &thr, &need);
    else
      radix_select(nc, k, [&](int i) { return S.ckey[i]; }, 0u, 0u, 31, S.hist, S.sel, &thr, &need);
    // keys above thr are all kept; keys == thr take `need` slots, lowest
    // index first.  Every thread owns a contiguous run of candidates, so
    // two block scans place the run's equal keys and its outputs in order.
    const int per = (nc + kThreads - 1) / kThreads;
    const int r0 = min(nc, threadIdx.x * per), r1 = min(nc, r0 + per);
    int n_eq = 0;
    for (int i = r0; i < r1; ++i) n_eq += S.ckey[i] == thr;
    int tot;
    int eq_rank = block_scan_excl(n_eq, S.tmp, &tot);
    int n_sel = 0;
    {
      int er = eq_rank;
      for (int i = r0; i < r1; ++i) {
        const uint32_t key = S.ckey[i];
        if (key > thr) ++n_sel;
        else if (key == thr) n_sel += (er++ < need);
      }
    }
    int pos = block_scan_excl(n_sel, S.tmp, &tot);
    for (int i = r0; i < r1; ++i) {
      const uint32_t key = S.ckey[i];
      bool take = key > thr;
      if (key == thr) take = eq_rank++ < need;
      if (take) out[pos++] = S.cidx[i];
    }
    return;
  }
  // fallback: radix select straight from global memory
  uint32_t thr;
  int need;
  radix_select(n_t, k, [&](int i) { return score_key(sc[i]); }, 0u, 0u, 31, S.hist, S.sel, &thr, &need);
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


// Multi-CTA candidate pass for long score rows: CTA (query, chunk) appends
// its chunk's candidates (bins >= b*) in index order to the chunk's slot of
// the scratch lists; topk_select then concatenates the slots in order.
__global__ void __launch_bounds__(kThreads, 1) topk_collect(const float* __restrict__ scores, int ld, int n_max,
                                                             const uint32_t* __restrict__ ghist,
                                                             const int32_t* __restrict__ q_pos0, int T, int m,
                                                             int k, int* __restrict__ cidx_g,
                                                             uint32_t* __restrict__ ckey_g, int* __restrict__ ccount,
                                                             int n_chunks) {
  extern __shared__ uint8_t smem_raw[];
  TopkSmem& S = *reinterpret_cast<TopkSmem*>(smem_raw);
  pdl_wait();
  pdl_trigger();
  const int qi = blockIdx.x, chunk = blockIdx.y;
  const int bs = qi / T, tq = qi % T;
  const int64_t t = (int64_t)q_pos0[bs] + tq;
  int64_t n64 = (t + 1) / m;
  if (n64 > n_max) n64 = n_max;
  const int n_t = (int)n64;
  const int64_t slot = (int64_t)qi * n_chunks + chunk;
  if (n_t <= k || chunk * kChunk >= n_t) {
    if (threadIdx.x == 0) ccount[slot] = 0;
    return;
  }
  int bstar, cgt, ncand;
  threshold_bin(ghist + (int64_t)qi * 4096, k, S, &bstar, &cgt, &ncand);
  if (ncand > kCap) {  // the selector falls back to a global radix select
    if (threadIdx.x == 0) ccount[slot] = -1;
    return;
  }
  // chunk lists are collected in shared memory, then copied out
  const int n = collect_chunk(scores + (int64_t)qi * ld, n_t, chunk * kChunk, bstar, S, S.cidx, S.ckey);
  __syncthreads();
  const int64_t off = slot * kCap;
  for (int i = threadIdx.x; i < n; i += kThreads) {
    cidx_g[off + i] = S.cidx[i];
    ckey_g[off + i] = S.ckey[i];
  }
  if (threadIdx.x == 0) ccount[slot] = n;
}

}  // namespace

size_t topk_hist_bytes(int queries) { return (size_t)queries * 4096 * sizeof(uint32_t); }

bool topk_use_hist(int queries) { return queries <= 4096; }

int topk_scores_ld(int n_max) { return (n_max + 31) & ~31; }

// Chunked candidate lists for long rows (histogram mode, n_max > 32768):
// [queries][chunks][kCap] indices and keys, then [queries][chunks] counts.
int topk_chunks(int n_max) { return (n_max + kChunk - 1) / kChunk; }

size_t topk_cand_bytes(int queries, int n_max) {
  const int c = topk_chunks(n_max);
  if (c <= 1) return 0;
  return (size_t)queries * c * ((size_t)kCap * 8 + 4);
}

cudaError_t launch_topk_select(const csa_params& p, const float* scores, int ld, int n_max,
                               const uint32_t* hist, const int32_t* q_pos0, int T, int32_t* out_idx,
                               void* cand, cudaStream_t st) {
  const size_t smem = sizeof(TopkSmem);
  const int nq = p.B * T;
  const int chunks = topk_chunks(n_max);
  int* cidx = nullptr;
  uint32_t* ckey = nullptr;
  int* ccount = nullptr;
  if (hist && chunks > 1 && cand) {
    cidx = reinterpret_cast<int*>(cand);
    ckey = reinterpret_cast<uint32_t*>(cidx + (size_t)nq * chunks * kCap);
    ccount = reinterpret_cast<int*>(ckey + (size_t)nq * chunks * kCap);
    cudaError_t e = cudaFuncSetAttribute(topk_collect, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    e = launch_pdl(topk_collect, dim3(nq, chunks), dim3(kThreads), smem, st, scores, ld, n_max, hist, q_pos0, T,
                   p.m, p.topk, cidx, ckey, ccount, chunks);
    if (e != cudaSuccess) return e;
  }
  cudaError_t e = cudaFuncSetAttribute(topk_select, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(topk_select, dim3(nq), dim3(kThreads), smem, st, scores, ld, n_max, hist, q_pos0, T, p.m,
                    p.topk, out_idx, (const int*)cidx, (const uint32_t*)ckey, (const int*)ccount,
                    ccount ? chunks : 0);
}

}  // namespace csa
