// Exact top-k selection of the Lightning Indexer scores.
//
// Qiaomu blog 混合注意力机制 and PACMAN notes 3.1: the selector keeps the
// index_topk (512 for V4-Flash, 1024 for V4-Pro) highest-scoring compressed
// entries of each query; ties go to the lower entry index, and the output
// lists the entries in ascending order, padded with -1.  kwkr.cn notes 4.4:
// the scores may be rounded from FP32 to BF16 before the selector (BF16
// scores select on 16-bit keys).
//
// Scores become order-preserving keys (larger score -> larger key, -0 ==
// +0): 32-bit for fp32 scores, 16-bit for BF16 scores.
//
// Histogram mode (the tensor-core scorer has counted every key's top 12
// bits into a 4096-bin per-query histogram):
//   1. threshold bin: a reverse scan of the histogram finds the bin b* that
//      holds the k-th largest key, how many keys lie above it (cgt, all
//      selected) and how many in it (nb, the ties of the first level);
//   2. one pass over the scores (coalesced 16-byte loads; warp ballots
//      re-packed into 32-entry words): every entry above b* sets its bit in
//      a selection bitmap; every entry in b* goes to a tie list and into a
//      second-level histogram of its next 8 key bits (the last 4 for BF16);
//   3. the second-level bin b2 holding the (k - cgt)-th tie: ties above it
//      are selected; ties in it are ranked by (key descending, index
//      ascending) -- pairwise for a handful, else by a radix select of the
//      exact threshold key and an index bitmap of the keys equal to it;
//   4. one block scan over the bitmap's popcounts writes the selected
//      indices in ascending order.
// Rows of up to 32768 entries run as one CTA per query (topk_fused, which
// copies the row's scores into shared memory while it runs step 1); longer
// rows run steps 1-2 as one CTA per 32768-entry chunk (topk_chunk_pass,
// bitmap and tie list in the workspace) and steps 1, 3, 4 as one CTA per
// query (topk_chunk_finish_s for rows up to 262144 entries, with the row's
// bitmap in shared memory; topk_chunk_finish beyond).  When the threshold
// bin holds more than kTieCap entries (heavy ties), the query falls back to
// a radix select read from global memory and an ordered compaction.
//
// Without a histogram (the CUDA-core scorer, or more than 4096 queries in
// a call: prefill), rows of up to kCap entries run as one 256-thread CTA
// each (topk_rows): the keys staged in shared memory, a radix select, an
// ordered compaction by warp slabs.  Longer rows use a 1024-thread CTA
// (topk_staged) and, beyond kCap, the global-memory fallback.
#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace csa {

namespace {

constexpr int kThreads = 1024;
constexpr int kPerThread = 32;
constexpr int kChunk = kThreads * kPerThread;  // 32768 entries per CTA pass
constexpr int kCap = 12288;                     // staged keys (no-histogram mode)
constexpr int kTieCap = 4096;                   // threshold-bin entries kept for steps 2-3
constexpr int kSub = 256;                       // second-level bins
constexpr int kSmallGroup = 64;                 // final tie groups ranked pairwise up to this size
constexpr int kEqWords = 8192;                  // index-bitmap window of equal keys (262144 entries)

// Keys of a score row: fp32 scores give 32-bit keys, BF16 scores 16-bit.
template <bool kB16>
struct ScoreKeys;

template <>
struct ScoreKeys<false> {
  static constexpr int kBits = 32;
  __device__ __forceinline__ static uint32_t key(const void* row, int s) {
    return score_key(reinterpret_cast<const float*>(row)[s]);
  }
  __device__ __forceinline__ static uint32_t bin(uint32_t key) { return key >> 20; }
  __device__ __forceinline__ static uint32_t sub(uint32_t key) { return (key >> 12) & 0xFFu; }
};

template <>
struct ScoreKeys<true> {
  static constexpr int kBits = 16;
  __device__ __forceinline__ static uint32_t key(const void* row, int s) {
    return score_key16(reinterpret_cast<const uint16_t*>(row)[s]);
  }
  __device__ __forceinline__ static uint32_t bin(uint32_t key) { return key >> 4; }
  __device__ __forceinline__ static uint32_t sub(uint32_t key) { return key & 0xFu; }
};

__device__ __forceinline__ int warp_sum_int(int v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

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

// In a 256-bin histogram h, the bin holding the `need`-th largest key
// (1 <= need <= total count) and the count in higher bins, written to
// out[0], out[1] by the one lane that finds them.  Warp 0 only.
__device__ __forceinline__ void find_bin256(const uint32_t* h, uint32_t need, uint32_t* out) {
  const int lane = threadIdx.x;
  uint32_t c[8], tot = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) { c[i] = h[255 - 8 * lane - i]; tot += c[i]; }
  uint32_t incl = tot;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  const uint32_t before = incl - tot;
  if (before < need && incl >= need) {
    uint32_t acc = before;
    for (int i = 0; i < 8; ++i) {
      if (acc + c[i] >= need) {
        out[0] = 255 - 8 * lane - i;
        out[1] = acc;
        break;
      }
      acc += c[i];
    }
  }
}

// Radix select over n keys held by `get(i)` (the top `kBits` bits): the
// key of the k-th largest (1 <= k <= n) and how many keys equal to it are
// among the top k.  Passes take 8 bits.
template <int kBits, class Get>
__device__ void radix_select(int n, int k, Get get, uint32_t* hist, uint32_t* sel, uint32_t* thr_out,
                             int* need_out) {
  uint32_t prefix = 0, mask = 0;
  int remaining = k;
  for (int shift = kBits - 8; shift >= 0; shift -= 8) {
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
      hist_add(hist, (key >> shift) & 0xFFu, act);
    }
    __syncthreads();
    if (threadIdx.x < 32) find_bin256(hist, (uint32_t)remaining, sel);
    __syncthreads();
    const uint32_t bsel = sel[0], asel = sel[1];
    __syncthreads();
    prefix |= bsel << shift;
    mask |= 0xFFu << shift;
    remaining -= (int)asel;
  }
  *thr_out = prefix;
  *need_out = remaining;
}

// The bin b* holding the k-th largest key, the count of entries in higher
// bins (all selected) and in bins >= b*, from a 4096-bin histogram of the
// keys' top 12 bits.  All threads must call.  *bstar < 0 when the
// histogram holds fewer than k keys (it then does not describe the scores,
// e.g. after the scorer gave up on a timed-out wait): callers fall back to
// the global-memory selection, which reads only the scores.
template <class Sm>
__device__ void threshold_bin(const uint32_t* h, int k, Sm& S, int* bstar, int* cgt, int* ncand) {
  if (threadIdx.x == 0) {
    S.bstar = -1;
    S.cgt = 0;
    S.ncand = 0;
  }
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

struct BitSmem {
  uint32_t bits[kThreads];  // selection bitmap of a 32768-entry chunk
  int tidx[kTieCap];        // threshold-bin entries: index and key
  uint32_t tkey[kTieCap];
  int grp[kTieCap];         // tie-list positions of the second-level bin b2
  uint32_t eq[kEqWords];    // entries whose key equals the final threshold (by index), one window
  uint32_t h2[kSub];        // second-level histogram (also the radix histogram)
  uint32_t sel[2];
  int tmp[40];
  int tie_count, grp_count;
  int bstar, cgt, ncand;
};

// topk_fused stages its row's scores after BitSmem (32768 fp32 scores at most).
constexpr size_t kRowStageOff = (sizeof(BitSmem) + 127) & ~size_t(127);

// Global-memory fallback for a row (heavy ties): radix select over the
// keys, then an ordered compaction, 1024 entries per step.
template <bool kB16>
__device__ void select_full(const void* row, int n_t, int k, int32_t* out, BitSmem& S) {
  uint32_t thr;
  int need;
  radix_select<ScoreKeys<kB16>::kBits>(n_t, k, [&](int i) { return ScoreKeys<kB16>::key(row, i); }, S.h2, S.sel,
                                       &thr, &need);
  int eq_base = 0, sel_base = 0;
  for (int i0 = 0; i0 < n_t; i0 += kThreads) {
    const int i = i0 + threadIdx.x;
    const uint32_t key = i < n_t ? ScoreKeys<kB16>::key(row, i) : 0u;
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

__device__ __forceinline__ int visible_entries(const int32_t* q_pos0, int T, int m, int qi, int n_max) {
  const int bs = qi / T, tq = qi % T;
  const int64_t t = (int64_t)q_pos0[bs] + tq;
  int64_t n64 = (t + 1) / m;
  if (n64 > n_max) n64 = n_max;
  return (int)n64;
}

// Bit j of the low 8 bits of x moved to bit 4j (j < 8), and bit j of the
// low 4 bits to bit 8j (j < 4).
__device__ __forceinline__ uint32_t spread4(uint32_t x) {
  x &= 0xFFu;
  x = (x | (x << 12)) & 0x000F000Fu;
  x = (x | (x << 6)) & 0x03030303u;
  x = (x | (x << 3)) & 0x11111111u;
  return x;
}
__device__ __forceinline__ uint32_t spread8(uint32_t x) {
  x &= 0xFu;
  x = (x | (x << 14)) & 0x00030003u;
  x = (x | (x << 7)) & 0x01010101u;
  return x;
}

// Step 2 over one 32768-entry chunk [base, base + 32768) of a score row, by
// the whole CTA with coalesced 16-byte loads: fp32 rows in 8 passes of 4096
// entries (lane l of warp w takes entries 4l..4l+3 of the warp's 128), BF16
// rows in 4 passes of 8192 (8 entries per lane, 256 per warp).  Keys above
// b* become bits of the selection bitmap: a warp's ballots, one per entry
// slot of a lane, are re-packed into 32-entry words (words[j] for entries
// base + 32j .. +31, written when j < n_words).  The threshold bin's
// entries are appended to the tie list (warp-aggregated slots from *count;
// slots past kTieCap are not written, and the caller then falls back) and
// counted into the second-level histogram.
template <bool kB16>
__device__ __forceinline__ void scan_chunk(const void* row, int base, int n_t, int bstar, uint32_t* words, int n_words,
                                           int* count, int* tidx, uint32_t* tkey, uint32_t* h2) {
  constexpr int kPer = kB16 ? 8 : 4;        // entries per lane per pass
  constexpr int kPasses = 32 / kPer;        // passes per chunk
  constexpr int kWarpSpan = 32 * kPer;      // entries per warp per pass
  constexpr int kPassSpan = kThreads * kPer;
  const int lane = threadIdx.x & 31, wp = threadIdx.x >> 5;
  uint32_t tie = 0;  // bit kPer*i + e: entry (pass i, slot e) is in the threshold bin
#pragma unroll
  for (int i = 0; i < kPasses; ++i) {
    const int s = base + kPassSpan * i + kWarpSpan * wp + kPer * lane;
    uint32_t k[kPer];
    if (s < n_t) {
      if (kB16) {
        const uint4 v = *reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(row) + s);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          k[2 * j] = score_key16(w[j]);
          k[2 * j + 1] = score_key16(w[j] >> 16);
        }
      } else {
        const float4 v = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(row) + s);
        k[0] = score_key(v.x);
        k[1] = score_key(v.y);
        k[2] = score_key(v.z);
        k[3] = score_key(v.w);
      }
    } else {
#pragma unroll
      for (int e = 0; e < kPer; ++e) k[e] = 0u;
    }
    uint32_t word = 0;
#pragma unroll
    for (int e = 0; e < kPer; ++e) {
      const bool in = s + e < n_t;
      const uint32_t b = ScoreKeys<kB16>::bin(k[e]);
      tie |= (uint32_t)(in && b == (uint32_t)bstar) << (kPer * i + e);
      const uint32_t m = __ballot_sync(0xffffffffu, in && b > (uint32_t)bstar);
      // word q of this warp's span: lanes (32/kPer) q .. +32/kPer-1, slot e
      word |= (kB16 ? spread8(m >> (4 * (lane & 7))) : spread4(m >> (8 * (lane & 3)))) << e;
    }
    const int j = (kPassSpan * i + kWarpSpan * wp) / 32 + lane;  // valid for lane < kPer
    if (lane < kPer && j < n_words) words[j] = word;
  }
  const int nt = __popc(tie);
  int incl = nt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  int pos = 0;
  if (lane == 31 && incl) pos = atomicAdd(count, incl);
  pos = __shfl_sync(0xffffffffu, pos, 31) + incl - nt;
  while (tie) {
    const int bit = __ffs(tie) - 1;
    tie &= tie - 1;
    const int i = bit / kPer, e = bit % kPer;
    const int idx = base + kPassSpan * i + kWarpSpan * wp + kPer * lane + e;
    const uint32_t key = ScoreKeys<kB16>::key(row, idx);  // re-read: ties are few, the line is cached
    if (pos < kTieCap) {
      tidx[pos] = idx;
      tkey[pos] = key;
    }
    atomicAdd(h2 + ScoreKeys<kB16>::sub(key), 1u);
    ++pos;
  }
}

// Step 3: given the tie list in shared memory (S.tidx/S.tkey, nb entries)
// and the second-level histogram, mark the ties that are selected via
// mark(index).  `need` >= 1 ties are to be taken from a row of n_t entries.
// The second-level bin b2 holding the need-th tie splits them: ties above
// b2 are taken, ties in it form the final group.  A small group is ranked
// pairwise by (key descending, index ascending).  A larger one (many equal
// scores) gets a radix select of its exact threshold key; keys above it are
// taken, and keys equal to it are flagged in an index bitmap whose prefix
// popcounts rank them by index, lowest first.
template <bool kB16, class Mark>
__device__ void resolve_ties(int nb, int need, int n_t, BitSmem& S, Mark mark) {
  if (threadIdx.x < 32) find_bin256(S.h2, (uint32_t)need, S.sel);
  if (threadIdx.x == 0) S.grp_count = 0;
  __syncthreads();
  const uint32_t b2 = S.sel[0];
  const int need2 = need - (int)S.sel[1];
  for (int c = threadIdx.x; c < nb; c += kThreads) {
    const uint32_t sb = ScoreKeys<kB16>::sub(S.tkey[c]);
    if (sb > b2) mark(S.tidx[c]);
    else if (sb == b2) S.grp[atomicAdd(&S.grp_count, 1)] = c;
  }
  __syncthreads();
  const int n2 = S.grp_count;
  if (n2 <= kSmallGroup) {
    if ((int)threadIdx.x < n2) {
      const int c = S.grp[threadIdx.x];
      const uint32_t kc = S.tkey[c];
      const int ic = S.tidx[c];
      int rank = 0;
      for (int h = 0; h < n2; ++h) {
        const int c2 = S.grp[h];
        const uint32_t k2 = S.tkey[c2];
        rank += (k2 > kc) || (k2 == kc && S.tidx[c2] < ic);
      }
      if (rank < need2) mark(ic);
    }
    __syncthreads();
    return;
  }
  uint32_t thr;
  int need_eq;
  radix_select<ScoreKeys<kB16>::kBits>(n2, need2, [&](int i) { return S.tkey[S.grp[i]]; }, S.h2, S.sel, &thr,
                                       &need_eq);
  for (int g = threadIdx.x; g < n2; g += kThreads)
    if (S.tkey[S.grp[g]] > thr) mark(S.tidx[S.grp[g]]);
  // equal keys: the need_eq lowest indices, window by window of the row
  const int n_words = (n_t + 31) / 32;
  int taken = 0;
  for (int w0 = 0; w0 < n_words && taken < need_eq; w0 += kEqWords) {
    for (int j = threadIdx.x; j < kEqWords; j += kThreads) S.eq[j] = 0u;
    __syncthreads();
    for (int g = threadIdx.x; g < n2; g += kThreads) {
      const int c = S.grp[g];
      const int w = (S.tidx[c] >> 5) - w0;
      if (S.tkey[c] == thr && w >= 0 && w < kEqWords) atomicOr(&S.eq[w], 1u << (S.tidx[c] & 31));
    }
    __syncthreads();
    constexpr int kPer = kEqWords / kThreads;  // words per thread, in index order
    int cnt = 0;
#pragma unroll
    for (int j = 0; j < kPer; ++j) cnt += __popc(S.eq[kPer * threadIdx.x + j]);
    int tot;
    int rank = taken + block_scan_excl(cnt, S.tmp, &tot);
#pragma unroll 1
    for (int j = 0; j < kPer && rank < need_eq; ++j) {
      uint32_t word = S.eq[kPer * threadIdx.x + j];
      while (word && rank < need_eq) {
        const int e = __ffs(word) - 1;
        word &= word - 1;
        mark(32 * (w0 + kPer * (int)threadIdx.x + j) + e);
        ++rank;
      }
    }
    taken += tot;
    __syncthreads();
  }
  __syncthreads();
}

template <bool kB16>
__device__ __forceinline__ const void* score_row(const void* scores, int64_t qi, int ld) {
  return reinterpret_cast<const uint8_t*>(scores) + qi * ld * (kB16 ? 2 : 4);
}

// Histogram mode, rows of up to 32768 entries: one CTA per query.
template <bool kB16>
__global__ void __launch_bounds__(kThreads, 1) topk_fused(const void* __restrict__ scores, int ld, int n_max,
                                                           const uint32_t* __restrict__ ghist,
                                                           const int32_t* __restrict__ q_pos0, int T, int m, int k,
                                                           int32_t* __restrict__ out_idx) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  BitSmem& S = *reinterpret_cast<BitSmem*>(smem_raw);
  // the row's scores, copied into shared memory while the threshold bin is found
  uint8_t* srow = smem_raw + kRowStageOff;
  __shared__ uint64_t rbar;
  __shared__ int rabort;
  pdl_wait();
  pdl_trigger();
  const int qi = blockIdx.x;
  const int n_t = visible_entries(q_pos0, T, m, qi, n_max);
  const void* row = score_row<kB16>(scores, qi, ld);
  int32_t* out = out_idx + (int64_t)qi * k;
  if (n_t <= k) {
    for (int i = threadIdx.x; i < k; i += kThreads) out[i] = i < n_t ? i : -1;
    return;
  }
  const uint32_t row_bytes = ((uint32_t)n_t * (kB16 ? 2u : 4u) + 15u) & ~15u;  // within the row's ld padding
  if (threadIdx.x == 0) {
    sm100::mbar_init(&rbar, 1);
    rabort = 0;
    sm100::fence_mbar_init();
  }
  if (threadIdx.x < kSub) S.h2[threadIdx.x] = 0u;
  if (threadIdx.x == 0) S.tie_count = 0;
  __syncthreads();
  if (threadIdx.x == 0) {
    sm100::mbar_arrive_expect_tx(&rbar, row_bytes);
    sm100::bulk_load(srow, row, row_bytes, &rbar);
  }
  int bstar, cgt, ncand;
  threshold_bin(ghist + (int64_t)qi * kScoreHistBins, k, S, &bstar, &cgt, &ncand);
  const int nb = ncand - cgt;
  // scores from shared memory once they have landed (from global memory if
  // the copy timed out)
  const bool staged = sm100::mbar_wait(&rbar, 0, &rabort);
  if (!staged && threadIdx.x == 0) {
    volatile int again = 0;  // the copy must not outlive the CTA: one more bounded wait
    sm100::mbar_wait(&rbar, 0, &again);
  }
  const void* src = __syncthreads_and(staged) ? (const void*)srow : row;
  if (bstar < 0 || nb > kTieCap) {
    select_full<kB16>(row, n_t, k, out, S);
    return;
  }
  scan_chunk<kB16>(src, 0, n_t, bstar, S.bits, kThreads, &S.tie_count, S.tidx, S.tkey, S.h2);
  __syncthreads();
  if (S.tie_count != nb) {  // the histogram does not describe these scores
    select_full<kB16>(row, n_t, k, out, S);
    return;
  }
  resolve_ties<kB16>(nb, k - cgt, n_t, S, [&](int i) { atomicOr(&S.bits[i >> 5], 1u << (i & 31)); });
  uint32_t word = S.bits[threadIdx.x];
  int tot;
  int pos = block_scan_excl(__popc(word), S.tmp, &tot);
  while (word) {
    const int e = __ffs(word) - 1;
    word &= word - 1;
    out[pos++] = kPerThread * threadIdx.x + e;
  }
}

// Histogram mode, longer rows, step 1-2 per 32768-entry chunk: bitmap words
// and tie list (with its count and second-level histogram) in the workspace.
template <bool kB16>
__global__ void __launch_bounds__(kThreads, 1) topk_chunk_pass(const void* __restrict__ scores, int ld, int n_max,
                                                                const uint32_t* __restrict__ ghist,
                                                                const int32_t* __restrict__ q_pos0, int T, int m,
                                                                int k, uint32_t* __restrict__ gbits,
                                                                int* __restrict__ gtidx, uint32_t* __restrict__ gtkey,
                                                                int* __restrict__ gcount, uint32_t* __restrict__ gh2) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  BitSmem& S = *reinterpret_cast<BitSmem*>(smem_raw);
  pdl_wait();
  pdl_trigger();
  const int qi = blockIdx.x, chunk = blockIdx.y;
  const int n_t = visible_entries(q_pos0, T, m, qi, n_max);
  const int base = chunk * kChunk;
  if (n_t <= k || base >= n_t) return;
  int bstar, cgt, ncand;
  threshold_bin(ghist + (int64_t)qi * kScoreHistBins, k, S, &bstar, &cgt, &ncand);
  if (bstar < 0 || ncand - cgt > kTieCap) return;  // topk_chunk_finish falls back
  // the chunk's bitmap words, up to the row's last word
  const int n_words = min(kThreads, (n_t + 31) / 32 - base / 32);
  scan_chunk<kB16>(score_row<kB16>(scores, qi, ld), base, n_t, bstar, gbits + (int64_t)qi * (ld / 32) + base / 32,
                   n_words, gcount + qi, gtidx + (int64_t)qi * kTieCap, gtkey + (int64_t)qi * kTieCap,
                   gh2 + (int64_t)qi * kSub);
}

// Histogram mode, longer rows, steps 3-4 per query.
template <bool kB16>
__global__ void __launch_bounds__(kThreads, 1) topk_chunk_finish(const void* __restrict__ scores, int ld, int n_max,
                                                                  const uint32_t* __restrict__ ghist,
                                                                  const int32_t* __restrict__ q_pos0, int T, int m,
                                                                  int k, int32_t* __restrict__ out_idx,
                                                                  uint32_t* __restrict__ gbits,
                                                                  const int* __restrict__ gtidx,
                                                                  const uint32_t* __restrict__ gtkey,
                                                                  const int* __restrict__ gcount,
                                                                  const uint32_t* __restrict__ gh2) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  BitSmem& S = *reinterpret_cast<BitSmem*>(smem_raw);
  pdl_wait();
  pdl_trigger();
  const int qi = blockIdx.x;
  const int n_t = visible_entries(q_pos0, T, m, qi, n_max);
  const void* row = score_row<kB16>(scores, qi, ld);
  int32_t* out = out_idx + (int64_t)qi * k;
  if (n_t <= k) {
    for (int i = threadIdx.x; i < k; i += kThreads) out[i] = i < n_t ? i : -1;
    return;
  }
  int bstar, cgt, ncand;
  threshold_bin(ghist + (int64_t)qi * kScoreHistBins, k, S, &bstar, &cgt, &ncand);
  const int nb = ncand - cgt;
  if (bstar < 0 || nb > kTieCap || __ldcg(gcount + qi) != nb) {
    select_full<kB16>(row, n_t, k, out, S);
    return;
  }
  if (threadIdx.x < kSub) S.h2[threadIdx.x] = __ldcg(gh2 + (int64_t)qi * kSub + threadIdx.x);
  for (int c = threadIdx.x; c < nb; c += kThreads) {
    S.tidx[c] = __ldcg(gtidx + (int64_t)qi * kTieCap + c);
    S.tkey[c] = __ldcg(gtkey + (int64_t)qi * kTieCap + c);
  }
  __syncthreads();
  uint32_t* rowbits = gbits + (int64_t)qi * (ld / 32);
  resolve_ties<kB16>(nb, k - cgt, n_t, S, [&](int i) { atomicOr(rowbits + (i >> 5), 1u << (i & 31)); });
  // output: each thread owns a contiguous run of bitmap words
  const int words = (n_t + 31) / 32;
  const int per = (words + kThreads - 1) / kThreads;
  const int w0 = min(words, (int)threadIdx.x * per), w1 = min(words, w0 + per);
  int cnt = 0;
  for (int w = w0; w < w1; ++w) cnt += __popc(__ldcg(rowbits + w));
  int tot;
  int pos = block_scan_excl(cnt, S.tmp, &tot);
  for (int w = w0; w < w1; ++w) {
    uint32_t word = __ldcg(rowbits + w);
    while (word) {
      const int e = __ffs(word) - 1;
      word &= word - 1;
      out[pos++] = 32 * w + e;
    }
  }
}

struct StageSmem {
  uint32_t ckey[kCap];
  uint32_t hist[256];
  uint32_t sel[2];
  int tmp[40];
};

// No-histogram mode: the whole row's keys staged in shared memory (rows up
// to kCap entries), radix select, ordered compaction.
template <bool kB16>
__global__ void __launch_bounds__(kThreads, 1) topk_staged(const void* __restrict__ scores, int ld, int n_max,
                                                            const int32_t* __restrict__ q_pos0, int T, int m, int k,
                                                            int32_t* __restrict__ out_idx) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  pdl_wait();
  pdl_trigger();
  const int qi = blockIdx.x;
  const int n_t = visible_entries(q_pos0, T, m, qi, n_max);
  const void* row = score_row<kB16>(scores, qi, ld);
  int32_t* out = out_idx + (int64_t)qi * k;
  if (n_t <= k) {
    for (int i = threadIdx.x; i < k; i += kThreads) out[i] = i < n_t ? i : -1;
    return;
  }
  if (n_t > kCap) {
    select_full<kB16>(row, n_t, k, out, *reinterpret_cast<BitSmem*>(smem_raw));
    return;
  }
  StageSmem& S = *reinterpret_cast<StageSmem*>(smem_raw);
  // coalesced 16-byte loads: 4 fp32 or 8 BF16 scores per thread per pass
  constexpr int kPer = kB16 ? 8 : 4;
  for (int s = kPer * threadIdx.x; s < n_t; s += kPer * kThreads) {
    uint32_t kk[kPer];
    if (kB16) {
      const uint4 v = *reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(row) + s);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        kk[2 * j] = score_key16(w[j]);
        kk[2 * j + 1] = score_key16(w[j] >> 16);
      }
    } else {
      const float4 v = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(row) + s);
      kk[0] = score_key(v.x);
      kk[1] = score_key(v.y);
      kk[2] = score_key(v.z);
      kk[3] = score_key(v.w);
    }
#pragma unroll
    for (int e = 0; e < kPer; ++e)
      if (s + e < n_t) S.ckey[s + e] = kk[e];
  }
  __syncthreads();
  uint32_t thr;
  int need;
  radix_select<ScoreKeys<kB16>::kBits>(n_t, k, [&](int i) { return S.ckey[i]; }, S.hist, S.sel, &thr, &need);
  // keys above thr are all kept; keys == thr take `need` slots, lowest
  // index first.  Every thread owns a contiguous run of entries, so two
  // block scans place the run's equal keys and its outputs in order.
  const int per = (n_t + kThreads - 1) / kThreads;
  const int r0 = min(n_t, (int)threadIdx.x * per), r1 = min(n_t, r0 + per);
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
    if (take) out[pos++] = i;
  }
}

template <class K>
cudaError_t set_smem(K kernel, size_t bytes) {
  return set_max_smem(reinterpret_cast<const void*>(kernel), bytes);
}

// Histogram mode, rows of up to kFinishWords * 32 entries, steps 3-4 per
// query, latency-trimmed: everything the step reads from global memory (the
// row's selection bitmap, the tie list and its count, the second-level
// histogram, the 4096-bin histogram) is requested at once, the tie
// winners are marked in a shared-memory copy of the bitmap, and each warp
// writes the indices of a contiguous run of bitmap words (lanes read
// consecutive words; shuffle prefix sums place them).
constexpr int kFinishWords = 8192;            // 262144 entries: 32 KB of bitmap in shared memory
constexpr int kFinishPer = kFinishWords / kThreads;
constexpr int kTiePer = kTieCap / kThreads;

template <bool kB16>
__global__ void __launch_bounds__(kThreads, 1) topk_chunk_finish_s(const void* __restrict__ scores, int ld,
                                                                    int n_max, const uint32_t* __restrict__ ghist,
                                                                    const int32_t* __restrict__ q_pos0, int T, int m,
                                                                    int k, int32_t* __restrict__ out_idx,
                                                                    const uint32_t* __restrict__ gbits,
                                                                    const int* __restrict__ gtidx,
                                                                    const uint32_t* __restrict__ gtkey,
                                                                    const int* __restrict__ gcount,
                                                                    const uint32_t* __restrict__ gh2) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  BitSmem& S = *reinterpret_cast<BitSmem*>(smem_raw);
  uint32_t* rbits = reinterpret_cast<uint32_t*>(smem_raw + sizeof(BitSmem));  // the row's bitmap
  pdl_wait();
  pdl_trigger();
  const int qi = blockIdx.x;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int n_t = visible_entries(q_pos0, T, m, qi, n_max);
  const void* row = score_row<kB16>(scores, qi, ld);
  int32_t* out = out_idx + (int64_t)qi * k;
  if (n_t <= k) {
    for (int i = threadIdx.x; i < k; i += kThreads) out[i] = i < n_t ? i : -1;
    return;
  }
  const int words = (n_t + 31) / 32;
  // all global reads issued up front, into registers
  const uint32_t* gb = gbits + (int64_t)qi * (ld / 32);
  uint32_t bw[kFinishPer];
#pragma unroll
  for (int j = 0; j < kFinishPer; ++j) {
    const int w = threadIdx.x + kThreads * j;
    bw[j] = w < words ? __ldcg(gb + w) : 0u;
  }
  const int gc = __ldcg(gcount + qi);
  const int nl = min(gc, kTieCap);
  int ti[kTiePer];
  uint32_t tk[kTiePer];
#pragma unroll
  for (int j = 0; j < kTiePer; ++j) {
    const int c = threadIdx.x + kThreads * j;
    ti[j] = c < nl ? __ldcg(gtidx + (int64_t)qi * kTieCap + c) : 0;
    tk[j] = c < nl ? __ldcg(gtkey + (int64_t)qi * kTieCap + c) : 0u;
  }
  const uint32_t h2v = threadIdx.x < kSub ? __ldcg(gh2 + (int64_t)qi * kSub + threadIdx.x) : 0u;
  int bstar, cgt, ncand;
  threshold_bin(ghist + (int64_t)qi * kScoreHistBins, k, S, &bstar, &cgt, &ncand);
  const int nb = ncand - cgt;
  if (bstar < 0 || nb > kTieCap || gc != nb) {
    select_full<kB16>(row, n_t, k, out, S);
    return;
  }
#pragma unroll
  for (int j = 0; j < kFinishPer; ++j) {
    const int w = threadIdx.x + kThreads * j;
    if (w < words) rbits[w] = bw[j];
  }
#pragma unroll
  for (int j = 0; j < kTiePer; ++j) {
    const int c = threadIdx.x + kThreads * j;
    if (c < nb) {
      S.tidx[c] = ti[j];
      S.tkey[c] = tk[j];
    }
  }
  if (threadIdx.x < kSub) S.h2[threadIdx.x] = h2v;
  __syncthreads();
  resolve_ties<kB16>(nb, k - cgt, n_t, S, [&](int i) { atomicOr(rbits + (i >> 5), 1u << (i & 31)); });
  __syncthreads();
  // ordered output: warp wid owns words [w0, w1), walked in 32-word slabs
  const int per_warp = ((words + kThreads / 32 - 1) / (kThreads / 32) + 31) & ~31;
  const int w0 = min(words, wid * per_warp), w1 = min(words, w0 + per_warp);
  int cnt = 0;
  for (int w = w0 + lane; w < w1; w += 32) cnt += __popc(rbits[w]);
  cnt = warp_sum_int(cnt);
  int tot;
  int pos = block_scan_excl(lane == 0 ? cnt : 0, S.tmp, &tot);
  pos = __shfl_sync(0xffffffffu, pos, 0);
  for (int wb = w0; wb < w1; wb += 32) {
    const int w = wb + lane;
    uint32_t word = w < w1 ? rbits[w] : 0u;
    const int c = __popc(word);
    int incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    int p = pos + incl - c;
    while (word) {
      const int e = __ffs(word) - 1;
      word &= word - 1;
      out[p++] = 32 * w + e;
    }
    pos += __shfl_sync(0xffffffffu, incl, 31);
  }
}

// ---- no-histogram mode, rows of up to kCap entries: 256 threads per query ----
//
// Many queries with short rows (prefill): one 8-warp CTA per query, several
// CTAs per SM.  The row's keys are staged in shared memory (sized by the
// row bound), the radix select takes 8-bit passes over them, and the
// ordered compaction gives each warp a contiguous run of entries walked in
// 32-entry slabs (lane-strided, so shared-memory reads are conflict-free;
// ballots give in-slab ranks): one pass counts the run's keys equal to the
// threshold, one counts its selected entries, one writes their indices.
constexpr int kRowThreads = 256;
constexpr int kRowWarps = kRowThreads / 32;

// exclusive scan of one int per warp (lane 0's value counts) over the
// kRowWarps warps; every thread gets its warp's prefix, *total the sum.
__device__ __forceinline__ int warp_prefix(int v, int* tmp, int* total) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  if (lane == 0) tmp[wid] = v;
  __syncthreads();
  int pre = 0, tot = 0;
#pragma unroll
  for (int w = 0; w < kRowWarps; ++w) {
    const int x = tmp[w];
    pre += w < wid ? x : 0;
    tot += x;
  }
  __syncthreads();
  *total = tot;
  return pre;
}

template <bool kB16>
__global__ void __launch_bounds__(kRowThreads) topk_rows(const void* __restrict__ scores, int ld, int n_max,
                                                         const int32_t* __restrict__ q_pos0, int T, int m, int k,
                                                         int32_t* __restrict__ out_idx) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  uint32_t* ckey = reinterpret_cast<uint32_t*>(smem_raw);
  __shared__ uint32_t hist[256];
  __shared__ uint32_t sel[2];
  __shared__ int tmp[kRowWarps];
  pdl_wait();
  pdl_trigger();
  const int qi = blockIdx.x;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int n_t = visible_entries(q_pos0, T, m, qi, n_max);
  const void* row = score_row<kB16>(scores, qi, ld);
  int32_t* out = out_idx + (int64_t)qi * k;
  if (n_t <= k) {
    for (int i = threadIdx.x; i < k; i += kRowThreads) out[i] = i < n_t ? i : -1;
    return;
  }
  // stage the keys (coalesced 16-byte loads: 4 fp32 or 8 BF16 scores)
  constexpr int kPer = kB16 ? 8 : 4;
  for (int s = kPer * threadIdx.x; s < n_t; s += kPer * kRowThreads) {
    uint32_t kk[kPer];
    if (kB16) {
      const uint4 v = *reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(row) + s);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        kk[2 * j] = score_key16(w[j]);
        kk[2 * j + 1] = score_key16(w[j] >> 16);
      }
    } else {
      const float4 v = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(row) + s);
      kk[0] = score_key(v.x);
      kk[1] = score_key(v.y);
      kk[2] = score_key(v.z);
      kk[3] = score_key(v.w);
    }
#pragma unroll
    for (int e = 0; e < kPer; ++e)
      if (s + e < n_t) ckey[s + e] = kk[e];
  }
  // radix select: the key thr of the k-th largest and how many keys equal
  // to it are taken (`need`)
  uint32_t prefix = 0, mask = 0;
  int need = k;
  for (int shift = ScoreKeys<kB16>::kBits - 8; shift >= 0; shift -= 8) {
    hist[threadIdx.x] = 0u;
    __syncthreads();
    for (int i = threadIdx.x; i < n_t; i += kRowThreads) {
      const uint32_t key = ckey[i];
      if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 0xFFu], 1u);
    }
    __syncthreads();
    if (wid == 0) find_bin256(hist, (uint32_t)need, sel);
    __syncthreads();
    prefix |= sel[0] << shift;
    mask |= 0xFFu << shift;
    need -= (int)sel[1];
  }
  const uint32_t thr = prefix;
  // ordered compaction over warp runs of whole 32-entry slabs
  const int slabs = (n_t + 31) / 32;
  const int per_warp = (slabs + kRowWarps - 1) / kRowWarps;
  const int s0 = wid * per_warp, s1 = min(slabs, s0 + per_warp);
  const unsigned below = (1u << lane) - 1u;
  int n_eq = 0;
  for (int sl = s0; sl < s1; ++sl) {
    const int i = 32 * sl + lane;
    n_eq += __popc(__ballot_sync(0xffffffffu, i < n_t && ckey[i] == thr));
  }
  int tot;
  const int eq0 = warp_prefix(n_eq, tmp, &tot);
  int n_sel = 0;
  {
    int er = eq0;
    for (int sl = s0; sl < s1; ++sl) {
      const int i = 32 * sl + lane;
      const uint32_t key = i < n_t ? ckey[i] : 0u;
      const unsigned eq = __ballot_sync(0xffffffffu, i < n_t && key == thr);
      const unsigned gt = __ballot_sync(0xffffffffu, i < n_t && key > thr);
      // equal keys of this slab ranked er, er+1, ... in index order
      const int avail = max(0, min(need - er, 32));
      n_sel += __popc(gt) + min(__popc(eq), avail);
      er += __popc(eq);
    }
  }
  const int pos0 = warp_prefix(n_sel, tmp, &tot);
  {
    int er = eq0, pos = pos0;
    for (int sl = s0; sl < s1; ++sl) {
      const int i = 32 * sl + lane;
      const uint32_t key = i < n_t ? ckey[i] : 0u;
      const bool is_eq = i < n_t && key == thr;
      const unsigned eq = __ballot_sync(0xffffffffu, is_eq);
      const bool take = (i < n_t && key > thr) || (is_eq && er + __popc(eq & below) < need);
      const unsigned tk = __ballot_sync(0xffffffffu, take);
      if (take) out[pos + __popc(tk & below)] = i;
      pos += __popc(tk);
      er += __popc(eq);
    }
  }
}

template <bool kB16>
cudaError_t launch_topk_t(const csa_params& p, const void* scores, int ld, int n_max, const uint32_t* hist,
                          void* extra, const int32_t* q_pos0, int T, int32_t* out_idx, cudaStream_t st) {
  const int nq = p.B * T;
  cudaError_t e;
  if (!hist && n_max <= kCap) {
    const size_t smem = (size_t)((n_max + 3) & ~3) * 4;
    if ((e = set_smem(topk_rows<kB16>, smem)) != cudaSuccess) return e;
    return launch_pdl(topk_rows<kB16>, dim3(nq), dim3(kRowThreads), smem, st, scores, ld, n_max, q_pos0, T, p.m,
                      p.topk, out_idx);
  }
  if (!hist) {
    const size_t smem = sizeof(StageSmem) > sizeof(BitSmem) ? sizeof(StageSmem) : sizeof(BitSmem);
    if ((e = set_smem(topk_staged<kB16>, smem)) != cudaSuccess) return e;
    return launch_pdl(topk_staged<kB16>, dim3(nq), dim3(kThreads), smem, st, scores, ld, n_max, q_pos0, T, p.m,
                      p.topk, out_idx);
  }
  const size_t smem = sizeof(BitSmem);
  if (n_max <= kChunk) {
    const size_t smem_f = kRowStageOff + (size_t)ld * (kB16 ? 2 : 4);
    if ((e = set_smem(topk_fused<kB16>, smem_f)) != cudaSuccess) return e;
    return launch_pdl(topk_fused<kB16>, dim3(nq), dim3(kThreads), smem_f, st, scores, ld, n_max, hist, q_pos0, T, p.m,
                      p.topk, out_idx);
  }
  // the counters and second-level histograms follow the per-query
  // histograms (cleared with them); bitmap and tie lists are in `extra`
  int* gcount = reinterpret_cast<int*>(const_cast<uint32_t*>(hist) + (size_t)nq * kScoreHistBins);
  uint32_t* gh2 = reinterpret_cast<uint32_t*>(gcount + ((nq + 3) & ~3));
  uint32_t* gbits = reinterpret_cast<uint32_t*>(extra);
  int* gtidx = reinterpret_cast<int*>(gbits + (size_t)nq * (ld / 32));
  uint32_t* gtkey = reinterpret_cast<uint32_t*>(gtidx + (size_t)nq * kTieCap);
  const int chunks = (n_max + kChunk - 1) / kChunk;
  if ((e = set_smem(topk_chunk_pass<kB16>, smem)) != cudaSuccess) return e;
  e = launch_pdl(topk_chunk_pass<kB16>, dim3(nq, chunks), dim3(kThreads), smem, st, scores, ld, n_max, hist, q_pos0,
                 T, p.m, p.topk, gbits, gtidx, gtkey, gcount, gh2);
  if (e != cudaSuccess) return e;
  if (ld / 32 <= kFinishWords) {
    const size_t smem_s = smem + (size_t)kFinishWords * 4;
    if ((e = set_smem(topk_chunk_finish_s<kB16>, smem_s)) != cudaSuccess) return e;
    return launch_pdl(topk_chunk_finish_s<kB16>, dim3(nq), dim3(kThreads), smem_s, st, scores, ld, n_max, hist,
                      q_pos0, T, p.m, p.topk, out_idx, (const uint32_t*)gbits, (const int*)gtidx,
                      (const uint32_t*)gtkey, (const int*)gcount, (const uint32_t*)gh2);
  }
  if ((e = set_smem(topk_chunk_finish<kB16>, smem)) != cudaSuccess) return e;
  return launch_pdl(topk_chunk_finish<kB16>, dim3(nq), dim3(kThreads), smem, st, scores, ld, n_max, hist, q_pos0, T,
                    p.m, p.topk, out_idx, gbits, (const int*)gtidx, (const uint32_t*)gtkey, (const int*)gcount,
                    (const uint32_t*)gh2);
}

}  // namespace

bool topk_use_hist(int queries) { return queries <= 4096; }

int topk_scores_ld(int n_max) { return (n_max + 31) & ~31; }

// Cleared region of histogram mode: per-query 4096-bin histograms, tie
// counts (padded to 16 bytes) and 256-bin second-level histograms.
size_t topk_zero_bytes(int queries) {
  return (size_t)queries * kScoreHistBins * 4 + (size_t)((queries + 3) & ~3) * 4 + (size_t)queries * kSub * 4;
}

// Histogram mode with rows over 32768 entries: selection bitmaps and tie
// lists.
size_t topk_extra_bytes(int queries, int n_max) {
  if (n_max <= kChunk) return 0;
  return (size_t)queries * (topk_scores_ld(n_max) / 32) * 4 + (size_t)queries * kTieCap * 8;
}

cudaError_t launch_topk_select(const csa_params& p, const void* scores, bool bf16, int ld, int n_max,
                               const uint32_t* hist, void* extra, const int32_t* q_pos0, int T, int32_t* out_idx,
                               cudaStream_t st) {
  return bf16 ? launch_topk_t<true>(p, scores, ld, n_max, hist, extra, q_pos0, T, out_idx, st)
              : launch_topk_t<false>(p, scores, ld, n_max, hist, extra, q_pos0, T, out_idx, st);
}

}  // namespace csa
