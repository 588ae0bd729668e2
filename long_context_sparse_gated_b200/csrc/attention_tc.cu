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
//   resolve   128 threads map the tile's slots to cache / window row
//             addresses (the next tile's selected entries are loaded at the
//             start of a tile and resolved after its S MMAs are issued,
//             when those rows are also prefetched into L2)
//   gather    every thread loads its share of the tile (row 8 warp +
//             lane/4, nine 16-byte chunks) and the row's scale straight into
//             registers, before the wait for the previous tile's O MMAs;
//             for the first tile the BF16 query (TMA) arrives meanwhile and
//             each head's amax is taken
//   convert   the four lanes of a row agree on its factors, convert it to
//             FP16 and store it into a 128-row x 512-dim K-major tile V'
//             (128-byte swizzle); the query is converted in place to FP16
//             times 2^-e (e from its amax, so that it fits FP16 whatever its
//             BF16 range; 2^e joins the logit factor).
//   S^T       tcgen05.mma kind::f16 (FP16 A/B, FP32 accumulate):
//             S^T[j, h] = sum_c V'[j, c] Q'[h, c]
//             (M = 128 rows, N = 64 heads, K = 512) into TMEM, 32
//             back-to-back MMAs from precomputed descriptors, plus 4 more
//             that add the FP16 rounding residue of the scaled RoPE dims
//             (hi + lo parts), so every logit is exact up to fp32 rounding
//   softmax   per row thread: z = tau * c_j * 2^e * S^T (base 2); per-head
//             maxima of u = z + log2 c_j and sums by warp-transposed
//             shuffles; the running max of u is raised lazily (only when a
//             tile exceeds it by > 11.5), so O is rarely rescaled;
//             P' = exp2(u - m_h) in FP16 (<= 2^11.5 whatever the row's
//             scale), stored MN-major; the denominator gets P' / c_j
//   O^T       tcgen05.mma: O^T[c, h] += sum_j V'[j, c] P'[j, h]
//             (A = V'^T, the same tile read MN-major; B = P' MN-major;
//             M = 128 dims x 4 blocks, N = 64 heads, K = 128 rows)
//   epilogue  normalise (with the sink term when the split is the whole
//             row set), inverse RoPE, then the 64 x 512 result is staged in
//             shared memory and written with one bulk store: the BF16
//             output, or with several splits the fp32 partial O/l and
//             (m, l) that attn_merge_f32 combines in split order.
//
// Range.  Row j is stored as V'_j = v_j / c_j with c_j = s_j * 2^-k_j: the
// E4M3 codes times 2^k_j (exact) and the BF16 RoPE dims times 2^k_j / s_j,
// where k_j <= 0 is the smallest shift that keeps the RoPE dims below 2^15
// (k_j = 0 unless they exceed about 2^14 s_j).  So every FP16 operand is in
// range for any finite row scale in [2^-90, 2^90] and any finite BF16 RoPE
// dims and query; the logit and the output accumulate in fp32.  Rows whose
// scale is outside that range, and logits that are not finite in fp32, are
// dropped with CSA_DEV_ERR_RANGE.
//
// 16 warps (four per TMEM lane quadrant, 16 heads each) gather, convert
// (warp w: row block w), run the softmax and the epilogue; thread 128 also
// issues the query TMA and the MMAs between block barriers.  Every wait is
// bounded (CSA_DEV_ERR_TIMEOUT).
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
constexpr int kThreads = 512;             // 16 warps: four per TMEM lane quadrant
constexpr int kWarps = kThreads / 32;
constexpr int kHPart = kHg / 4;           // heads per softmax / epilogue thread (16)
constexpr int kLoads = kRows * kChunks / kThreads;  // 9 loads per thread per tile
static_assert(kRows * kChunks % kThreads == 0, "gather must divide evenly");
static_assert(kChunks == 36 && kLoads == 9 && kRows / 8 == kWarps, "warp w converts row block w, chunk groups 0..8");
constexpr float kLog2e = 1.4426950408889634f;
// logits are kept in base-2 units (z * log2 e) so that probabilities are
// exp2f of a difference; the running max is raised only when a tile exceeds
// it by more than 11.5 (2^11.5 < 3000), so O is rarely rescaled
constexpr float kLazy = 11.5f;
constexpr uint32_t kTmemCols = 512;        // S^T: 64, O^T: 4 x 64

struct __align__(1024) AttnSmem {
  uint8_t v[8][kRows * 128];  // 8 K-chunks of 64 dims: [128 rows][128 B], 128B swizzle;
                              // after the last tile: the [64 heads][512 dims] output stage
  uint8_t p[kRows * 128];     // P' MN-major: [128 rows][64 heads] FP16, 128B swizzle
  uint8_t q[8][kHg * 128];    // 8 K-chunks: [64 heads][128 B]
  const uint8_t* rowp[2][kRows];  // stored row of each tile slot (null: empty), tiles i and i+1
  const float* rscp[2][kRows];    // its scale s_j
  float row_f[kRows];         // tau * log2(e) * c_j  (c_j = s_j 2^-k_j)
  float row_lc[kRows];        // log2 c_j
  float row_ic[kRows];        // 1 / c_j
  int live[kRows];            // row takes part (non-empty slot with a valid scale)
  uint32_t qamax[kHg];        // fp32 bits of each head's largest query magnitude
  float qg[kHg];              // 2^e_h: Q'_h = Q_h 2^-e_h
  float red[kWarps][32];
  float mh[kHg], lh[kHg], alpha[kHg];
  float rope_c[kR / 2], rope_s[kR / 2];  // inverse-RoPE rotation of this query
  uint64_t bar_q, bar_s, bar_o;
  uint32_t tmem_base;
  int abort;
  int rescale;
};


__device__ __forceinline__ uint32_t sw128(int row, int chunk16) {
  return (uint32_t)(row * 128 + ((chunk16 ^ (row & 7)) << 4));
}

// descriptor + byte offset (start-address field, 16-byte units; shared
// addresses stay below 2^18, so the 14-bit field does not overflow)
__device__ __forceinline__ uint64_t dadd(uint64_t d, uint32_t bytes) { return d + (uint64_t)(bytes >> 4); }

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

// 8 BF16 values times s as FP16 hi + lo pairs: hi = fp16(x), lo =
// fp16(x - hi), so that hi + lo carries x to about 22 bits.
__device__ __forceinline__ void bf16x8_scale_to_f16_hilo(const uint4& in, float s, uint4& hi, uint4& lo) {
  const uint32_t w[4] = {in.x, in.y, in.z, in.w};
  uint32_t h[4], l[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float a = bf16_bits_to_f32(w[i]) * s, b = bf16_bits_to_f32(w[i] >> 16) * s;
    const __half2 hh = __floats2half2_rn(a, b);
    const float2 hf = __half22float2(hh);
    const __half2 ll = __floats2half2_rn(a - hf.x, b - hf.y);
    h[i] = *reinterpret_cast<const uint32_t*>(&hh);
    l[i] = *reinterpret_cast<const uint32_t*>(&ll);
  }
  hi = make_uint4(h[0], h[1], h[2], h[3]);
  lo = make_uint4(l[0], l[1], l[2], l[3]);
}

// Largest-magnitude bits of the 8 BF16 values in a 16-byte word (sign
// cleared; as integers these order like the magnitudes).
__device__ __forceinline__ uint32_t bf16x8_amax_bits(const uint4& in) {
  const uint32_t w[4] = {in.x, in.y, in.z, in.w};
  uint32_t m = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) m = max(m, max(w[i] & 0x7FFFu, (w[i] >> 16) & 0x7FFFu));
  return m;
}

// Shift k <= 0 of row j: with R the row's largest RoPE magnitude (BF16
// bits) and s its scale, R * 2^k / s < 2^15 for k = min(0, 14 + e_s - e_R)
// (e = unbiased exponent: R < 2^(e_R+1), s >= 2^e_s).
__device__ __forceinline__ int row_shift(float s, uint32_t rbits) {
  if (rbits == 0u) return 0;
  const int e_s = (int)((__float_as_uint(s) >> 23) & 0xFFu) - 127;
  const int e_r = (int)((rbits >> 7) & 0xFFu) - 127;
  return min(0, 14 + e_s - e_r);
}

__device__ __forceinline__ uint32_t pack_half2(float a, float b) {
  const __half2 r = __floats2half2_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&r);
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

// max / sum over the 32 lanes of a warp for each of 16 values: afterwards
// lane l holds the reduction of value index l % 16.
template <bool kMax>
__device__ __forceinline__ float warp_transpose_reduce16(float (&v)[16]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int s = 8; s >= 1; s >>= 1) {
    const bool up = lane & s;
#pragma unroll
    for (int i = 0; i < s; ++i) {
      const float keep = up ? v[i + s] : v[i];
      const float send = up ? v[i] : v[i + s];
      const float recv = __shfl_xor_sync(0xffffffffu, send, s);
      v[i] = kMax ? fmaxf(keep, recv) : keep + recv;
    }
  }
  const float o = __shfl_xor_sync(0xffffffffu, v[0], 16);
  return kMax ? fmaxf(v[0], o) : v[0] + o;
}

// The selected entry held by candidate slot `slot` of query qi (sparse
// mode, slot < n_sel < se), loaded ahead of its use; -1 otherwise.
template <bool kDense>
__device__ __forceinline__ int slot_entry(int slot, int se, int n_sel, int qi, const int32_t* __restrict__ idx,
                                          int topk) {
  if (kDense || slot >= se || slot >= n_sel) return -1;
  return __ldg(idx + (int64_t)qi * topk + slot);
}

// Row of candidate slot `slot` (< se) of query t, given its entry e from
// slot_entry: src 1 = cache row, 2 = window ring row, 0 = empty; *off =
// element row index into that array.
template <bool kDense>
__device__ __forceinline__ int resolve_slot(int slot, int e, int se, int n_sel, int64_t t, int64_t n_t, int W, int bs,
                                            int64_t cache_cap, int64_t win_cap, int32_t* err, int64_t* off) {
  int src = 0;
  int64_t row = 0;
  if (slot < se) {
    if (slot < n_sel) {
      if (kDense) {
        if (slot < n_t && slot < cache_cap) { src = 1; row = slot; }
      } else {
        if (e >= 0 && e < n_t && e < cache_cap) { src = 1; row = e; }
        else if (e != -1) raise_err(err, CSA_DEV_ERR_INDEX);
      }
    } else {
      const int64_t pos = t - W + 1 + (slot - n_sel);
      if (pos >= 0) { src = 2; row = pos % win_cap; }
    }
  }
  *off = src == 1 ? (int64_t)bs * cache_cap + row : (src == 2 ? (int64_t)bs * win_cap + row : -1);
  return src;
}

template <bool kDense>
__global__ void __launch_bounds__(kThreads, 1) attn_tc(
    const __grid_constant__ CUtensorMap tm_q, const uint8_t* __restrict__ cache_rows,
    const float* __restrict__ cache_scale, int64_t cache_cap, const uint8_t* __restrict__ win_rows,
    const float* __restrict__ win_scale, int64_t win_cap, const int32_t* __restrict__ idx, int topk,
    const int32_t* __restrict__ q_pos0, int T, int m, int W, int n_sel, int n_heads, float tau,
    float theta, const float* __restrict__ sink, int rows_per_split, int n_splits, uint16_t* __restrict__ out,
    float* __restrict__ ws_o, float* __restrict__ ws_ml, int32_t* __restrict__ err) {
  extern __shared__ uint8_t smem_raw[];
  AttnSmem& S = *reinterpret_cast<AttnSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int wt = threadIdx.x;                // 0..255
  const int quad = warp & 3;                 // TMEM lane quadrant of this warp
  const int part = warp >> 2;                // head part: 16*part .. +15
  const int j = quad * 32 + lane;            // tile row of this thread
  const int qi = blockIdx.x, split = blockIdx.y, hg = blockIdx.z;
  const int bs = qi / T, tq = qi % T;
  const int h0 = hg * kHg;
  volatile int* abort = &S.abort;
  // MMA / TMA issuer: warp 4 resolves no rows and updates no head sums, so
  // its lane 0 is free when a tile's operands are ready
  const bool issuer = threadIdx.x == 128;

  if (issuer) {
    sm100::mbar_init(&S.bar_q, 1);
    sm100::mbar_init(&S.bar_s, 1);
    sm100::mbar_init(&S.bar_o, 1);
    S.abort = 0;
    sm100::fence_mbar_init();
  }
  if (threadIdx.x < kHg) {
    S.qamax[threadIdx.x] = 0u;
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
  // this query's own slots: its entries (CSA: the k selected; HCA: its n_t
  // visible ones), then its window; split boundaries depend on nothing else
  const int own_sel = kDense ? (int)min((int64_t)n_sel, n_t) : n_sel;
  const int total = own_sel + W;
  const int own_splits = (total + rows_per_split - 1) / rows_per_split;
  const bool single = own_splits == 1;
  const int sb = split * rows_per_split;
  const int se = min(total, sb + rows_per_split);
  const int n_tiles = se > sb ? (se - sb + kRows - 1) / kRows : 0;
  const uint32_t tmem = S.tmem_base;
  const uint32_t s_col = tmem;         // S^T: 64 columns
  const uint32_t o_col = tmem + 64;    // O^T block b: columns 64 + 64 b
  if (issuer) {
    sm100::prefetch_tmap(&tm_q);
    sm100::mbar_arrive_expect_tx(&S.bar_q, 8 * kHg * 128);
    for (int c = 0; c < 8; ++c) sm100::tma_load_2d(S.q[c], &tm_q, &S.bar_q, 64 * c, qi * n_heads + h0);
  }
  // the inverse-RoPE rotation by -t of the 32 RoPE pairs, once per CTA
  if (single && wt >= 64 && wt < 64 + kR / 2) {
    float c, sn;
    rope_cos_sin(-(double)t, wt - 64, kR, (double)theta, &c, &sn);
    S.rope_c[wt - 64] = c;
    S.rope_s[wt - 64] = sn;
  }
  const uint32_t idS = sm100::idesc_f16(kRows, kHg, 0, 0);
  const uint32_t idO = sm100::idesc_f16(128, kHg, 1, 1);
  // K-major V' (A of S^T), K-major Q (B of S^T), MN-major V'^T (A of O^T:
  // 64-dim atoms 16 KB apart, 8-row groups 1 KB apart), MN-major P' (B of
  // O^T: one 64-head atom, 8-row groups 1 KB apart)
  const uint64_t dV = sm100::smem_desc(sm100::smem_u32(S.v[0]), 16, 1024, 2);
  const uint64_t dQ = sm100::smem_desc(sm100::smem_u32(S.q[0]), 16, 1024, 2);
  const uint64_t dVt = sm100::smem_desc(sm100::smem_u32(S.v[0]), kRows * 128, 1024, 2);
  const uint64_t dP = sm100::smem_desc(sm100::smem_u32(S.p), kRows * 128, 1024, 2);
  const uint64_t dPk = sm100::smem_desc(sm100::smem_u32(S.p), 16, 1024, 2);  // P' buffer read K-major (RoPE lo parts)

  // Row of this thread (wt < kRows) in the current tile, resolved one tile
  // ahead: while tile i is computed, tile i+1's rows are resolved, their
  // scales loaded and their bytes prefetched into L2.
  // the row and scale addresses of a slot (its entry pre-loaded); the
  // scales are loaded together with the rows' bytes
  auto resolve_to = [&](int buf, int slot, int e) {
    int64_t off = -1;
    const int src = resolve_slot<kDense>(slot, e, se, own_sel, t, n_t, W, bs, cache_cap, win_cap, err, &off);
    const uint8_t* rp = nullptr;
    const float* sp = nullptr;
    if (src == 1) { rp = cache_rows + off * kRowBytes; sp = cache_scale + off; }
    if (src == 2) { rp = win_rows + off * kRowBytes; sp = win_scale + off; }
    S.rowp[buf][wt] = rp;
    S.rscp[buf][wt] = sp;
    return rp;
  };
  if (wt < kRows && n_tiles > 0) resolve_to(0, sb + wt, slot_entry<kDense>(sb + wt, se, own_sel, qi, idx, topk));

  // Control flow is uniform across the CTA (every __syncthreads is reached
  // by all threads); a failed bounded wait only raises the abort flag,
  // after which every later wait returns at once and no MMA is issued.
  for (int i = 0; i < n_tiles; ++i) {
    const int tb = sb + i * kRows;
    if (i == 0) __syncthreads();  // tile 0's row pointers visible
    if (wt == 0) S.rescale = 0;
    // -- gather: this thread's share of the tile, row r (8-row block `warp`),
    //    16-byte chunks 4k + lane%4 (k < 7: E4M3 codes of K-chunk k; k = 7, 8:
    //    RoPE dims), straight from global memory into registers.  The loads
    //    are issued before the wait for the previous tile's O MMA, so they
    //    overlap it; the rows were prefetched into L2 during that tile.
    const int r = 8 * warp + (lane >> 2);
    const uint8_t* rp = S.rowp[i & 1][r];
    const float* sp = S.rscp[i & 1][r];
    uint4 raw[kLoads];
#pragma unroll
    for (int k = 0; k < kLoads; ++k)
      raw[k] = rp ? __ldg(reinterpret_cast<const uint4*>(rp + (4 * k + (lane & 3)) * 16)) : make_uint4(0, 0, 0, 0);
    float sc = sp ? __ldg(sp) : 1.f;
    // the next tile's selected entries: loaded now, resolved after this
    // tile's S MMAs are issued
    const int nx_slot = tb + kRows + wt;
    const int nx_e = (wt < kRows && i + 1 < n_tiles) ? slot_entry<kDense>(nx_slot, se, own_sel, qi, idx, topk) : -1;
    if (i > 0) sm100::mbar_wait(&S.bar_o, (i - 1) & 1, abort);  // V' and P' buffers free
    if (i == 0) {
      // each head's largest BF16 query magnitude (converted after the
      // barrier).  Word e of the query tile is head ((e >> 3) & 63): this
      // thread's words (e = wt + 512 n) all belong to head wt/8
      sm100::mbar_wait(&S.bar_q, 0, abort);
      const uint4* qv = reinterpret_cast<const uint4*>(&S.q[0][0]);
      uint32_t ma = 0;
#pragma unroll 4
      for (int e = wt; e < 8 * kHg * 128 / 16; e += kThreads) ma = max(ma, bf16x8_amax_bits(qv[e]));
#pragma unroll
      for (int o = 1; o < 8; o <<= 1) ma = max(ma, __shfl_xor_sync(0xffffffffu, ma, o));
      if ((lane & 7) == 0) atomicMax(&S.qamax[wt >> 3], ma << 16);
    }
    // -- row factors (the four lanes of row r agree): the row's largest RoPE
    //    magnitude, its shift k_j, the factors of its codes and RoPE dims, and
    //    for the softmax those of its logits and denominator terms
    bool live = rp != nullptr;
    if (!(sc >= 0x1p-90f) || !(sc <= 0x1p90f)) {  // outside the supported scale range
      if (live) raise_err(err, CSA_DEV_ERR_RANGE);
      live = false;  // the row is dropped (zeros)
      sc = 1.f;
    }
    float code_mul, rope_mul;
    {
      uint32_t rb = max(bf16x8_amax_bits(raw[kLoads - 2]), bf16x8_amax_bits(raw[kLoads - 1]));
      rb = max(rb, __shfl_xor_sync(0xffffffffu, rb, 1));
      rb = max(rb, __shfl_xor_sync(0xffffffffu, rb, 2));
      const int kr = row_shift(sc, rb);
      const float cj = ldexpf(sc, -kr);
      code_mul = kr >= -24 ? __uint_as_float((uint32_t)(127 + kr) << 23) : 0.f;
      rope_mul = ldexpf(1.f / sc, kr);
      if ((lane & 3) == 0) {
        S.live[r] = live;
        S.row_f[r] = live ? tau * kLog2e * cj : 0.f;
        S.row_lc[r] = log2f(cj);
        S.row_ic[r] = 1.f / cj;
      }
    }
    if (i == 0) {
      __syncthreads();  // query amax complete
      // each head's power-of-two range factor 2^e_h: Q'_h = Q_h 2^-e_h has
      // its largest magnitude in [2^14, 2^15)
      auto head_exp = [&](int h) {
        const uint32_t a = S.qamax[h];
        return a ? min(126, max(-126, (int)((a >> 23) & 0xFFu) - 127 - 14)) : 0;
      };
      if (wt < kHg) S.qg[wt] = __uint_as_float((uint32_t)(127 + head_exp(wt)) << 23);
      const float qia = __uint_as_float((uint32_t)(127 - head_exp(wt >> 3)) << 23);
      uint4* qv = reinterpret_cast<uint4*>(&S.q[0][0]);
#pragma unroll 4
      for (int e = wt; e < 8 * kHg * 128 / 16; e += kThreads) qv[e] = bf16x8_scale_to_f16(qv[e], qia);
    }
    // -- convert + store V' (empty and dropped rows as zeros)
#pragma unroll
    for (int k = 0; k < kLoads; ++k) {
      const int c = 4 * k + (lane & 3);
      if (k < kNope / 64) {
        // dims 16c .. 16c+15 -> K-chunk (16c)/64, 16-byte slots 2(c%4), 2(c%4)+1;
        // codes times 2^k (exact down to 2^-24)
        uint4 lo = make_uint4(0, 0, 0, 0), hi = lo;
        if (live) {
          e4m3x16_to_f16(raw[k], lo, hi);
          if (code_mul != 1.f) {
            const __half2 f = __float2half2_rn(code_mul);
            __half2* ph = reinterpret_cast<__half2*>(&lo);
            __half2* qh = reinterpret_cast<__half2*>(&hi);
#pragma unroll
            for (int x = 0; x < 4; ++x) { ph[x] = __hmul2(ph[x], f); qh[x] = __hmul2(qh[x], f); }
          }
        }
        uint8_t* ch = S.v[c >> 2];
        *reinterpret_cast<uint4*>(ch + sw128(r, 2 * (c & 3))) = lo;
        *reinterpret_cast<uint4*>(ch + sw128(r, 2 * (c & 3) + 1)) = hi;
      } else {
        // RoPE dims 448 + 8(c-28) .. times 2^k / s: hi in chunk 7 (slot
        // c-28, read by both MMAs), lo at the same place of the P' buffer
        // (free until the softmax; read by the S MMA only)
        uint4 hi = make_uint4(0, 0, 0, 0), lo = hi;
        if (live) bf16x8_scale_to_f16_hilo(raw[k], rope_mul, hi, lo);
        *reinterpret_cast<uint4*>(S.v[7] + sw128(r, c - kNope / 16)) = hi;
        *reinterpret_cast<uint4*>(S.p + sw128(r, c - kNope / 16)) = lo;
      }
    }
    sm100::fence_proxy_async_smem();
    __syncthreads();
    // -- S^T = V' Q^T over K = 512 (32 steps of 16), plus the RoPE dims'
    //    lo parts against the query's RoPE dims (4 steps)
    if (issuer) {
      sm100::tc_fence_after();
      if (!*abort) {
#pragma unroll
        for (int kk = 0; kk < 32; ++kk) {
          const uint32_t o = (uint32_t)((kk >> 2) * kRows * 128 + (kk & 3) * 32);
          const uint32_t oq = (uint32_t)((kk >> 2) * kHg * 128 + (kk & 3) * 32);
          sm100::mma_f16(s_col, dadd(dV, o), dadd(dQ, oq), idS, kk > 0);
        }
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          sm100::mma_f16(s_col, dadd(dPk, (uint32_t)(kk * 32)), dadd(dQ, (uint32_t)(7 * kHg * 128 + kk * 32)), idS, 1u);
        sm100::tc_commit(&S.bar_s);
      }
    }
    // -- next tile: resolve, scale load and L2 prefetch while this one runs
    if (wt < kRows && i + 1 < n_tiles) {
      const uint8_t* nx = resolve_to((i + 1) & 1, nx_slot, nx_e);
      if (nx) sm100::bulk_prefetch_l2(nx, kRowBytes);
    }
    sm100::mbar_wait(&S.bar_s, i & 1, abort);
    sm100::tc_fence_after();
    // -- this thread's row: c_j = s_j 2^-k_j, and u = z + log2 c_j (base-2
    //    logit plus the row's log-scale) for its 16 heads
    const float inv_c = S.row_ic[j];  // 1 / c_j
    float z[kHPart];
    {
      uint32_t a[16];
      sm100::tmem_ld_x16(s_col + ((uint32_t)(quad * 32) << 16) + kHPart * part, a);
      sm100::tmem_ld_wait();
      sm100::tmem_pin16(a);
      const bool valid = S.live[j] != 0;
      const float f = S.row_f[j];
      const float lc = S.row_lc[j];
      bool bad = false;
#pragma unroll
      for (int c = 0; c < kHPart; ++c) {
        const float za = f * S.qg[kHPart * part + c] * __uint_as_float(a[c]);
        const bool ba = !(fabsf(za) < INFINITY);
        bad |= valid && ba;
        z[c] = (valid && !ba) ? za + lc : -INFINITY;
      }
      if (bad) raise_err(err, CSA_DEV_ERR_RANGE);  // a logit beyond fp32: dropped
    }
    // per-head tile maxima
    {
      float v[kHPart];
#pragma unroll
      for (int c = 0; c < kHPart; ++c) v[c] = z[c];
      S.red[warp][lane] = warp_transpose_reduce16<true>(v);  // head 16*part + lane%16, this warp's rows
    }
    __syncthreads();
    if (wt < kHg) {
      const int h = wt, hp = h / kHPart, hl = h % kHPart;
      float tmax = -INFINITY;
      for (int q4 = 0; q4 < 4; ++q4) tmax = fmaxf(tmax, S.red[4 * hp + q4][hl]);
      const float mo = S.mh[h];
      float al = 1.f;
      int resc = 0;
      if (i == 0) {
        S.mh[h] = tmax;
      } else if (tmax > mo + kLazy) {
        al = (mo == -INFINITY) ? 0.f : exp2f(mo - tmax);
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
        uint32_t r16[16];
        const uint32_t ta = o_col + 64 * blk + ((uint32_t)(quad * 32) << 16) + kHPart * part;
        sm100::tmem_ld_x16(ta, r16);
        sm100::tmem_ld_wait();
        sm100::tmem_pin16(r16);
#pragma unroll
        for (int c = 0; c < 16; ++c) r16[c] = __float_as_uint(__uint_as_float(r16[c]) * S.alpha[kHPart * part + c]);
        sm100::tmem_st_x16(ta, r16);
      }
      sm100::tmem_st_wait();
    }
    // P' = exp2(u - m_h) (FP16 stores: row j, heads 16*part .. +15 = two
    // 16-byte words) and the per-head sums of exp2(z - m_h) = P' / c_j
    {
      float v[kHPart];
#pragma unroll
      for (int c = 0; c < kHPart; ++c) {
        const float mh = S.mh[kHPart * part + c];
        v[c] = (mh == -INFINITY || z[c] == -INFINITY) ? 0.f : exp2f(z[c] - mh);
      }
#pragma unroll
      for (int w2 = 0; w2 < 2; ++w2) {
        const int b = 8 * w2;
        const uint4 pk = make_uint4(pack_half2(v[b], v[b + 1]), pack_half2(v[b + 2], v[b + 3]),
                                    pack_half2(v[b + 4], v[b + 5]), pack_half2(v[b + 6], v[b + 7]));
        *reinterpret_cast<uint4*>(S.p + sw128(j, 2 * part + w2)) = pk;
      }
#pragma unroll
      for (int c = 0; c < kHPart; ++c) v[c] *= inv_c;
      S.red[warp][lane] = warp_transpose_reduce16<false>(v);
    }
    sm100::tc_fence_before();
    sm100::fence_proxy_async_smem();
    __syncthreads();
    if (wt < kHg) {
      const int h = wt, hp = h / kHPart, hl = h % kHPart;
      float ts = 0.f;
      for (int q4 = 0; q4 < 4; ++q4) ts += S.red[4 * hp + q4][hl];
      S.lh[h] += ts;
    }
    // -- O^T[blk] += V'^T[blk] P' over K = 128 rows (8 steps of 16)
    if (issuer) {
      sm100::tc_fence_after();
      if (!*abort) {
#pragma unroll
        for (int blk = 0; blk < 4; ++blk) {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t oa = (uint32_t)(2 * blk * kRows * 128 + kk * 2048);
            sm100::mma_f16(o_col + 64 * blk, dadd(dVt, oa), dadd(dP, (uint32_t)(kk * 2048)), idO,
                           (i > 0 || kk > 0) ? 1u : 0u);
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
  __syncthreads();  // lh final; abort flag now uniform; V' free
  // per-head output factor: single split, normalised with the sink term
  // here; several splits, the partial normalised by its own sum (FP16) plus
  // (max, sum)
  if (wt < kHg) {
    const float mh = S.mh[wt], lh = S.lh[wt];
    float fh;
    if (single) {
      const float sg = sink[h0 + wt] * kLog2e;
      const float ms = fmaxf(sg, mh);
      const float den = exp2f(sg - ms) + (mh == -INFINITY ? 0.f : lh * exp2f(mh - ms));
      fh = (mh == -INFINITY || !(den > 0.f)) ? 0.f : exp2f(mh - ms) / den;
    } else {
      fh = lh > 0.f ? 1.f / lh : 0.f;
    }
    S.alpha[wt] = fh;
  }
  __syncthreads();
  const bool ok = !S.abort;
  if (ok && n_tiles > 0) {
    float f[kHPart];
#pragma unroll
    for (int c = 0; c < kHPart; ++c) f[c] = S.alpha[kHPart * part + c];
    // [64 heads][512 dims]: BF16 output, or the fp32 partial (128 KB, all of V')
    uint16_t* stage = reinterpret_cast<uint16_t*>(&S.v[0][0]);
    float* stage32 = reinterpret_cast<float*>(&S.v[0][0]);
#pragma unroll 1
    for (int b2 = 0; b2 < 4; b2 += 2) {
      // two TMEM loads in flight: blocks b2, b2+1, this warp's 16 heads
      uint32_t rr[2][16];
#pragma unroll
      for (int x = 0; x < 2; ++x)
        sm100::tmem_ld_x16(o_col + 64 * (b2 + x) + ((uint32_t)(quad * 32) << 16) + kHPart * part, rr[x]);
      sm100::tmem_ld_wait();
      sm100::tmem_pin16(rr[0]);
      sm100::tmem_pin16(rr[1]);
#pragma unroll
      for (int x = 0; x < 2; ++x) {
        const int blk = b2 + x;
        const int c_dim = 128 * blk + quad * 32 + lane;
        float cs = 1.f, sn = 0.f;
        if (single && c_dim >= kNope) {
          cs = S.rope_c[(c_dim - kNope) >> 1];
          sn = S.rope_s[(c_dim - kNope) >> 1];
        }
        const bool odd = lane & 1;
#pragma unroll
        for (int c = 0; c < kHPart; ++c) {
          const int h = kHPart * part + c;
          float y = __uint_as_float(rr[x][c]) * f[c];
          if (single) {
            const float pv = __shfl_xor_sync(0xffffffffu, y, 1);
            if (c_dim >= kNope) y = odd ? (pv * sn + y * cs) : (y * cs - pv * sn);
            stage[h * kD + c_dim] = f32_to_bf16_bits(y);
          } else {
            stage32[h * kD + c_dim] = y;
          }
        }
      }
    }
    sm100::fence_proxy_async_smem();
    __syncthreads();
    // the 64 x 512 block is contiguous in the output (64 rows of 1 KB BF16)
    // and in the split partials (2 KB fp32 rows): one bulk store
    if (issuer) {
      if (single)
        sm100::bulk_store(out + ((int64_t)qi * n_heads + h0) * kD, stage, kHg * kD * 2);
      else
        sm100::bulk_store(ws_o + (((int64_t)qi * n_splits + split) * n_heads + h0) * kD, stage32, kHg * kD * 4);
      sm100::bulk_commit();
      sm100::bulk_wait_read();  // shared memory read before the CTA exits
    }
    if (!single && wt < kHg) {
      const int64_t base = ((int64_t)qi * n_splits + split) * n_heads + h0 + wt;
      ws_ml[base * 2 + 0] = S.mh[wt] * (1.0f / kLog2e);  // natural units
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

// Combine the fp32 split partials (each O_s / l_s) of one query: for head h,
// M = max(sink, m_s), w_s = l_s e^(m_s - M) / (e^(sink - M) + sum l_s
// e^(m_s - M)), o = sum_s w_s (O_s / l_s) in split order, then the inverse
// RoPE and a BF16 store.  grid (queries, n_heads / 8), 256 threads: warp =
// head, lane = 16 dims.  The (m, l) of the first 32 splits are read once,
// one split per lane, and shared by shuffles.
__global__ void __launch_bounds__(256) attn_merge_f32(const float* __restrict__ ws_o, const float* __restrict__ ws_ml,
                                                      int n_splits, int n_heads, const float* __restrict__ sink,
                                                      const int32_t* __restrict__ q_pos0, int T, int m, int W,
                                                      int n_sel, int dense, int rows_per_split, float theta,
                                                      uint16_t* __restrict__ out) {
  __shared__ float rope_c[kR / 2], rope_s[kR / 2];
  pdl_wait();
  const int qi = blockIdx.x;
  const int h = blockIdx.y * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  const int bs = qi / T, tq = qi % T;
  const int64_t t = (int64_t)q_pos0[bs] + tq;
  // the query's own split count (a query with one split was finalised by
  // attn_tc itself); n_splits is only the workspace stride
  const int own_sel = dense ? (int)min((int64_t)n_sel, (t + 1) / m) : n_sel;
  const int own_splits = (own_sel + W + rows_per_split - 1) / rows_per_split;
  if (own_splits <= 1) return;
  if (threadIdx.x < kR / 2) {
    float c, sn;
    rope_cos_sin(-(double)t, threadIdx.x, kR, (double)theta, &c, &sn);
    rope_c[threadIdx.x] = c;
    rope_s[threadIdx.x] = sn;
  }
  // lane's dims: 4 lane + 128 e (e < 4), so that every float4 load of the
  // warp reads 512 contiguous bytes; the first four splits' partials are
  // loaded before their weights are known
  const float* src0 = ws_o + ((int64_t)qi * n_splits * n_heads + h) * kD + 4 * lane;
  const int64_t sstride = (int64_t)n_heads * kD;
  float4 pre[4][4];
#pragma unroll
  for (int sp = 0; sp < 4; ++sp)
#pragma unroll
    for (int e = 0; e < 4; ++e)
      pre[sp][e] = sp < own_splits ? __ldg(reinterpret_cast<const float4*>(src0 + sp * sstride + 128 * e))
                                   : make_float4(0.f, 0.f, 0.f, 0.f);
  const float sg = sink[h];
  const int64_t ml0 = ((int64_t)qi * n_splits * n_heads + h) * 2;  // split sp at ml0 + 2 sp n_heads
  float m_l = -INFINITY, l_l = 0.f;
  if (lane < own_splits) {
    m_l = ws_ml[ml0 + (int64_t)2 * lane * n_heads];
    l_l = ws_ml[ml0 + (int64_t)2 * lane * n_heads + 1];
  }
  float M = fmaxf(sg, warp_max(m_l));
  for (int sp = 32 + lane; sp < own_splits; sp += 32) M = fmaxf(M, ws_ml[ml0 + (int64_t)2 * sp * n_heads]);
  M = warp_max(M);
  const float p_l = (m_l == -INFINITY) ? 0.f : l_l * expf(m_l - M);  // split `lane`
  float part = p_l;
  for (int sp = 32 + lane; sp < own_splits; sp += 32) {
    const float ms = ws_ml[ml0 + (int64_t)2 * sp * n_heads];
    if (ms != -INFINITY) part += ws_ml[ml0 + (int64_t)2 * sp * n_heads + 1] * expf(ms - M);
  }
  const float den = expf(sg - M) + warp_sum(part);
  const float inv = den > 0.f ? 1.f / den : 0.f;
  const float a_l = p_l * inv;  // weight of split `lane` (for lane < 32)
  float acc[16];
#pragma unroll
  for (int e = 0; e < 16; ++e) acc[e] = 0.f;
  // splits in order; a split of weight zero (empty, or its max far below)
  // is skipped: its partial may be stale
  auto add = [&](float a, const float4 (&v)[4]) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      acc[4 * e] = fmaf(a, v[e].x, acc[4 * e]);
      acc[4 * e + 1] = fmaf(a, v[e].y, acc[4 * e + 1]);
      acc[4 * e + 2] = fmaf(a, v[e].z, acc[4 * e + 2]);
      acc[4 * e + 3] = fmaf(a, v[e].w, acc[4 * e + 3]);
    }
  };
#pragma unroll
  for (int sp = 0; sp < 4; ++sp) {
    const float a = __shfl_sync(0xffffffffu, a_l, sp);
    if (sp < own_splits && a != 0.f) add(a, pre[sp]);
  }
#pragma unroll 2
  for (int sp = 4; sp < own_splits; ++sp) {
    float a;
    if (sp < 32) {
      a = __shfl_sync(0xffffffffu, a_l, sp);
    } else {
      const float ms = ws_ml[ml0 + (int64_t)2 * sp * n_heads];
      a = ms == -INFINITY ? 0.f : ws_ml[ml0 + (int64_t)2 * sp * n_heads + 1] * expf(ms - M) * inv;
    }
    if (a == 0.f) continue;
    float4 v[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) v[e] = __ldg(reinterpret_cast<const float4*>(src0 + sp * sstride + 128 * e));
    add(a, v);
  }
  __syncthreads();  // rope table
  // inverse RoPE on dims 448..511 (block e = 3, lanes 16..31: pairs (4 lane, +1), (4 lane + 2, +3))
  if (lane >= (kNope - 384) / 4) {
#pragma unroll
    for (int x = 0; x < 2; ++x) {
      const int pr = (384 + 4 * lane - kNope) / 2 + x;
      const float cs = rope_c[pr], sn = rope_s[pr];
      const float u = acc[12 + 2 * x], y = acc[12 + 2 * x + 1];
      acc[12 + 2 * x] = u * cs - y * sn;
      acc[12 + 2 * x + 1] = u * sn + y * cs;
    }
  }
  uint16_t* dst = out + ((int64_t)qi * n_heads + h) * kD + 4 * lane;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const uint32_t lo = (uint32_t)f32_to_bf16_bits(acc[4 * e]) | ((uint32_t)f32_to_bf16_bits(acc[4 * e + 1]) << 16);
    const uint32_t hi = (uint32_t)f32_to_bf16_bits(acc[4 * e + 2]) | ((uint32_t)f32_to_bf16_bits(acc[4 * e + 3]) << 16);
    *reinterpret_cast<uint2*>(dst + 128 * e) = make_uint2(lo, hi);
  }
}

}  // namespace

bool attn_tc_supported(const csa_params& p) {
  return p.kv_fmt == CSA_KV_FP8_BF16 && p.act_fmt == CSA_ACT_BF16 && p.d == kD && p.r == kR &&
         p.n_heads % kHg == 0 && tensor_maps_available();
}

// Rows per split, a function of the call's parameters and T only -- never
// of the batch size, the other sequences' lengths or the device -- so that
// a query's output is bit-identical whatever batch it runs in (the
// batch-invariant contract of the DeepSeek-V4 write-ups: kwkr.cn notes 4.3,
// Qiaomu blog 批次不变和确定性内核).  Prefill (T > 4): all of a query's slots
// in one split.  Sparse decode (k + W slots, fixed by the parameters): up
// to 16 tiles, splits of 2 tiles (one 64-head group) or 1 tile (several
// groups already multiply the CTAs), else 8 tiles.  Dense decode (a query's
// slot count is its own n_t + W): splits of 8 tiles.
int attn_tc_rows_per_split(int total_slots, int nhg, int T, bool dense) {
  const int tiles = (total_slots + kRows - 1) / kRows;
  if (T > 4) return (tiles > 1 ? tiles : 1) * kRows;
  if (dense) return 8 * kRows;
  if (tiles <= 16) return (nhg == 1 ? 2 : 1) * kRows;
  return 8 * kRows;
}

size_t attn_tc_smem_bytes() { return sizeof(AttnSmem) + 1024; }

cudaError_t launch_attn_tc(const csa_params& p, const void* q, const csa_kv& cache, const int32_t* idx,
                           const csa_kv& win, const float* sink, const int32_t* q_pos0, int T, int n_sel,
                           bool dense, void* out, float* ws, int32_t* err, cudaStream_t st) {
  const int nq = p.B * T;
  CUtensorMap tq;
  {
    uint64_t dims[2] = {(uint64_t)kD, (uint64_t)nq * p.n_heads};
    uint64_t str[1] = {(uint64_t)kD * 2};
    uint32_t box[2] = {64, (uint32_t)kHg};
    if (!encode_tensor_map(&tq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, q, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  }
  const int total = n_sel + p.window;
  const int nhg = p.n_heads / kHg;
  const int rps = attn_tc_rows_per_split(total, nhg, T, dense);
  const int n_splits = (total + rps - 1) / rps;
  // workspace: fp32 partials O/l, then (max, sum) per (query, split, head)
  const size_t n_part = (size_t)nq * n_splits * p.n_heads;
  float* ws_o = ws;
  float* ws_ml = ws ? ws + n_part * p.d : nullptr;
  const size_t smem = attn_tc_smem_bytes();
  auto kfn = dense ? attn_tc<true> : attn_tc<false>;
  cudaError_t e = set_max_smem(reinterpret_cast<const void*>(kfn), smem);
  if (e != cudaSuccess) return e;
  dim3 grid(nq, n_splits, nhg);
  e = launch_pdl(kfn, grid, dim3(kThreads), smem, st, tq, reinterpret_cast<const uint8_t*>(cache.rows), cache.scale,
                 cache.cap, reinterpret_cast<const uint8_t*>(win.rows), win.scale, win.cap, idx, p.topk, q_pos0, T,
                 p.m, p.window, n_sel, p.n_heads, p.softmax_scale, p.rope_theta, sink, rps, n_splits,
                 reinterpret_cast<uint16_t*>(out), ws_o, ws_ml, err);
  if (e != cudaSuccess || n_splits == 1) return e;
  return launch_pdl(attn_merge_f32, dim3(nq, p.n_heads / 8), dim3(256), 0, st, (const float*)ws_o,
                    (const float*)ws_ml, n_splits, p.n_heads, sink, q_pos0, T, p.m, p.window, n_sel, dense ? 1 : 0,
                    rps, p.rope_theta, reinterpret_cast<uint16_t*>(out));
}

size_t attn_tc_workspace_bytes(const csa_params& p, int T, int n_sel, bool dense) {
  const int total = n_sel + p.window;
  const int rps = attn_tc_rows_per_split(total, p.n_heads / kHg, T, dense);
  const int n_splits = (total + rps - 1) / rps;
  if (n_splits == 1) return 0;
  const size_t n_part = (size_t)p.B * T * n_splits * p.n_heads;
  return n_part * (p.d + 2) * sizeof(float);
}

}  // namespace csa
