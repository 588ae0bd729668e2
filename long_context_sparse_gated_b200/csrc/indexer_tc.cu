// Lightning Indexer scores on the 5th-generation tensor cores (sm_100a).
//
// Qiaomu blog 混合注意力机制 / FP4量化感知训练 and kwkr.cn notes 3.4, 4.4: the
// indexer QK runs in FP4.  Here it runs as a block-scaled MXFP4 MMA
// (tcgen05.mma kind::mxf4, E2M1 operands, one UE8M0 scale per 32 elements):
//
//   D[s, h] = sum_c k[s, c] * q[h, c]       (A = 128 index keys, K-major,
//                                            B = the query's 64 heads)
//   I(t, s) = sum_h w_h * max(D[s, h], 0)   (epilogue, fp32, h = 0..63)
//
// Persistent, warp-specialised CTA (one per SM), 320 threads, walking
// stages of 256 entries (two 128-entry MMA tiles):
//   warp 0     TMA producer: per stage two 128x64 B key boxes (64B swizzle,
//              rows permuted by a 3-D view, see Stage) and the stage's 1 KB
//              of scales into a kStages-deep ring; per query (not per
//              stage) the 64x64 B query block and its scales into one of
//              two slots
//   warp 1     MMA issuer (one lane): per query, permutes the query scales
//              into the 32x16 B layout and copies them to TMEM; per stage,
//              copies the two tiles' key scales to TMEM (tcgen05.cp), issues
//              four K=64 MMAs (two per tile) into one of three TMEM
//              accumulator pairs, and commits twice: to the pair's "full"
//              barrier and to the stage's "empty" barrier, so the ring slot
//              goes back to the producer as soon as the MMAs have read it
//   warps 2-9  two epilogue warpgroups; warpgroup g takes tile g of every
//              stage: once the stage's MMAs are complete it tcgen05.ld's the
//              64 head columns of one entry per thread, frees the
//              accumulator, applies ReLU and the weighted head sum (four
//              independent partial sums), stores the fp32 score and
//              (optionally) counts the score's top 12 key bits into the
//              warpgroup's shared-memory histogram of the current query,
//              which is added to the global per-query histogram (the top-k
//              selector's starting point) when the warpgroup moves to
//              another query and at the end
// Two ways of walking the work, chosen by the host from the call's shape:
//   decode (T <= 4): a stage is 256 entries of one query (two 128-entry
//       MMA tiles, N = 64 heads); each CTA walks a contiguous range of
//       (query, stage) pairs, so the key stream it reads is sequential and
//       a long row is spread over many CTAs.  Stages past n_t are skipped.
//   prefill (T > 4): a stage is 128 entries of a pair of consecutive
//       queries of one sequence (one MMA tile with N = 128: both queries'
//       64 heads), so every key tile read from L2 serves two queries and
//       each MMA is twice as wide.  CTA b takes query pairs b, b + grid,
//       ... with all their visible stages, which balances the causal
//       (growing) rows over the CTAs.  Epilogue warpgroup g takes query g
//       of the pair.
// In both modes an accumulator is 128 TMEM columns and each epilogue
// warpgroup reads 64 of them per stage.
//
// Numerics: with MXFP4 inputs whose per-32 scales are >= 2^-2 and dyadic
// head weights, every partial sum is exactly representable in fp32 (the
// workloads check a bound), so the scores equal the exact scores.
#include <cuda.h>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace csa {

namespace {

constexpr int kStages = 10;
constexpr int kTileM = 128;   // entries per MMA tile
constexpr int kTiles = 2;     // MMA tiles per stage
constexpr int kStageKeys = kTileM * kTiles;     // 256 entries per stage
constexpr int kHeads = 64;    // index heads (N)
constexpr int kRowBytes = 64; // 128 E2M1 values
constexpr int kKeyBytes = kTileM * kRowBytes;   // 8192 per tile
constexpr int kQBytes = kHeads * kRowBytes;     // 4096
constexpr int kSfkBytes = kTileM * 4;           // 512 per tile (4 UE8M0 per row)
constexpr int kSfqBytes = kHeads * 4;           // 256

// A tile's 128 keys are loaded through a 3-D view of the key array, so that
// MMA row 32q + i holds key 4i + q (q < 4, i < 32).  With that order the
// keys' 512 contiguous scale bytes are already the 32-line x 16-byte block
// tcgen05.cp expects (line i = scale words of MMA rows i, 32+i, 64+i, 96+i),
// and no per-tile permutation is needed.
struct __align__(1024) Stage {
  uint8_t key[kTiles][kKeyBytes];   // 1024-aligned (64B-swizzle atoms are 512 B)
  uint32_t sfk[kTiles][kTileM];     // the stage's 256 scale words, in entry order
};

constexpr int kPair = 2;       // queries per stage in prefill mode

struct __align__(1024) QuerySlot {
  uint8_t q[kPair * kQBytes];         // one query (decode) or a pair (prefill)
  uint32_t sfq_raw[kPair * kHeads];
  uint32_t sfq[kTileM];     // permuted for tcgen05.cp (decode: rows 64..127 zero)
};

constexpr int kAcc = 3;         // TMEM accumulator pairs (one tile each per epilogue warpgroup)
constexpr int kEpiGroups = kTiles;  // epilogue warpgroup g takes tile g of every stage
constexpr int kHistBins = 4096; // score histogram bins (top 12 key bits)

struct Smem {
  Stage st[kStages];
  QuerySlot qs[2];
  uint32_t hist[kEpiGroups][kHistBins];  // per-warpgroup histogram of its current query
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t qfull[2];
  uint64_t qempty[2];
  uint64_t tfull[kAcc];
  uint64_t tempty[kAcc];
  uint32_t tmem_base;
  int abort;
};

// TMEM columns: accumulator a at 128 a (0..383): decode tile g at
// 128 a + 64 g, prefill query g at 128 a + 64 g; key scales 384 + 8 a + 4 g;
// query scales 408 + 4 slot.
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSfaCol = kAcc * kTiles * kHeads;
constexpr uint32_t kSfbCol = kSfaCol + 4 * kTiles * kAcc;

__device__ __forceinline__ int visible(const int32_t* q_pos0, int T, int m, int qi, int n_max) {
  const int bs = qi / T, tq = qi % T;
  const int64_t t = (int64_t)q_pos0[bs] + tq;
  int64_t n = (t + 1) / m;
  return (int)(n < n_max ? n : n_max);
}

static_assert(sizeof(Smem) + 1024 <= 232448, "shared memory per CTA");

constexpr int kThreadsTc = 64 + 128 * kEpiGroups;  // producer, MMA, 2 epilogue warpgroups

// Shape of one walking mode (see the header).
template <bool kPrefill>
struct Mode {
  static constexpr int kQn = kPrefill ? kPair : 1;          // queries per stage
  static constexpr int kT = kPrefill ? 1 : kTiles;          // MMA tiles per stage
  static constexpr int kKeys = kT * kTileM;                 // entries per stage
  static constexpr int kN = kQn * kHeads;                   // MMA N
  static constexpr uint32_t kStageTx = kT * (kKeyBytes + kSfkBytes);
  static constexpr uint32_t kQueryTx = kQn * (kQBytes + kSfqBytes);
};

// The stages one CTA walks, in order.  After next() returns true: q0 is
// the stage's first query, j its stage index within the row, nvis the
// visible entries of the stage's last query, and fresh is set when the
// query (pair) differs from the previous stage's.
template <bool kPrefill>
struct Walker;

// decode: a contiguous range of (query, 256-entry stage) pairs.  One 64-bit
// division at the start; afterwards a step is an increment, so the
// single-thread producer and MMA loops do not pay a division latency per
// stage.  visible() is re-read only when the query changes.
template <>
struct Walker<false> {
  int64_t t, end;
  int qi, jj, tpq;
  int q0 = -1, j = 0, nvis = 0;
  bool fresh = false;
  __device__ __forceinline__ Walker(int n_queries, int n_max) {
    tpq = (n_max + Mode<false>::kKeys - 1) / Mode<false>::kKeys;
    const int64_t n_units = (int64_t)n_queries * tpq;
    t = n_units * blockIdx.x / gridDim.x;
    end = n_units * (blockIdx.x + 1) / gridDim.x;
    qi = (int)(t / tpq);
    jj = (int)(t - (int64_t)qi * tpq);
  }
  __device__ __forceinline__ bool next(const int32_t* q_pos0, int T, int m, int n_max) {
    while (t < end) {
      const int q = qi, js = jj;
      ++t;
      if (++jj == tpq) { jj = 0; ++qi; }
      const bool nq = q != q0;
      if (nq) nvis = visible(q_pos0, T, m, q, n_max);
      if (js * Mode<false>::kKeys >= nvis) {
        if (nq) { q0 = q; fresh_pending = true; }
        continue;
      }
      fresh = nq || fresh_pending;
      fresh_pending = false;
      q0 = q;
      j = js;
      return true;
    }
    return false;
  }
  bool fresh_pending = false;
};

// prefill: query pairs b, b + grid, ... of the batch (pairs never cross a
// sequence), each with all of its visible 128-entry stages.
template <>
struct Walker<true> {
  int g, n_groups, gps;
  int q0 = 0, qn = 0, j = 0, nst = 0, nvis = 0;
  bool fresh = false;
  __device__ __forceinline__ Walker(int n_queries, int T) {
    gps = (T + kPair - 1) / kPair;
    n_groups = (n_queries / T) * gps;
    g = (int)blockIdx.x - (int)gridDim.x;
  }
  __device__ __forceinline__ bool next(const int32_t* q_pos0, int T, int m, int n_max) {
    if (++j < nst) {
      fresh = false;
      return true;
    }
    while (true) {
      g += gridDim.x;
      if (g >= n_groups) return false;
      const int bs = g / gps, tq = kPair * (g - bs * gps);
      q0 = bs * T + tq;
      qn = T - tq < kPair ? T - tq : kPair;
      nvis = visible(q_pos0, T, m, q0 + qn - 1, n_max);
      nst = (nvis + Mode<true>::kKeys - 1) / Mode<true>::kKeys;
      if (nst > 0) break;
    }
    j = 0;
    fresh = true;
    return true;
  }
};

template <bool kPrefill>
__device__ __forceinline__ Walker<kPrefill> make_walker(int n_queries, int T, int n_max) {
  if constexpr (kPrefill) return Walker<true>(n_queries, T);
  else return Walker<false>(n_queries, n_max);
}

template <bool kPrefill>
__global__ void __launch_bounds__(kThreadsTc, 1) index_scores_tc(
    const __grid_constant__ CUtensorMap tm_key, const __grid_constant__ CUtensorMap tm_q,
    const __grid_constant__ CUtensorMap tm_sfk, const __grid_constant__ CUtensorMap tm_sfq,
    const float* __restrict__ w, const int32_t* __restrict__ q_pos0, int T, int m, int64_t k_cap,
    int n_queries, int n_max, void* __restrict__ scores, int ld, int b16, uint32_t* __restrict__ hist,
    int32_t* __restrict__ err) {
  using M = Mode<kPrefill>;
  extern __shared__ uint8_t smem_raw[];
  Smem& S = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort = &S.abort;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      sm100::mbar_init(&S.full[i], 1);
      sm100::mbar_init(&S.empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      sm100::mbar_init(&S.qfull[i], 1);
      sm100::mbar_init(&S.qempty[i], 1);
    }
    for (int i = 0; i < kAcc; ++i) {
      sm100::mbar_init(&S.tfull[i], 1);
      sm100::mbar_init(&S.tempty[i], 4 * kEpiGroups);
    }
    S.abort = 0;
    sm100::fence_mbar_init();
  }
  if (warp == 1) {
    sm100::tmem_alloc(&S.tmem_base, kTmemCols);
    sm100::tmem_relinquish();
  }
  sm100::tc_fence_before();
  __syncthreads();
  sm100::tc_fence_after();
  const uint32_t tmem = S.tmem_base;
  pdl_wait();  // inputs may come from the previous kernel on the stream

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      sm100::prefetch_tmap(&tm_key);
      sm100::prefetch_tmap(&tm_q);
      sm100::prefetch_tmap(&tm_sfk);
      sm100::prefetch_tmap(&tm_sfq);
      uint32_t it = 0, nq = 0;
      int bs = 0;
      const uint64_t key_policy = sm100::l2_policy_evict_first();
      auto wk = make_walker<kPrefill>(n_queries, T, n_max);
      while (wk.next(q_pos0, T, m, n_max)) {
        if (wk.fresh) {  // the stage's query (pair): 64 heads each, once per query
          bs = wk.q0 / T;
          const int sl = nq & 1;
          if (!sm100::mbar_wait(&S.qempty[sl], ((nq >> 1) & 1) ^ 1, abort)) break;
          sm100::mbar_arrive_expect_tx(&S.qfull[sl], M::kQueryTx);
          sm100::tma_load_2d(S.qs[sl].q, &tm_q, &S.qfull[sl], 0, wk.q0 * kHeads);
          sm100::tma_load_1d(S.qs[sl].sfq_raw, &tm_sfq, &S.qfull[sl], wk.q0 * kHeads);
          ++nq;
        }
        const int s = it % kStages;
        const uint32_t ph = (it / kStages) & 1;
        if (!sm100::mbar_wait(&S.empty[s], ph ^ 1, abort)) break;
        Stage& st = S.st[s];
        sm100::mbar_arrive_expect_tx(&S.full[s], M::kStageTx);
        const int64_t row = (int64_t)bs * k_cap + (int64_t)wk.j * M::kKeys;
#pragma unroll
        for (int g = 0; g < M::kT; ++g) {
          const int32_t y = (int32_t)(row / 4) + g * (kTileM / 4);
          // decode streams every key once: evict-first keeps the scores the
          // selector reads next in L2; prefill re-reads a sequence's keys
          if (kPrefill) sm100::tma_load_3d(st.key[g], &tm_key, &S.full[s], 0, y, 0);
          else sm100::tma_load_3d_hint(st.key[g], &tm_key, &S.full[s], 0, y, 0, key_policy);
        }
        sm100::tma_load_1d(st.sfk, &tm_sfk, &S.full[s], (int32_t)row);
        ++it;
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer (one lane) ----------------
    if (lane == 0) {
      uint32_t it = 0, nq = 0;
      int sl = 0;
      auto wk = make_walker<kPrefill>(n_queries, T, n_max);
      while (wk.next(q_pos0, T, m, n_max)) {
        if (wk.fresh) {
          // the previous query's slot is free once its MMAs complete
          if (nq > 0) sm100::tc_commit(&S.qempty[sl]);
          sl = nq & 1;
          if (!sm100::mbar_wait(&S.qfull[sl], (nq >> 1) & 1, abort)) break;
          // query scales: MMA column n's word goes to line n % 32, word n / 32
          QuerySlot& qs = S.qs[sl];
#pragma unroll 4
          for (int l = 0; l < 32; ++l)
            reinterpret_cast<uint4*>(qs.sfq)[l] =
                kPrefill ? make_uint4(qs.sfq_raw[l], qs.sfq_raw[l + 32], qs.sfq_raw[l + 64], qs.sfq_raw[l + 96])
                         : make_uint4(qs.sfq_raw[l], qs.sfq_raw[l + 32], 0u, 0u);
          sm100::fence_proxy_async_smem();
          sm100::tc_fence_after();
          sm100::tc_cp_32x128b_warpx4(tmem + kSfbCol + 4 * sl, sm100::smem_desc(sm100::smem_u32(qs.sfq), 0, 128, 0));
          ++nq;
        }
        const int s = it % kStages;
        const uint32_t ph = (it / kStages) & 1;
        const int acc = it % kAcc;
        const uint32_t aph = (it / kAcc) & 1;
        if (!sm100::mbar_wait_poll(&S.tempty[acc], aph ^ 1, abort) || !sm100::mbar_wait_poll(&S.full[s], ph, abort))
          break;
        sm100::tc_fence_after();
        Stage& st = S.st[s];
        const uint32_t sfb_col = tmem + kSfbCol + 4 * sl;
        const uint32_t qa = sm100::smem_u32(S.qs[sl].q);
#pragma unroll
        for (int g = 0; g < M::kT; ++g) {
          const uint32_t d_col = tmem + acc * kTiles * kHeads + g * kHeads;
          const uint32_t sfa_col = tmem + kSfaCol + 4 * (acc * kTiles + g);
          sm100::tc_cp_32x128b_warpx4(sfa_col, sm100::smem_desc(sm100::smem_u32(st.sfk[g]), 0, 128, 0));
          const uint32_t ka = sm100::smem_u32(st.key[g]);
#pragma unroll
          for (int kk = 0; kk < 2; ++kk) {
            // K elements [64kk, 64kk+64) = bytes [32kk, 32kk+32) of every row
            const uint64_t adesc = sm100::smem_desc(ka + 32 * kk, 16, 512, 4);
            const uint64_t bdesc = sm100::smem_desc(qa + 32 * kk, 16, 512, 4);
            sm100::mma_mxf4(d_col, adesc, bdesc, sm100::idesc_mxf4(kTileM, M::kN, 2 * kk, 2 * kk), sfa_col,
                            sfb_col, kk);
          }
        }
        // completion: the accumulator is ready for the epilogue, and the
        // stage's shared memory goes back to the producer
        sm100::tc_commit(&S.tfull[acc]);
        sm100::tc_commit(&S.empty[s]);
        ++it;
      }
    }
  } else {
    // ---------------- epilogue (warps 2..9: two warpgroups) ----------------
    const int eg = (warp - 2) >> 2;  // warpgroup: tile (decode) or query (prefill) eg of every stage
    const int quad = warp & 3;       // TMEM lane quadrant this warp may access
    // TMEM lane 32*quad + lane holds key 4*lane + quad of the tile
    const int key_in_tile = 4 * lane + quad;
    const int et = threadIdx.x - 64 - 128 * eg;  // 0..127 within the warpgroup
    uint32_t* sh = S.hist[eg];
    // add the warpgroup's histogram of query q to the global one and clear it
    auto flush = [&](int q) {
      sm100::named_bar_sync(1 + eg, 128);
      for (int b = et; b < kHistBins; b += 128) {
        const uint32_t v = sh[b];
        if (v) {
          atomicAdd(hist + (int64_t)q * kScoreHistBins + b, v);
          sh[b] = 0u;
        }
      }
      sm100::named_bar_sync(1 + eg, 128);
    };
    if (hist) {
      for (int b = et; b < kHistBins; b += 128) sh[b] = 0u;
      sm100::named_bar_sync(1 + eg, 128);
    }
    uint32_t it = 0;
    int wq = -1, n_t = 0;
    float wv[kHeads];
    auto wk = make_walker<kPrefill>(n_queries, T, n_max);
    while (wk.next(q_pos0, T, m, n_max)) {
      const uint32_t my = it++;
      const int acc = my % kAcc;
      const uint32_t aph = (my / kAcc) & 1;
      if (wk.fresh) {  // this warpgroup's query changed: flush, load its head weights
        if (hist && wq >= 0) flush(wq);
        int q = wk.q0;
        n_t = wk.nvis;
        if constexpr (kPrefill) {
          q = eg < wk.qn ? wk.q0 + eg : -1;
          n_t = q >= 0 ? visible(q_pos0, T, m, q, n_max) : 0;
        }
        if (q >= 0) {
          const float4* wp = reinterpret_cast<const float4*>(w + (int64_t)q * kHeads);
#pragma unroll
          for (int h4 = 0; h4 < kHeads / 4; ++h4) {
            const float4 v = __ldg(wp + h4);
            wv[4 * h4] = v.x; wv[4 * h4 + 1] = v.y; wv[4 * h4 + 2] = v.z; wv[4 * h4 + 3] = v.w;
          }
        }
        wq = q;
      }
      int ok = 1;
      if (lane == 0) ok = sm100::mbar_wait_poll(&S.tfull[acc], aph, abort);
      // no break on a failed wait: every warp of the warpgroup keeps walking
      // the same stages so that the histogram flushes' named barriers match;
      // after an abort every wait returns at once and no work is done
      if (!__shfl_sync(0xffffffffu, ok, 0)) continue;
      sm100::tc_fence_after();
      // the 64 head columns in two halves: the second half's load is in
      // flight while the first half is summed
      uint32_t d[64];
      auto grp = [&](int g) -> uint32_t(&)[16] { return *reinterpret_cast<uint32_t(*)[16]>(d + 16 * g); };
      const uint32_t base = tmem + ((uint32_t)(quad * 32) << 16) + (acc * kTiles + eg) * kHeads;
      sm100::tmem_ld_x16(base + 0, grp(0));
      sm100::tmem_ld_x16(base + 16, grp(1));
      sm100::tmem_ld_wait();
      sm100::tmem_pin16(grp(0));
      sm100::tmem_pin16(grp(1));
      sm100::tmem_ld_x16(base + 32, grp(2));
      sm100::tmem_ld_x16(base + 48, grp(3));
      // four independent partial sums (every partial sum of these
      // scores is exact, so the grouping does not change the result)
      float p4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int h = 0; h < kHeads / 2; ++h) p4[h & 3] = fmaf(wv[h], fmaxf(__uint_as_float(d[h]), 0.f), p4[h & 3]);
      sm100::tmem_ld_wait();
      sm100::tmem_pin16(grp(2));
      sm100::tmem_pin16(grp(3));
      sm100::tc_fence_before();
      __syncwarp();
      if (lane == 0) sm100::mbar_arrive(&S.tempty[acc]);
#pragma unroll
      for (int h = kHeads / 2; h < kHeads; ++h) p4[h & 3] = fmaf(wv[h], fmaxf(__uint_as_float(d[h]), 0.f), p4[h & 3]);
      const float sc = (p4[0] + p4[1]) + (p4[2] + p4[3]);
      const int s_idx = wk.j * M::kKeys + (kPrefill ? 0 : eg * kTileM) + key_in_tile;
      if (s_idx < n_t) {
        // fp32 score, or rounded to BF16 (nearest even) for the BF16
        // selector; the histogram bins the key the selector will rank
        if (b16) {
          const uint32_t bits = f32_to_bf16_bits(sc);
          reinterpret_cast<uint16_t*>(scores)[(int64_t)wq * ld + s_idx] = (uint16_t)bits;
          if (hist) atomicAdd(sh + score_bin16(bits), 1u);
        } else {
          reinterpret_cast<float*>(scores)[(int64_t)wq * ld + s_idx] = sc;
          if (hist) atomicAdd(sh + score_bin(sc), 1u);
        }
      }
    }
    if (hist && wq >= 0) flush(wq);
  }

  pdl_trigger();
  sm100::tc_fence_before();
  __syncthreads();
  if (S.abort && threadIdx.x == 0) raise_err(err, CSA_DEV_ERR_TIMEOUT);
  if (warp == 1) {
    sm100::tc_fence_after();
    sm100::tmem_dealloc(tmem, kTmemCols);
  }
}

// ---- host side ----------------------------------------------------------------

}  // namespace

bool index_scores_tc_supported(const csa_params& p, int64_t k_cap, const void* q_idx, const uint8_t* q_sf,
                               const void* k_idx, const uint8_t* k_sf) {
  if (p.idx_fmt != CSA_IDX_MXFP4 || p.n_idx_heads != kHeads || p.idx_dim != 128) return false;
  if (k_cap % 4 != 0) return false;  // scale rows must start 16-byte aligned for TMA
  return tensor_maps_available();
}

cudaError_t launch_index_scores_tc(const csa_params& p, const void* q_idx, const uint8_t* q_sf, const float* w,
                                   const void* k_idx, const uint8_t* k_sf, int64_t k_cap,
                                   const int32_t* q_pos0, int T, void* scores, int ld, uint32_t* hist,
                                   int n_max, int32_t* err, cudaStream_t st) {
  const int nq = p.B * T;
  // prefill (more than 4 queries per sequence): query pairs, 128-entry stages
  const bool prefill = T > 4;
  const int qn = prefill ? kPair : 1;
  const int stage_keys = prefill ? kTileM : kStageKeys;
  CUtensorMap tk, tq, tsk, tsq;
  const uint64_t key_rows = (uint64_t)p.B * (uint64_t)k_cap;
  {
    // (byte, i, q) -> byte + 256 i + 64 q: key row 4i + q lands in shared
    // row 32q + (i mod 32)
    uint64_t dims[3] = {kRowBytes, key_rows / 4, 4};
    uint64_t str[2] = {4 * kRowBytes, kRowBytes};
    uint32_t box[3] = {kRowBytes, kTileM / 4, 4};
    if (!encode_tensor_map(&tk, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, k_idx, dims, str, box, CU_TENSOR_MAP_SWIZZLE_64B))
      return cudaErrorInvalidValue;
  }
  {
    uint64_t dims[2] = {kRowBytes, (uint64_t)nq * kHeads};
    uint64_t str[1] = {kRowBytes};
    uint32_t box[2] = {kRowBytes, (uint32_t)(qn * kHeads)};
    if (!encode_tensor_map(&tq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, q_idx, dims, str, box, CU_TENSOR_MAP_SWIZZLE_64B))
      return cudaErrorInvalidValue;
  }
  {
    uint64_t dims[1] = {key_rows};
    uint64_t str[1] = {4};
    uint32_t box[1] = {(uint32_t)stage_keys};
    if (!encode_tensor_map(&tsk, CU_TENSOR_MAP_DATA_TYPE_UINT32, 1, k_sf, dims, str, box, CU_TENSOR_MAP_SWIZZLE_NONE))
      return cudaErrorInvalidValue;
  }
  {
    uint64_t dims[1] = {(uint64_t)nq * kHeads};
    uint64_t str[1] = {4};
    uint32_t box[1] = {(uint32_t)(qn * kHeads)};
    if (!encode_tensor_map(&tsq, CU_TENSOR_MAP_DATA_TYPE_UINT32, 1, q_sf, dims, str, box, CU_TENSOR_MAP_SWIZZLE_NONE))
      return cudaErrorInvalidValue;
  }
  const int sms = sm_count();
  int64_t units;
  if (prefill) {
    units = (int64_t)p.B * ((T + kPair - 1) / kPair);  // query pairs
  } else {
    const int tpq = (n_max + kStageKeys - 1) / kStageKeys;
    units = (int64_t)nq * tpq;
  }
  const int grid = (int)(units < sms ? units : sms);
  if (grid == 0) return cudaSuccess;
  const size_t smem = sizeof(Smem) + 1024;
  auto kfn = prefill ? index_scores_tc<true> : index_scores_tc<false>;
  cudaError_t e = set_max_smem(reinterpret_cast<const void*>(kfn), smem);
  if (e != cudaSuccess) return e;
  e = launch_pdl(kfn, dim3(grid), dim3(kThreadsTc), smem, st, tk, tq, tsk, tsq, w, q_pos0, T, p.m, k_cap, nq,
                 n_max, scores, ld, p.score_fmt == CSA_SCORE_BF16 ? 1 : 0, hist, err);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace csa
