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
// Each CTA walks a contiguous range of (query, 256-entry block) stages, so
// the key stream it reads is sequential.  Stages past a query's n_t are
// skipped.
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
constexpr uint32_t kStageTx = kTiles * (kKeyBytes + kSfkBytes);
constexpr uint32_t kQueryTx = kQBytes + kSfqBytes;

// A tile's 128 keys are loaded through a 3-D view of the key array, so that
// MMA row 32q + i holds key 4i + q (q < 4, i < 32).  With that order the
// keys' 512 contiguous scale bytes are already the 32-line x 16-byte block
// tcgen05.cp expects (line i = scale words of MMA rows i, 32+i, 64+i, 96+i),
// and no per-tile permutation is needed.
struct __align__(1024) Stage {
  uint8_t key[kTiles][kKeyBytes];   // 1024-aligned (64B-swizzle atoms are 512 B)
  uint32_t sfk[kTiles][kTileM];     // the stage's 256 scale words, in entry order
};

struct __align__(1024) QuerySlot {
  uint8_t q[kQBytes];
  uint32_t sfq_raw[kHeads];
  uint32_t sfq[kTileM];     // permuted for tcgen05.cp; rows 64..127 zero
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

// TMEM columns: accumulator pair a, tile g at 128 a + 64 g (0..383); key
// scales 384 + 8 a + 4 g; query scales 408 + 4 slot.
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSfaCol = kAcc * kTiles * kHeads;
constexpr uint32_t kSfbCol = kSfaCol + 4 * kTiles * kAcc;

__device__ __forceinline__ int visible(const int32_t* q_pos0, int T, int m, int qi, int n_max) {
  const int bs = qi / T, tq = qi % T;
  const int64_t t = (int64_t)q_pos0[bs] + tq;
  int64_t n = (t + 1) / m;
  return (int)(n < n_max ? n : n_max);
}

// visible() of the current query, re-read only when the query changes: the
// single producer thread must not pay a global-load latency per tile.
struct VisibleCache {
  int qi = -1, n = 0;
  __device__ __forceinline__ int get(const int32_t* q_pos0, int T, int m, int q, int n_max) {
    if (q != qi) {
      qi = q;
      n = visible(q_pos0, T, m, q, n_max);
    }
    return n;
  }
};

constexpr int kThreadsTc = 64 + 128 * kEpiGroups;  // producer, MMA, 2 epilogue warpgroups

// Walks the CTA's tile range as (query, block) pairs.  One 64-bit division
// at the start; afterwards a step is an increment, so the single-thread
// producer and MMA loops do not pay a division latency per tile.
struct TileCursor {
  int64_t t, end;
  int qi, j, tpq;
  __device__ __forceinline__ TileCursor(int64_t begin, int64_t e, int tiles_per_query)
      : t(begin), end(e), tpq(tiles_per_query) {
    qi = (int)(begin / tiles_per_query);
    j = (int)(begin - (int64_t)qi * tiles_per_query);
  }
  __device__ __forceinline__ bool more() const { return t < end; }
  __device__ __forceinline__ void next() {
    ++t;
    if (++j == tpq) { j = 0; ++qi; }
  }
};

__global__ void __launch_bounds__(kThreadsTc, 1) index_scores_tc(
    const __grid_constant__ CUtensorMap tm_key, const __grid_constant__ CUtensorMap tm_q,
    const __grid_constant__ CUtensorMap tm_sfk, const __grid_constant__ CUtensorMap tm_sfq,
    const float* __restrict__ w, const int32_t* __restrict__ q_pos0, int T, int m, int64_t k_cap,
    int n_queries, int n_max, void* __restrict__ scores, int ld, int b16, uint32_t* __restrict__ hist,
    int32_t* __restrict__ err) {
  extern __shared__ uint8_t smem_raw[];
  Smem& S = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tpq = (n_max + kStageKeys - 1) / kStageKeys;  // stages per query
  const int64_t n_tiles = (int64_t)n_queries * tpq;
  const int64_t t_begin = n_tiles * blockIdx.x / gridDim.x;
  const int64_t t_end = n_tiles * (blockIdx.x + 1) / gridDim.x;
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
      int cur_q = -1;
      VisibleCache vc;
      int bs = 0;
      for (TileCursor c(t_begin, t_end, tpq); c.more(); c.next()) {
        const int qi = c.qi, j = c.j;
        if (j * kStageKeys >= vc.get(q_pos0, T, m, qi, n_max)) continue;
        if (qi != cur_q) {  // the query's 64 heads, once per query
          bs = qi / T;
          const int sl = nq & 1;
          if (!sm100::mbar_wait(&S.qempty[sl], ((nq >> 1) & 1) ^ 1, abort)) break;
          sm100::mbar_arrive_expect_tx(&S.qfull[sl], kQueryTx);
          sm100::tma_load_2d(S.qs[sl].q, &tm_q, &S.qfull[sl], 0, qi * kHeads);
          sm100::tma_load_1d(S.qs[sl].sfq_raw, &tm_sfq, &S.qfull[sl], qi * kHeads);
          cur_q = qi;
          ++nq;
        }
        const int s = it % kStages;
        const uint32_t ph = (it / kStages) & 1;
        if (!sm100::mbar_wait(&S.empty[s], ph ^ 1, abort)) break;
        Stage& st = S.st[s];
        sm100::mbar_arrive_expect_tx(&S.full[s], kStageTx);
        const int64_t row = (int64_t)bs * k_cap + (int64_t)j * kStageKeys;
        sm100::tma_load_3d(st.key[0], &tm_key, &S.full[s], 0, (int32_t)(row / 4), 0);
        sm100::tma_load_3d(st.key[1], &tm_key, &S.full[s], 0, (int32_t)(row / 4) + kTileM / 4, 0);
        sm100::tma_load_1d(st.sfk, &tm_sfk, &S.full[s], (int32_t)row);
        ++it;
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer (one lane) ----------------
    if (lane == 0) {
      uint32_t it = 0, nq = 0;
      int cur_q = -1, sl = 0;
      VisibleCache vc;
      for (TileCursor c(t_begin, t_end, tpq); c.more(); c.next()) {
        const int qi = c.qi, j = c.j;
        if (j * kStageKeys >= vc.get(q_pos0, T, m, qi, n_max)) continue;
        if (qi != cur_q) {
          // the previous query's slot is free once its MMAs complete
          if (cur_q >= 0) sm100::tc_commit(&S.qempty[sl]);
          sl = nq & 1;
          if (!sm100::mbar_wait(&S.qfull[sl], (nq >> 1) & 1, abort)) break;
          // query scales: head h's word goes to line h%32, slot h/32
          QuerySlot& qs = S.qs[sl];
#pragma unroll 4
          for (int l = 0; l < 32; ++l)
            reinterpret_cast<uint4*>(qs.sfq)[l] = make_uint4(qs.sfq_raw[l], qs.sfq_raw[l + 32], 0u, 0u);
          sm100::fence_proxy_async_smem();
          sm100::tc_fence_after();
          sm100::tc_cp_32x128b_warpx4(tmem + kSfbCol + 4 * sl, sm100::smem_desc(sm100::smem_u32(qs.sfq), 0, 128, 0));
          cur_q = qi;
          ++nq;
        }
        const int s = it % kStages;
        const uint32_t ph = (it / kStages) & 1;
        const int acc = it % kAcc;
        const uint32_t aph = (it / kAcc) & 1;
        if (!sm100::mbar_wait(&S.tempty[acc], aph ^ 1, abort) || !sm100::mbar_wait(&S.full[s], ph, abort)) break;
        sm100::tc_fence_after();
        Stage& st = S.st[s];
        const uint32_t sfb_col = tmem + kSfbCol + 4 * sl;
        const uint32_t qa = sm100::smem_u32(S.qs[sl].q);
#pragma unroll
        for (int g = 0; g < kTiles; ++g) {
          const uint32_t d_col = tmem + (acc * kTiles + g) * kHeads;
          const uint32_t sfa_col = tmem + kSfaCol + 4 * (acc * kTiles + g);
          sm100::tc_cp_32x128b_warpx4(sfa_col, sm100::smem_desc(sm100::smem_u32(st.sfk[g]), 0, 128, 0));
          const uint32_t ka = sm100::smem_u32(st.key[g]);
#pragma unroll
          for (int kk = 0; kk < 2; ++kk) {
            // K elements [64kk, 64kk+64) = bytes [32kk, 32kk+32) of every row
            const uint64_t adesc = sm100::smem_desc(ka + 32 * kk, 16, 512, 4);
            const uint64_t bdesc = sm100::smem_desc(qa + 32 * kk, 16, 512, 4);
            sm100::mma_mxf4(d_col, adesc, bdesc, sm100::idesc_mxf4(kTileM, kHeads, 2 * kk, 2 * kk), sfa_col,
                            sfb_col, kk);
          }
        }
        // completion: the accumulator pair is ready for the epilogue, and
        // the stage's shared memory goes back to the producer
        sm100::tc_commit(&S.tfull[acc]);
        sm100::tc_commit(&S.empty[s]);
        ++it;
      }
    }
  } else {
    // ---------------- epilogue (warps 2..9: two warpgroups) ----------------
    const int eg = (warp - 2) >> 2;  // warpgroup: tile eg of every stage
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
    int wq = -1;
    float wv[kHeads];
    VisibleCache vc;
    for (TileCursor c(t_begin, t_end, tpq); c.more(); c.next()) {
      const int qi = c.qi, j = c.j;
      const int n_t = vc.get(q_pos0, T, m, qi, n_max);
      if (j * kStageKeys >= n_t) continue;
      const uint32_t my = it++;
      const int acc = my % kAcc;
      const uint32_t aph = (my / kAcc) & 1;
      if (qi != wq) {  // head weights of this tile's query, kept in registers
        if (hist && wq >= 0) flush(wq);
        const float4* wp = reinterpret_cast<const float4*>(w + (int64_t)qi * kHeads);
#pragma unroll
        for (int h4 = 0; h4 < kHeads / 4; ++h4) {
          const float4 v = __ldg(wp + h4);
          wv[4 * h4] = v.x; wv[4 * h4 + 1] = v.y; wv[4 * h4 + 2] = v.z; wv[4 * h4 + 3] = v.w;
        }
        wq = qi;
      }
      int ok = 1;
      if (lane == 0) ok = sm100::mbar_wait(&S.tfull[acc], aph, abort);
      // no break on a failed wait: every warp of the warpgroup keeps walking
      // the same tiles so that the histogram flushes' named barriers match;
      // after an abort every wait returns at once and no work is done
      if (!__shfl_sync(0xffffffffu, ok, 0)) continue;
      sm100::tc_fence_after();
      uint32_t d[64];
      const uint32_t base = tmem + ((uint32_t)(quad * 32) << 16) + (acc * kTiles + eg) * kHeads;
      sm100::tmem_ld_x16(base + 0, *reinterpret_cast<uint32_t(*)[16]>(d + 0));
      sm100::tmem_ld_x16(base + 16, *reinterpret_cast<uint32_t(*)[16]>(d + 16));
      sm100::tmem_ld_x16(base + 32, *reinterpret_cast<uint32_t(*)[16]>(d + 32));
      sm100::tmem_ld_x16(base + 48, *reinterpret_cast<uint32_t(*)[16]>(d + 48));
      sm100::tmem_ld_wait();
      sm100::tc_fence_before();
      __syncwarp();
      if (lane == 0) sm100::mbar_arrive(&S.tempty[acc]);
      // four independent partial sums (every partial sum of these
      // scores is exact, so the grouping does not change the result)
      float p4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int h = 0; h < kHeads; ++h) p4[h & 3] = fmaf(wv[h], fmaxf(__uint_as_float(d[h]), 0.f), p4[h & 3]);
      const float sc = (p4[0] + p4[1]) + (p4[2] + p4[3]);
      const int s_idx = j * kStageKeys + eg * kTileM + key_in_tile;
      if (s_idx < n_t) {
        // fp32 score, or rounded to BF16 (nearest even) for the BF16
        // selector; the histogram bins the key the selector will rank
        if (b16) {
          const uint32_t bits = f32_to_bf16_bits(sc);
          reinterpret_cast<uint16_t*>(scores)[(int64_t)qi * ld + s_idx] = (uint16_t)bits;
          if (hist) atomicAdd(sh + score_bin16(bits), 1u);
        } else {
          reinterpret_cast<float*>(scores)[(int64_t)qi * ld + s_idx] = sc;
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

bool make_map(CUtensorMap* map, CUtensorMapDataType dt, int rank, const void* base, const uint64_t* dims,
              const uint64_t* strides_bytes, const uint32_t* box, CUtensorMapSwizzle sw) {
  EncodeFn f = encode_fn();
  if (!f) return false;
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = f(map, dt, (cuuint32_t)rank, const_cast<void*>(base), (const cuuint64_t*)dims,
                 (const cuuint64_t*)strides_bytes, (const cuuint32_t*)box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                 CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace

bool index_scores_tc_supported(const csa_params& p, int64_t k_cap, const void* q_idx, const uint8_t* q_sf,
                               const void* k_idx, const uint8_t* k_sf) {
  if (p.idx_fmt != CSA_IDX_MXFP4 || p.n_idx_heads != kHeads || p.idx_dim != 128) return false;
  if (k_cap % 4 != 0) return false;  // scale rows must start 16-byte aligned for TMA
  return encode_fn() != nullptr;
}

cudaError_t launch_index_scores_tc(const csa_params& p, const void* q_idx, const uint8_t* q_sf, const float* w,
                                   const void* k_idx, const uint8_t* k_sf, int64_t k_cap,
                                   const int32_t* q_pos0, int T, void* scores, int ld, uint32_t* hist,
                                   int n_max, int32_t* err, cudaStream_t st) {
  const int nq = p.B * T;
  CUtensorMap tk, tq, tsk, tsq;
  const uint64_t key_rows = (uint64_t)p.B * (uint64_t)k_cap;
  {
    // (byte, i, q) -> byte + 256 i + 64 q: key row 4i + q lands in shared
    // row 32q + (i mod 32)
    uint64_t dims[3] = {kRowBytes, key_rows / 4, 4};
    uint64_t str[2] = {4 * kRowBytes, kRowBytes};
    uint32_t box[3] = {kRowBytes, kTileM / 4, 4};
    if (!make_map(&tk, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, k_idx, dims, str, box, CU_TENSOR_MAP_SWIZZLE_64B))
      return cudaErrorInvalidValue;
  }
  {
    uint64_t dims[2] = {kRowBytes, (uint64_t)nq * kHeads};
    uint64_t str[1] = {kRowBytes};
    uint32_t box[2] = {kRowBytes, kHeads};
    if (!make_map(&tq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, q_idx, dims, str, box, CU_TENSOR_MAP_SWIZZLE_64B))
      return cudaErrorInvalidValue;
  }
  {
    uint64_t dims[1] = {key_rows};
    uint64_t str[1] = {4};
    uint32_t box[1] = {kStageKeys};
    if (!make_map(&tsk, CU_TENSOR_MAP_DATA_TYPE_UINT32, 1, k_sf, dims, str, box, CU_TENSOR_MAP_SWIZZLE_NONE))
      return cudaErrorInvalidValue;
  }
  {
    uint64_t dims[1] = {(uint64_t)nq * kHeads};
    uint64_t str[1] = {4};
    uint32_t box[1] = {kHeads};
    if (!make_map(&tsq, CU_TENSOR_MAP_DATA_TYPE_UINT32, 1, q_sf, dims, str, box, CU_TENSOR_MAP_SWIZZLE_NONE))
      return cudaErrorInvalidValue;
  }
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int tpq = (n_max + kStageKeys - 1) / kStageKeys;
  const int64_t tiles = (int64_t)nq * tpq;
  const int grid = (int)(tiles < sms ? tiles : sms);
  if (grid == 0) return cudaSuccess;
  const size_t smem = sizeof(Smem) + 1024;
  cudaError_t e = cudaFuncSetAttribute(index_scores_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  e = launch_pdl(index_scores_tc, dim3(grid), dim3(kThreadsTc), smem, st, tk, tq, tsk, tsq, w, q_pos0, T, p.m, k_cap,
                 nq, n_max, scores, ld, p.score_fmt == CSA_SCORE_BF16 ? 1 : 0, hist, err);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace csa
