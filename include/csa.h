/*
 * csa.h -- C ABI of the B200 (sm_100a) CSA/HCA hot-path library, libcsa.so.
 *
 * DeepSeek-V4's hybrid compressed attention, as the public write-ups of the
 * DeepSeek-V4 technical report describe it:
 *
 *   csa_compress / hca_compress  gated two-stream token compressor (m = 4 for
 *                                CSA, m = 128 for HCA), RMSNorm, partial
 *                                RoPE, packed into the mixed FP8/BF16 layout
 *   csa_index_topk               Lightning Indexer (FP4 block-scaled QK,
 *                                ReLU-weighted head sum) + exact top-k
 *   csa_sparse_attn              MQA over the selected entries + sliding
 *                                window + attention sink, inverse RoPE
 *   hca_dense_attn               the same attention over every entry
 *
 * Sources, by page title and section:
 *   [kwkr]    kwkr.cn DeepSeek-V4 notes, 3.1 CSA 的工作方式, 3.2 HCA 的工作方式,
 *             3.3 层间排布与滑窗补充, 3.4 两个降开销的设计, 4.4 FP4 QAT 与 KV Cache 层级
 *   [Qiaomu]  乔木博客 "DeepSeek-V4论文解析：百万上下文、水平接近闭源模型是如何做到的？",
 *             混合注意力机制, FP4量化感知训练, 训练配置
 *   [WeChat]  未来科技 article on DeepSeek-V4 (cdjax.com), 1.1 混合注意力
 *   [PACMAN]  "DeepSeek-V4 技术报告分享" talk notes (10100.com), 3.1 CSA, 3.2 HCA
 *   [fengweifeng] "DeepSeek-V4: Towards Highly Efficient Million-Token Context
 *             Intelligence" notes, 2. 技术实现与架构细节 (inverse RoPE offset -i)
 *
 * Conventions for every call
 * --------------------------
 * - Pointers are DEVICE pointers unless stated otherwise; `params` is a HOST
 *   pointer read only during the call.  `stream` is a cudaStream_t passed as
 *   void* (NULL = the legacy default stream).  Every call only enqueues work
 *   on `stream`; nothing synchronises and nothing is allocated: the caller
 *   owns every buffer, including the workspace.  Calls hold no global
 *   mutable state and are re-entrant.
 * - Every array is C-contiguous.  The caller keeps buffers alive until the
 *   enqueued work completes.
 * - Return value: host-side validation only (csa_status).  Nothing is
 *   launched when it is not CSA_OK.  Anomalies found on the device (an index
 *   out of range, a token outside the stream buffer) are OR-ed as
 *   CSA_DEV_ERR_* bits into *err (nullable) and the offending item is
 *   skipped; the device never traps.
 * - Every pointer must be 16-byte aligned (CSA_ERR_ALIGN).
 *
 * Storage formats
 * ---------------
 * KV row, CSA_KV_FP8_BF16 ([WeChat 1.1]: RoPE dims BF16, other dims FP8):
 *     bytes [0, d-r)      E4M3 codes of the non-RoPE dims (value = code*scale)
 *     bytes [d-r, d+r)    r BF16 values of the RoPE dims
 *   row_bytes = d + r (576 for d = 512, r = 64); one fp32 scale per row in a
 *   separate array.  CSA_KV_F32: d floats per row (row_bytes = 4d), no scale.
 * Index key / index query, CSA_IDX_MXFP4 (OCP MX, E2M1 elements + UE8M0 scale
 *   per 32): idx_dim/2 bytes, element 2i in the low nibble of byte i, plus
 *   idx_dim/32 scale bytes in a separate array.  CSA_IDX_F32: idx_dim floats.
 * Activations (streams, queries, outputs), CSA_ACT_BF16 or CSA_ACT_F32.
 */
#ifndef CSA_H_
#define CSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes (return values) ------------------------------------- */
typedef int32_t csa_status;
#define CSA_OK 0
#define CSA_ERR_INVALID -1     /* null pointer, bad size or count            */
#define CSA_ERR_UNSUPPORTED -2 /* shape/format outside the supported set     */
#define CSA_ERR_ALIGN -3       /* a pointer is not 16-byte aligned           */
#define CSA_ERR_WORKSPACE -4   /* ws too small (see the *_workspace_bytes)   */
#define CSA_ERR_LAUNCH -5      /* a kernel launch failed (cudaGetLastError)  */

/* ---- device anomaly bits, OR-ed into *err ------------------------------ */
#define CSA_DEV_ERR_INDEX 1  /* a top-k index >= visible entries or < -1   */
#define CSA_DEV_ERR_RANGE 2  /* a token/entry range outside its buffer     */
#define CSA_DEV_ERR_TIMEOUT 4 /* a bounded on-chip wait gave up (no hang)  */

/* ---- formats ------------------------------------------------------------ */
#define CSA_KV_F32 0
#define CSA_KV_FP8_BF16 1
#define CSA_IDX_F32 0
#define CSA_IDX_MXFP4 1
#define CSA_ACT_F32 0
#define CSA_ACT_BF16 1
#define CSA_SCORE_F32 0  /* index scores kept in fp32 before selection      */
#define CSA_SCORE_BF16 1 /* index scores rounded to BF16 (RNE) before it   */

/* Layer configuration (host struct, plain old data).
 *   B            sequences in the batch
 *   d, r         entry dim and RoPE dims (the last r dims; r even, r <= d);
 *                supported: d in {128, 512}, r multiple of 4, 0 < r < d
 *   m            compression ratio: 4 (CSA) or 128 (HCA); 1..256 accepted
 *   n_idx_heads  indexer heads H_I (1..64); idx_dim its dim c_I (64 or 128)
 *   topk         k (1..2048) -- entries kept per query
 *   n_heads      query heads n_h (1..128)
 *   window       sliding-window length W in raw tokens (1..1024)
 *   kv_fmt, idx_fmt, act_fmt   CSA_KV_*, CSA_IDX_*, CSA_ACT_*
 *   softmax_scale  tau (logit = tau * q.v)
 *   rope_theta     RoPE base (pair j of the last r dims turns by
 *                  pos * theta^(-2j/r))
 *   eps            RMSNorm epsilon
 *   score_fmt      CSA_SCORE_F32 or CSA_SCORE_BF16: the precision of the
 *                  index scores the top-k selector ranks ([kwkr 4.4]: the
 *                  scores are quantised from FP32 to BF16 before the
 *                  selector; ties after rounding go to the lower index)
 */
typedef struct csa_params {
  int32_t B, d, r, m;
  int32_t n_idx_heads, idx_dim;
  int32_t topk, n_heads, window;
  int32_t kv_fmt, idx_fmt, act_fmt;
  float softmax_scale, rope_theta, eps;
  int32_t score_fmt;
} csa_params;

/* A KV-row buffer: the compressed-entry cache, or the raw-token window ring.
 *   rows   [B][cap][row_bytes]   (row layout above)
 *   scale  [B][cap] fp32         (CSA_KV_FP8_BF16 only; NULL for CSA_KV_F32)
 *   cap    rows per sequence.  For the cache, entry i of sequence b is row i.
 *          For the window ring, the token at position p is row p mod cap. */
typedef struct csa_kv {
  void* rows;
  float* scale;
  int64_t cap;
} csa_kv;

/* ------------------------------------------------------------------------
 * csa_compress / hca_compress  [kwkr 3.1, 3.2; Qiaomu 混合注意力机制;
 *                               WeChat 1.1; PACMAN 3.1, 3.2]
 *
 * For every sequence b and entry e in [e_begin[b], e_end[b]):
 *   logits  ga_u (u in block e: tokens m*e .. m*e+m-1, stream a) and
 *           gb_u (u in block e-1, stream b; empty for e = 0)
 *   w       = softmax over the union of those <= 2m logits
 *   x       = sum_u w_u a_u + sum_u w_u b_u
 *   y       = norm_w * x / sqrt(mean(x^2) + eps)
 *   entry   = y with pair j of the last r dims rotated by (m*e)*theta^(-2j/r)
 * and stores it as row e of `out` (FP8: scale = amax_nope/448, codes =
 * E4M3 RNE-satfinite of x/scale; RoPE dims BF16 RNE), out_pos[b*cap+e] = m*e.
 *
 *   a, b       [B][S][d] streams (act_fmt), token at absolute position p of
 *              sequence b is row p - tok_base[b]
 *   gate       [B][S][2] fp32 logits (column 0: stream a, column 1: stream b)
 *   tok_base, e_begin, e_end   int32 [B] (device)
 *   max_entries  host upper bound on e_end[b]-e_begin[b] (sizes the grid)
 *   norm_w     [d] fp32 RMSNorm weight, or NULL for ones
 *   out_pos    int32 [B][out.cap], nullable
 * Entries whose tokens fall outside [tok_base, tok_base+S) or whose slot is
 * >= out.cap are skipped with CSA_DEV_ERR_RANGE.  csa_compress and
 * hca_compress are the same operator; each is tuned for its own m.
 * ---------------------------------------------------------------------- */
csa_status csa_compress(const csa_params* params, const void* a, const void* b,
                        const float* gate, int64_t S, const int32_t* tok_base,
                        const int32_t* e_begin, const int32_t* e_end,
                        int32_t max_entries, const float* norm_w, csa_kv out,
                        int32_t* out_pos, int32_t* err, void* stream);
csa_status hca_compress(const csa_params* params, const void* a, const void* b,
                        const float* gate, int64_t S, const int32_t* tok_base,
                        const int32_t* e_begin, const int32_t* e_end,
                        int32_t max_entries, const float* norm_w, csa_kv out,
                        int32_t* out_pos, int32_t* err, void* stream);

/* ------------------------------------------------------------------------
 * csa_index_compress  [kwkr 3.1 (the indexer scores the compressed
 *                      entries), 3.4 and 4.4 (its QK runs in FP4);
 *                      Qiaomu FP4量化感知训练]
 *
 * Index keys of entries e in [e_begin[b], e_end[b]): the compressor of
 * csa_compress (gated two-stream merge, RMSNorm, RoPE at position m*e)
 * run over the idx_dim-dim indexer streams, with RoPE on their last
 * rope_dims dims (0 <= rope_dims <= idx_dim, a multiple of 4), then
 * converted to MXFP4 by the OCP MX v1.0 rule: per block of 32 dims the
 * shared exponent X = floor(log2 max|v|) - 2 (E2M1's largest exponent),
 * clamped to [-127, 127] (-127 for an all-zero block), stored as the UE8M0
 * byte X + 127; each element the E2M1 code of v / 2^X, rounded to nearest
 * even and saturated to +-6.
 *
 *   a, b       [B][S][idx_dim] indexer streams (act_fmt), row p - tok_base[b]
 *   gate       [B][S][2] fp32 logits
 *   tok_base, e_begin, e_end, max_entries, norm_w ([idx_dim] or NULL): as
 *              for csa_compress
 *   k_idx      [B][k_cap][idx_dim/2] MXFP4 key rows (row e written),
 *   k_idx_sf   [B][k_cap][idx_dim/32] UE8M0 scales
 * Entries whose tokens fall outside the buffer or whose slot is >= k_cap
 * are skipped with CSA_DEV_ERR_RANGE.  idx_dim must be 64 or 128.
 * ---------------------------------------------------------------------- */
csa_status csa_index_compress(const csa_params* params, const void* a, const void* b,
                              const float* gate, int64_t S, const int32_t* tok_base,
                              const int32_t* e_begin, const int32_t* e_end,
                              int32_t max_entries, int32_t rope_dims, const float* norm_w,
                              void* k_idx, uint8_t* k_idx_sf, int64_t k_cap, int32_t* err,
                              void* stream);

/* ------------------------------------------------------------------------
 * csa_index_quantize  [kwkr 3.4: the indexer QK runs directly in FP4]
 *
 * n_rows rows of idx_dim values x [n_rows][idx_dim] (act_fmt) -> MXFP4
 * rows out [n_rows][idx_dim/2] and scales out_sf [n_rows][idx_dim/32], by
 * the OCP MX rule of csa_index_compress.  For the index queries of a call,
 * n_rows = B * T * n_idx_heads.
 * ---------------------------------------------------------------------- */
csa_status csa_index_quantize(const csa_params* params, const void* x, int64_t n_rows,
                              void* out, uint8_t* out_sf, void* stream);

/* ------------------------------------------------------------------------
 * csa_index_topk  [Qiaomu 混合注意力机制, FP4量化感知训练; kwkr 3.4, 4.4;
 *                  PACMAN 3.1]
 *
 * Query tau of sequence b sits at position t = q_pos0[b] + tau (tau < T)
 * and sees the n_t = floor((t+1)/m) entries whose last token is <= t.
 *   I(t, s) = sum_h w[b,tau,h] * max(0, q_idx[b,tau,h,:] . k_idx[b,s,:])
 * for s < n_t, then out_idx[b][tau][0..k) = the min(k, n_t) entries with
 * the largest I (ties -> lower s), in ascending order, padded with -1.
 *
 *   q_idx     [B][T][H_I] index queries (MXFP4 bytes or f32), q_idx_sf
 *             [B][T][H_I][c_I/32] UE8M0 scales (MXFP4 only, else NULL)
 *   w         [B][T][H_I] fp32 head weights
 *   k_idx     [B][k_cap] index keys, k_idx_sf [B][k_cap][c_I/32]
 *   n_max     host upper bound on n_t over the batch (<= k_cap)
 *   out_idx   int32 [B][T][k]
 *   ws        workspace of csa_index_topk_workspace_bytes(params, T, n_max)
 * Execution depends only on the shape and formats, never on the data:
 * MXFP4 with 64 index heads of 128 dims and k_cap a multiple of 4 (each
 * sequence's key-scale rows then start 16-byte aligned for TMA) runs on the
 * tensor cores; every other accepted shape, k_cap not a multiple of 4
 * included, runs on the CUDA cores.  Both compute the scores exactly when
 * every partial sum is representable in fp32, and then agree bit for bit.
 * ---------------------------------------------------------------------- */
csa_status csa_index_topk(const csa_params* params, const void* q_idx,
                          const uint8_t* q_idx_sf, const float* w,
                          const void* k_idx, const uint8_t* k_idx_sf,
                          int64_t k_cap, const int32_t* q_pos0, int32_t T,
                          int32_t n_max, int32_t* out_idx, void* ws,
                          size_t ws_bytes, int32_t* err, void* stream);
size_t csa_index_topk_workspace_bytes(const csa_params* params, int32_t T,
                                      int32_t n_max);

/* ------------------------------------------------------------------------
 * csa_sparse_attn  [WeChat 1.1; kwkr 3.3; fengweifeng 2.; Qiaomu 混合注意力机制]
 *
 * For query tau of sequence b at t = q_pos0[b] + tau, head h:
 *   J      = {cache row idx[b,tau,j] : idx >= 0} followed by the window
 *            tokens max(0, t-W+1) .. t (ring row p mod win.cap)
 *   z_j    = softmax_scale * q[b,tau,h,:] . v_j     (v_j is key and value)
 *   p_j    = exp(z_j) / (exp(sink[h]) + sum_j exp(z_j))
 *   o      = sum_j p_j v_j, the last r dims then rotated by angle -t
 *            pair-wise (pair j by -t*theta^(-2j/r)); written in act_fmt.
 *   q, out [B][T][n_h][d]; idx int32 [B][T][k]; sink fp32 [n_h]
 * An idx value >= the cache capacity or < -1 is skipped with
 * CSA_DEV_ERR_INDEX.  The window ring must hold every position in
 * [max(0, q_pos0-W+1), q_pos0+T-1] (win.cap >= W + T - 1 suffices).
 * Batch invariance: a query's slots are split over CTAs by a rule that
 * depends only on its own slot count, n_heads and T -- never on the batch,
 * the other sequences or the device -- and split partials are merged in a
 * fixed order, so a query's output is bit-identical run to run and whatever
 * batch it is in (for the same T).
 * Input range: FP8 row scales must lie in [2^-90, 2^90] (rows outside are
 * skipped with CSA_DEV_ERR_RANGE); RoPE dims and queries may be any finite
 * BF16.  Logits tau*q.v are formed exactly up to fp32 rounding and must be
 * finite in fp32 (a row with a non-finite logit is skipped with
 * CSA_DEV_ERR_RANGE).
 * ---------------------------------------------------------------------- */
csa_status csa_sparse_attn(const csa_params* params, const void* q,
                           csa_kv cache, const int32_t* idx, csa_kv win,
                           const float* sink, const int32_t* q_pos0, int32_t T,
                           void* out, void* ws, size_t ws_bytes, int32_t* err,
                           void* stream);
size_t csa_sparse_attn_workspace_bytes(const csa_params* params, int32_t T);

/* ------------------------------------------------------------------------
 * hca_dense_attn  [PACMAN 3.2; kwkr 3.2, 3.3; WeChat 1.1]
 *
 * As csa_sparse_attn with J = every visible cache entry 0 .. n_t-1
 * (n_t = floor((t+1)/m)) followed by the window.  n_max is a host upper
 * bound on n_t (<= cache.cap).
 * ---------------------------------------------------------------------- */
csa_status hca_dense_attn(const csa_params* params, const void* q,
                          csa_kv cache, csa_kv win, const float* sink,
                          const int32_t* q_pos0, int32_t T, int32_t n_max,
                          void* out, void* ws, size_t ws_bytes, int32_t* err,
                          void* stream);
size_t hca_dense_attn_workspace_bytes(const csa_params* params, int32_t T,
                                      int32_t n_max);

/* ------------------------------------------------------------------------
 * csa_index_topk_noalloc  (no counterpart in the DeepSeek-V4 write-ups: it
 * is a deployment variant of csa_index_topk, not part of the method)
 *
 * csa_index_topk for callers that cannot allocate device memory -- e.g. a
 * plugin handed only its inputs and outputs, or a loop that must not touch
 * the allocator -- and so cannot provide the workspace.  Same arguments and
 * results as csa_index_topk, minus ws/ws_bytes: the workspace is a static
 * 16 MiB device array inside libcsa (held on every GPU that loads the
 * library until the process exits).  Returns CSA_ERR_WORKSPACE, launching
 * nothing, when csa_index_topk_workspace_bytes(params, T, n_max) exceeds
 * 16 MiB.  It allocates nothing (no cudaMalloc/cudaFree, no allocating
 * library call) itself, but the array lives in a library module that the
 * CUDA runtime loads on a device lazily: the first call on a device loads it
 * there, which reserves the 16 MiB (an out-of-memory failure then returns
 * CSA_ERR_LAUNCH), and looks up the array's device address
 * (cudaGetSymbolAddress, with that device current).  Make that first call
 * during set-up, before any allocation-free region and before any stream
 * capture.  If the device's context is destroyed (cudaDeviceReset), the next
 * call loads the module again and looks the address up anew.  Every call
 * shares the one array: calls whose work overlaps on the GPU race on it.
 * ---------------------------------------------------------------------- */
csa_status csa_index_topk_noalloc(const csa_params* params, const void* q_idx,
                                  const uint8_t* q_idx_sf, const float* w,
                                  const void* k_idx, const uint8_t* k_idx_sf,
                                  int64_t k_cap, const int32_t* q_pos0, int32_t T,
                                  int32_t n_max, int32_t* out_idx, int32_t* err,
                                  void* stream);

/* ------------------------------------------------------------------------
 * Decode-time state  [kwkr 4.4: the KV cache splits into a classical KV
 *                     cache and a state cache; periodic checkpointing every
 *                     1024 tokens; kwkr 3.1 / 3.3 for what the state holds]
 *
 * A sequence's state beside its compressed entries (the classical cache):
 *   win     the sliding window's raw tokens, in the cache's row layout,
 *           token p in ring row p mod win.cap (the `win` of the attention
 *           calls)
 *   a, b    the compressor's two stream rings [B][s_cap][d] (act_fmt) and
 *   gate    its gate logits [B][s_cap][2] fp32, token p in row p mod s_cap;
 *           s_cap must be a multiple of m and at least T + 2m for every
 *           append of T tokens (an entry merges its own block of stream a
 *           with the previous block of stream b).
 * A checkpoint store keeps the state at multiples P of `every` (a multiple
 * of m; 1024 on the pages) in n_slots slots per sequence, slot
 * (P/every - 1) mod n_slots:
 *   win_rows  [B][n_slots][W][row_bytes], win_scale [B][n_slots][W]
 *             (CSA_KV_FP8_BF16, else NULL): window rows of positions
 *             P-W .. P-1 (rows of negative positions stored as zeros)
 *   a, b      [B][n_slots][m][d] (act_fmt), gate [B][n_slots][m][2]: the
 *             stream rows of positions P-m .. P-1, all the compressor needs
 *             to continue at P.
 * ---------------------------------------------------------------------- */
typedef struct csa_state {
  csa_kv win;
  void* a;
  void* b;
  float* gate;
  int64_t s_cap;
} csa_state;

typedef struct csa_ckpt {
  void* win_rows;
  float* win_scale;
  void* a;
  void* b;
  float* gate;
  int32_t n_slots;
  int32_t every;
} csa_ckpt;

/* csa_state_append: append T tokens of every sequence b at positions
 * pos0[b] .. pos0[b]+T-1:
 *   - token tau's KV vector kv_new[b][tau] ([B][T][d], act_fmt, already
 *     normalised and rotated like the window tokens the attention reads) is
 *     packed into its window row like a compressed entry (FP8 format:
 *     scale = amax of the non-RoPE dims / 448, E4M3 codes RNE saturating,
 *     BF16 RoPE dims);
 *   - its stream rows a_new[b][tau], b_new[b][tau] ([B][T][d]) and gate
 *     logits gate_new[b][tau] ([B][T][2]) go into the stream rings;
 *   - every entry these tokens complete (entries pos0/m .. (pos0+T)/m - 1)
 *     is compressed from the rings exactly as csa_compress would, into row
 *     e of `cache` (cache_pos[b][e] = m*e when cache_pos is not NULL);
 *   - with a checkpoint store (ckpt not NULL), the state at the last
 *     multiple P of ckpt->every in (pos0, pos0+T] is copied into its slot.
 * Requirements: win.cap >= window + T - 1 (the attention's own bound),
 * s_cap a multiple of m with s_cap >= T + 2m.  HCA (m = 128) uses the same
 * call with its own cache. */
csa_status csa_state_append(const csa_params* params, const void* kv_new, const void* a_new,
                            const void* b_new, const float* gate_new, const int32_t* pos0,
                            int32_t T, csa_state state, csa_kv cache, int32_t* cache_pos,
                            const csa_ckpt* ckpt, int32_t* err, void* stream);

/* csa_state_restore: put the state checkpointed at pos[b] (a positive
 * multiple of ckpt->every, still held by its slot) back into the window and
 * stream rings of sequence b, so that appending can continue at pos[b]
 * (entries below pos[b]/m must still be in the cache).  A pos[b] that is
 * not a positive multiple of `every` raises CSA_DEV_ERR_RANGE and leaves
 * that sequence's rings untouched. */
csa_status csa_state_restore(const csa_params* params, const int32_t* pos, const csa_ckpt* ckpt,
                             csa_state state, int32_t* err, void* stream);

/* Human-readable name of a csa_status. */
const char* csa_status_string(csa_status s);

/* The CUDA error string behind the last CSA_ERR_LAUNCH returned on the
 * calling host thread ("no error" if there was none).  Diagnostic only. */
const char* csa_last_error_string(void);

#ifdef __cplusplus
}
#endif
#endif /* CSA_H_ */
