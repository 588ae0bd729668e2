// C ABI of libcsa: host-side validation and dispatch.  Nothing here
// allocates, synchronises or keeps state; every call only enqueues kernels
// on the caller's stream.
#include <cuda_runtime.h>

#include "csa.h"
#include "kernels.h"

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

csa_status check_params(const csa_params* p) {
  if (!p) return CSA_ERR_INVALID;
  if (p->B < 1 || p->d < 1 || p->r < 0 || p->m < 1) return CSA_ERR_INVALID;
  if (p->d != 128 && p->d != 512) return CSA_ERR_UNSUPPORTED;
  if (p->r <= 0 || p->r >= p->d || (p->r & 3)) return CSA_ERR_UNSUPPORTED;
  if (p->m > 256) return CSA_ERR_UNSUPPORTED;
  if (p->kv_fmt != CSA_KV_F32 && p->kv_fmt != CSA_KV_FP8_BF16) return CSA_ERR_UNSUPPORTED;
  if (p->idx_fmt != CSA_IDX_F32 && p->idx_fmt != CSA_IDX_MXFP4) return CSA_ERR_UNSUPPORTED;
  if (p->act_fmt != CSA_ACT_F32 && p->act_fmt != CSA_ACT_BF16) return CSA_ERR_UNSUPPORTED;
  if (!(p->eps >= 0.f) || !(p->rope_theta > 0.f)) return CSA_ERR_INVALID;
  return CSA_OK;
}

csa_status check_attn_params(const csa_params* p) {
  csa_status s = check_params(p);
  if (s != CSA_OK) return s;
  if (p->n_heads < 1 || p->n_heads > 128) return CSA_ERR_UNSUPPORTED;
  if (p->window < 1 || p->window > 1024) return CSA_ERR_UNSUPPORTED;
  return CSA_OK;
}

csa_status check_kv(const csa_params* p, const csa_kv& kv) {
  if (!kv.rows || kv.cap < 1) return CSA_ERR_INVALID;
  if (!aligned16(kv.rows)) return CSA_ERR_ALIGN;
  if (p->kv_fmt == CSA_KV_FP8_BF16) {
    if (!kv.scale) return CSA_ERR_INVALID;
    if (!aligned16(kv.scale)) return CSA_ERR_ALIGN;
  }
  return CSA_OK;
}

thread_local const char* g_last_error = "no error";

csa_status launched(cudaError_t e) {
  if (e == cudaSuccess) return CSA_OK;
  g_last_error = cudaGetErrorString(e);
  return CSA_ERR_LAUNCH;
}

}  // namespace

namespace csa {
void set_last_error(const char* msg) { g_last_error = msg; }
}  // namespace csa

namespace {

csa_status compress_impl(const csa_params* p, const void* a, const void* b, const float* gate,
                         int64_t S, const int32_t* tok_base, const int32_t* e_begin,
                         const int32_t* e_end, int32_t max_entries, const float* norm_w,
                         csa_kv out, int32_t* out_pos, int32_t* err, void* stream) {
  csa_status s = check_params(p);
  if (s != CSA_OK) return s;
  if (!a || !b || !gate || !tok_base || !e_begin || !e_end || S < 1 || max_entries < 0)
    return CSA_ERR_INVALID;
  for (const void* ptr : {a, b, (const void*)gate, (const void*)tok_base, (const void*)e_begin,
                          (const void*)e_end})
    if (!aligned16(ptr)) return CSA_ERR_ALIGN;
  if ((norm_w && !aligned16(norm_w)) || (out_pos && !aligned16(out_pos))) return CSA_ERR_ALIGN;
  s = check_kv(p, out);
  if (s != CSA_OK) return s;
  if (max_entries == 0) return CSA_OK;
  return launched(csa::launch_compress(*p, a, b, gate, S, tok_base, e_begin, e_end, max_entries,
                                       norm_w, out, out_pos, err,
                                       reinterpret_cast<cudaStream_t>(stream)));
}

// Index workspace: scores [B*T][ld] (ld = n_max rounded up to 32; fp32, or
// BF16 with CSA_SCORE_BF16), then, for decode-sized batches, the region the
// call clears (4096-bin histogram, tie count and 256-bin second-level
// histogram per query) and, for rows over 32768 entries, selection bitmaps
// and tie lists.
size_t round256(size_t b) { return (b + 255) & ~(size_t)255; }

size_t scores_bytes(const csa_params* p, int32_t T, int32_t n_max) {
  const size_t el = p->score_fmt == CSA_SCORE_BF16 ? 2 : 4;
  return round256((size_t)p->B * (size_t)T * (size_t)csa::topk_scores_ld(n_max) * el);
}

size_t index_ws_bytes(const csa_params* p, int32_t T, int32_t n_max) {
  size_t b = scores_bytes(p, T, n_max);
  const int nq = p->B * T;
  if (csa::topk_use_hist(nq)) b += round256(csa::topk_zero_bytes(nq)) + csa::topk_extra_bytes(nq, n_max);
  return b;
}

}  // namespace

extern "C" {

csa_status csa_compress(const csa_params* p, const void* a, const void* b, const float* gate,
                        int64_t S, const int32_t* tok_base, const int32_t* e_begin,
                        const int32_t* e_end, int32_t max_entries, const float* norm_w, csa_kv out,
                        int32_t* out_pos, int32_t* err, void* stream) {
  return compress_impl(p, a, b, gate, S, tok_base, e_begin, e_end, max_entries, norm_w, out,
                       out_pos, err, stream);
}

csa_status hca_compress(const csa_params* p, const void* a, const void* b, const float* gate,
                        int64_t S, const int32_t* tok_base, const int32_t* e_begin,
                        const int32_t* e_end, int32_t max_entries, const float* norm_w, csa_kv out,
                        int32_t* out_pos, int32_t* err, void* stream) {
  return compress_impl(p, a, b, gate, S, tok_base, e_begin, e_end, max_entries, norm_w, out,
                       out_pos, err, stream);
}

csa_status csa_index_compress(const csa_params* p, const void* a, const void* b, const float* gate, int64_t S,
                              const int32_t* tok_base, const int32_t* e_begin, const int32_t* e_end,
                              int32_t max_entries, int32_t rope_dims, const float* norm_w, void* k_idx,
                              uint8_t* k_idx_sf, int64_t k_cap, int32_t* err, void* stream) {
  if (!p) return CSA_ERR_INVALID;
  if (p->B < 1 || p->m < 1 || max_entries < 0 || S < 1 || k_cap < 1) return CSA_ERR_INVALID;
  if (p->m > 256) return CSA_ERR_UNSUPPORTED;
  if (p->idx_dim != 64 && p->idx_dim != 128) return CSA_ERR_UNSUPPORTED;
  if (rope_dims < 0 || rope_dims > p->idx_dim || (rope_dims & 3)) return CSA_ERR_UNSUPPORTED;
  if (p->act_fmt != CSA_ACT_F32 && p->act_fmt != CSA_ACT_BF16) return CSA_ERR_UNSUPPORTED;
  if (!(p->eps >= 0.f) || !(p->rope_theta > 0.f)) return CSA_ERR_INVALID;
  if (!a || !b || !gate || !tok_base || !e_begin || !e_end || !k_idx || !k_idx_sf) return CSA_ERR_INVALID;
  for (const void* ptr : {a, b, (const void*)gate, (const void*)tok_base, (const void*)e_begin,
                          (const void*)e_end, (const void*)k_idx, (const void*)k_idx_sf})
    if (!aligned16(ptr)) return CSA_ERR_ALIGN;
  if (norm_w && !aligned16(norm_w)) return CSA_ERR_ALIGN;
  if (max_entries == 0) return CSA_OK;
  return launched(csa::launch_index_compress(*p, rope_dims, a, b, gate, S, tok_base, e_begin, e_end, max_entries,
                                             norm_w, k_idx, k_idx_sf, k_cap, err,
                                             reinterpret_cast<cudaStream_t>(stream)));
}

csa_status csa_index_quantize(const csa_params* p, const void* x, int64_t n_rows, void* out, uint8_t* out_sf,
                              void* stream) {
  if (!p || n_rows < 0) return CSA_ERR_INVALID;
  if (p->idx_dim != 64 && p->idx_dim != 128) return CSA_ERR_UNSUPPORTED;
  if (p->act_fmt != CSA_ACT_F32 && p->act_fmt != CSA_ACT_BF16) return CSA_ERR_UNSUPPORTED;
  if (n_rows == 0) return CSA_OK;
  if (!x || !out || !out_sf) return CSA_ERR_INVALID;
  for (const void* ptr : {x, (const void*)out, (const void*)out_sf})
    if (!aligned16(ptr)) return CSA_ERR_ALIGN;
  return launched(csa::launch_index_quantize(*p, x, n_rows, out, out_sf, reinterpret_cast<cudaStream_t>(stream)));
}

size_t csa_index_topk_workspace_bytes(const csa_params* p, int32_t T, int32_t n_max) {
  if (!p || T < 1 || n_max < 0 || p->B < 1) return 0;
  return index_ws_bytes(p, T, n_max);
}

csa_status csa_index_topk(const csa_params* p, const void* q_idx, const uint8_t* q_idx_sf,
                          const float* w, const void* k_idx, const uint8_t* k_idx_sf,
                          int64_t k_cap, const int32_t* q_pos0, int32_t T, int32_t n_max,
                          int32_t* out_idx, void* ws, size_t ws_bytes, int32_t* err,
                          void* stream) {
  csa_status s = check_params(p);
  if (s != CSA_OK) return s;
  if (p->n_idx_heads < 1 || p->n_idx_heads > 64) return CSA_ERR_UNSUPPORTED;
  if (p->idx_dim != 64 && p->idx_dim != 128) return CSA_ERR_UNSUPPORTED;
  if (p->topk < 1 || p->topk > 2048) return CSA_ERR_UNSUPPORTED;
  if (p->score_fmt != CSA_SCORE_F32 && p->score_fmt != CSA_SCORE_BF16) return CSA_ERR_UNSUPPORTED;
  if (!q_idx || !w || !k_idx || !q_pos0 || !out_idx || T < 1 || n_max < 0 || k_cap < 1 ||
      n_max > k_cap)
    return CSA_ERR_INVALID;
  const bool mx = p->idx_fmt == CSA_IDX_MXFP4;
  if (mx && (!q_idx_sf || !k_idx_sf)) return CSA_ERR_INVALID;
  for (const void* ptr : {q_idx, (const void*)w, k_idx, (const void*)q_pos0, (const void*)out_idx})
    if (!aligned16(ptr)) return CSA_ERR_ALIGN;
  if (mx && (!aligned16(q_idx_sf) || !aligned16(k_idx_sf))) return CSA_ERR_ALIGN;
  const size_t need = index_ws_bytes(p, T, n_max);
  if (ws_bytes < need || (need && !ws)) return CSA_ERR_WORKSPACE;
  if (ws && !aligned16(ws)) return CSA_ERR_ALIGN;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  void* scores = ws;
  const int ld = csa::topk_scores_ld(n_max);
  const int nq = p->B * T;
  const bool tc = csa::index_scores_tc_supported(*p, k_cap, q_idx, q_idx_sf, k_idx, k_idx_sf);
  uint32_t* hist = nullptr;
  void* extra = nullptr;
  if (tc && csa::topk_use_hist(nq) && n_max > p->topk) {
    hist = reinterpret_cast<uint32_t*>(reinterpret_cast<char*>(ws) + scores_bytes(p, T, n_max));
    extra = reinterpret_cast<char*>(hist) + round256(csa::topk_zero_bytes(nq));
    cudaError_t e = cudaMemsetAsync(hist, 0, csa::topk_zero_bytes(nq), st);
    if (e != cudaSuccess) return launched(e);
  }
  if (n_max > 0) {
    cudaError_t e;
    if (tc)
      e = csa::launch_index_scores_tc(*p, q_idx, q_idx_sf, w, k_idx, k_idx_sf, k_cap, q_pos0, T, scores, ld,
                                      hist, n_max, err, st);
    else
      e = csa::launch_index_scores(*p, q_idx, q_idx_sf, w, k_idx, k_idx_sf, k_cap, q_pos0, T, scores, ld,
                                   n_max, err, st);
    if (e != cudaSuccess) return launched(e);
  }
  return launched(csa::launch_topk_select(*p, scores, p->score_fmt == CSA_SCORE_BF16, ld, n_max, hist, extra,
                                          q_pos0, T, out_idx, st));
}

size_t csa_sparse_attn_workspace_bytes(const csa_params* p, int32_t T) {
  if (!p || T < 1 || p->B < 1) return 0;
  return csa::attn_workspace_bytes(*p, T, p->topk, false);
}

size_t hca_dense_attn_workspace_bytes(const csa_params* p, int32_t T, int32_t n_max) {
  if (!p || T < 1 || p->B < 1 || n_max < 0) return 0;
  return csa::attn_workspace_bytes(*p, T, n_max, true);
}

static csa_status attn_impl(const csa_params* p, const void* q, csa_kv cache, const int32_t* idx,
                            csa_kv win, const float* sink, const int32_t* q_pos0, int32_t T,
                            int32_t n_sel, bool dense, void* out, void* ws, size_t ws_bytes,
                            int32_t* err, void* stream) {
  csa_status s = check_attn_params(p);
  if (s != CSA_OK) return s;
  if (!q || !sink || !q_pos0 || !out || T < 1) return CSA_ERR_INVALID;
  if (!dense && (!idx || p->topk < 1 || p->topk > 2048)) return CSA_ERR_INVALID;
  if (dense && (n_sel < 0 || n_sel > cache.cap)) return CSA_ERR_INVALID;
  for (const void* ptr : {q, (const void*)sink, (const void*)q_pos0, (const void*)out})
    if (!aligned16(ptr)) return CSA_ERR_ALIGN;
  if (idx && !aligned16(idx)) return CSA_ERR_ALIGN;
  if ((s = check_kv(p, cache)) != CSA_OK) return s;
  if ((s = check_kv(p, win)) != CSA_OK) return s;
  if (win.cap < p->window || win.cap < T) return CSA_ERR_INVALID;
  const size_t need = csa::attn_workspace_bytes(*p, T, n_sel, dense);
  if (ws_bytes < need || (need && !ws)) return CSA_ERR_WORKSPACE;
  if (ws && !aligned16(ws)) return CSA_ERR_ALIGN;
  return launched(csa::launch_attn(*p, q, cache, idx, win, sink, q_pos0, T, n_sel, dense, out,
                                   reinterpret_cast<float*>(ws), err,
                                   reinterpret_cast<cudaStream_t>(stream)));
}

csa_status csa_sparse_attn(const csa_params* p, const void* q, csa_kv cache, const int32_t* idx,
                           csa_kv win, const float* sink, const int32_t* q_pos0, int32_t T,
                           void* out, void* ws, size_t ws_bytes, int32_t* err, void* stream) {
  if (!p) return CSA_ERR_INVALID;
  return attn_impl(p, q, cache, idx, win, sink, q_pos0, T, p->topk, false, out, ws, ws_bytes, err,
                   stream);
}

csa_status hca_dense_attn(const csa_params* p, const void* q, csa_kv cache, csa_kv win,
                          const float* sink, const int32_t* q_pos0, int32_t T, int32_t n_max,
                          void* out, void* ws, size_t ws_bytes, int32_t* err, void* stream) {
  return attn_impl(p, q, cache, nullptr, win, sink, q_pos0, T, n_max, true, out, ws, ws_bytes, err,
                   stream);
}

static csa_status check_state(const csa_params* p, const csa_state& s, int32_t T) {
  csa_status st = check_kv(p, s.win);
  if (st != CSA_OK) return st;
  if (!s.a || !s.b || !s.gate) return CSA_ERR_INVALID;
  for (const void* ptr : {(const void*)s.a, (const void*)s.b, (const void*)s.gate})
    if (!aligned16(ptr)) return CSA_ERR_ALIGN;
  if (s.s_cap < (int64_t)T + 2 * p->m || s.s_cap % p->m) return CSA_ERR_INVALID;
  if (s.win.cap < (int64_t)p->window + T - 1) return CSA_ERR_INVALID;
  return CSA_OK;
}

static csa_status check_ckpt(const csa_params* p, const csa_ckpt& c) {
  if (c.n_slots < 1 || c.every < p->m || c.every % p->m) return CSA_ERR_INVALID;
  if (!c.win_rows || !c.a || !c.b || !c.gate) return CSA_ERR_INVALID;
  if (p->kv_fmt == CSA_KV_FP8_BF16 && !c.win_scale) return CSA_ERR_INVALID;
  for (const void* ptr : {(const void*)c.win_rows, (const void*)c.a, (const void*)c.b, (const void*)c.gate})
    if (!aligned16(ptr)) return CSA_ERR_ALIGN;
  if (c.win_scale && !aligned16(c.win_scale)) return CSA_ERR_ALIGN;
  return CSA_OK;
}

csa_status csa_state_append(const csa_params* p, const void* kv_new, const void* a_new, const void* b_new,
                            const float* gate_new, const int32_t* pos0, int32_t T, csa_state state, csa_kv cache,
                            int32_t* cache_pos, const csa_ckpt* ckpt, int32_t* err, void* stream) {
  csa_status s = check_params(p);
  if (s != CSA_OK) return s;
  if (p->window < 1 || p->window > 1024) return CSA_ERR_UNSUPPORTED;
  if (T < 1 || T > 65535 || !kv_new || !a_new || !b_new || !gate_new || !pos0) return CSA_ERR_INVALID;
  for (const void* ptr : {kv_new, a_new, b_new, (const void*)gate_new, (const void*)pos0})
    if (!aligned16(ptr)) return CSA_ERR_ALIGN;
  if (cache_pos && !aligned16(cache_pos)) return CSA_ERR_ALIGN;
  if ((s = check_state(p, state, T)) != CSA_OK) return s;
  if ((s = check_kv(p, cache)) != CSA_OK) return s;
  if (ckpt && (s = check_ckpt(p, *ckpt)) != CSA_OK) return s;
  return launched(csa::launch_state_append(*p, kv_new, a_new, b_new, gate_new, pos0, T, state, cache, cache_pos, ckpt,
                                           err, reinterpret_cast<cudaStream_t>(stream)));
}

csa_status csa_state_restore(const csa_params* p, const int32_t* pos, const csa_ckpt* ckpt, csa_state state,
                             int32_t* err, void* stream) {
  csa_status s = check_params(p);
  if (s != CSA_OK) return s;
  if (p->window < 1 || p->window > 1024) return CSA_ERR_UNSUPPORTED;
  if (!pos || !ckpt) return CSA_ERR_INVALID;
  if (!aligned16(pos)) return CSA_ERR_ALIGN;
  if ((s = check_state(p, state, 1)) != CSA_OK) return s;
  if ((s = check_ckpt(p, *ckpt)) != CSA_OK) return s;
  return launched(csa::launch_state_restore(*p, pos, *ckpt, state, err, reinterpret_cast<cudaStream_t>(stream)));
}

const char* csa_last_error_string(void) { return g_last_error; }

const char* csa_status_string(csa_status s) {
  switch (s) {
    case CSA_OK: return "CSA_OK";
    case CSA_ERR_INVALID: return "CSA_ERR_INVALID";
    case CSA_ERR_UNSUPPORTED: return "CSA_ERR_UNSUPPORTED";
    case CSA_ERR_ALIGN: return "CSA_ERR_ALIGN";
    case CSA_ERR_WORKSPACE: return "CSA_ERR_WORKSPACE";
    case CSA_ERR_LAUNCH: return "CSA_ERR_LAUNCH";
    default: return "CSA_ERR_UNKNOWN";
  }
}

}  // extern "C"
