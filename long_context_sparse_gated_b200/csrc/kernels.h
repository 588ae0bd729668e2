// Internal launchers of libcsa (not part of the public ABI).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "csa.h"

namespace csa {

// Message returned by csa_last_error_string() on this host thread (a string
// with static storage duration).
void set_last_error(const char* msg);

// Host-side work done once (host_cache.cu).  Id of the calling thread's
// current context (0 if none); SM count of the current device; raise a
// kernel's dynamic shared-memory limit once per device and context; encode
// a TMA tensor map (no multicast, L2 256-byte promotion, zero fill), reusing
// a recent identical encode of this host thread.
unsigned long long current_ctx_id();
int sm_count();
cudaError_t set_max_smem(const void* kernel, size_t bytes);
bool tensor_maps_available();
bool encode_tensor_map(CUtensorMap* map, CUtensorMapDataType dt, int rank, const void* base, const uint64_t* dims,
                       const uint64_t* strides_bytes, const uint32_t* box, CUtensorMapSwizzle sw);

// Launch with programmatic stream serialisation (see pdl_wait in
// common.cuh): the kernel may begin while its predecessor on the stream
// drains.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

cudaError_t launch_compress(const csa_params& p, const void* a, const void* b, const float* gate,
                            int64_t S, const int32_t* tok_base, const int32_t* e_begin,
                            const int32_t* e_end, int32_t max_entries, const float* norm_w,
                            const csa_kv& out, int32_t* out_pos, int32_t* err, cudaStream_t st);

cudaError_t launch_index_compress(const csa_params& p, int rope_dims, const void* a, const void* b,
                                  const float* gate, int64_t S, const int32_t* tok_base, const int32_t* e_begin,
                                  const int32_t* e_end, int32_t max_entries, const float* norm_w, void* k_idx,
                                  uint8_t* k_idx_sf, int64_t k_cap, int32_t* err, cudaStream_t st);

cudaError_t launch_index_quantize(const csa_params& p, const void* x, int64_t n_rows, void* out, uint8_t* out_sf,
                                  cudaStream_t st);

cudaError_t launch_compress_ring(const csa_params& p, const void* a, const void* b, const float* gate, int64_t ring,
                                 const int32_t* pos0, int T_new, const csa_kv& out, int32_t* out_pos, int32_t* err,
                                 cudaStream_t st);

cudaError_t launch_state_append(const csa_params& p, const void* kv_new, const void* a_new, const void* b_new,
                                const float* gate_new, const int32_t* pos0, int T, const csa_state& s,
                                const csa_kv& cache, int32_t* cache_pos, const csa_ckpt* ck, int32_t* err,
                                cudaStream_t st);

cudaError_t launch_state_restore(const csa_params& p, const int32_t* pos, const csa_ckpt& ck, const csa_state& s,
                                 int32_t* err, cudaStream_t st);

// Scores are fp32, or BF16 (round to nearest even) when p.score_fmt is
// CSA_SCORE_BF16; `scores` points to [B*T][ld] of either.
cudaError_t launch_index_scores(const csa_params& p, const void* q_idx, const uint8_t* q_sf,
                                const float* w, const void* k_idx, const uint8_t* k_sf,
                                int64_t k_cap, const int32_t* q_pos0, int T, void* scores,
                                int ld, int n_max, int32_t* err, cudaStream_t st);

bool index_scores_tc_supported(const csa_params& p, int64_t k_cap, const void* q_idx, const uint8_t* q_sf,
                               const void* k_idx, const uint8_t* k_sf);

cudaError_t launch_index_scores_tc(const csa_params& p, const void* q_idx, const uint8_t* q_sf, const float* w,
                                   const void* k_idx, const uint8_t* k_sf, int64_t k_cap,
                                   const int32_t* q_pos0, int T, void* scores, int ld, uint32_t* hist,
                                   int n_max, int32_t* err, cudaStream_t st);

bool topk_use_hist(int queries);
int topk_scores_ld(int n_max);
size_t topk_zero_bytes(int queries);
size_t topk_extra_bytes(int queries, int n_max);
cudaError_t launch_topk_select(const csa_params& p, const void* scores, bool bf16, int ld, int n_max,
                               const uint32_t* hist, void* extra, const int32_t* q_pos0, int T, int32_t* out_idx,
                               cudaStream_t st);

size_t attn_workspace_bytes(const csa_params& p, int T, int n_sel, bool dense);

cudaError_t launch_attn_merge(const csa_params& p, const float* ws_o, const float* ws_ml, int n_splits,
                              const float* sink, const int32_t* q_pos0, int T, int n_sel, bool dense,
                              int rows_per_split, void* out, cudaStream_t st);

bool attn_tc_supported(const csa_params& p);
size_t attn_tc_workspace_bytes(const csa_params& p, int T, int n_sel, bool dense);
cudaError_t launch_attn_tc(const csa_params& p, const void* q, const csa_kv& cache, const int32_t* idx,
                           const csa_kv& win, const float* sink, const int32_t* q_pos0, int T, int n_sel,
                           bool dense, void* out, float* ws, int32_t* err, cudaStream_t st);

cudaError_t launch_attn(const csa_params& p, const void* q, const csa_kv& cache, const int32_t* idx,
                        const csa_kv& win, const float* sink, const int32_t* q_pos0, int T,
                        int n_sel, bool dense, void* out, float* ws, int32_t* err,
                        cudaStream_t st);

}  // namespace csa
