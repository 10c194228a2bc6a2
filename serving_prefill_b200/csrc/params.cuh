// Kernel parameter blocks shared by the host API and the kernel units, and
// the launchers each unit exports.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "common.cuh"

namespace rag {
struct FwdParams {
  BatchDev batch;
  int32_t num_pages, num_kv_heads, num_q_heads, group, layer;
  int32_t tiles_per_split;
  int32_t direct;
  float scale_log2;
  __nv_bfloat16* o;
  float* row_lse;
  float* row_m2;
  float* row_il;
  float* part;
  int32_t* item_prefix;
  int32_t* err;
  float* impact_zero;
  int64_t impact_len;
  int64_t max_items;              // partial slots the workspace holds
};
struct CombineParams {
  BatchDev batch;
  int32_t num_kv_heads, num_q_heads, group, tiles_per_split;
  const float* part;
  const int32_t* item_prefix;
  int64_t max_items;
  __nv_bfloat16* o;
  float* row_lse;
  float* row_m2;
  float* row_il;
};
struct ImpactParams {
  BatchDev batch;
  int32_t num_pages, num_kv_heads, num_q_heads, group, layer;
  int32_t tiles_per_split;
  float scale_log2;
  const float* row_m2;
  const float* row_il;
  float* impact;
  int32_t* err;
};
struct TopkParams {
  BatchDev batch;
  const float* impact;
  double r;
  int32_t k_cap;
  int32_t k_max;           // k of the longest request
  int32_t* topk_idx;
  float* topk_val;
  int32_t* k_out;
};
struct SimtParams {
  BatchDev batch;
  int32_t num_pages, num_kv_heads, num_q_heads, group, layer, head_dim;
  float scale;
  const float* pool_k;
  const float* pool_v;
  const float* q;
  const float* kq;
  const float* vq;
  float* o;
  float* row_lse;
  float* row_m;
  float* row_l;
  float* impact;
  int32_t* err;
};
struct PoolWriteParams {
  uint8_t* pool_k;
  uint8_t* pool_v;
  const uint8_t* k;
  const uint8_t* v;
  const int32_t* page_ids;
  int32_t* err;
  int32_t layer, num_pages, num_kv_heads, n_tokens;
  int32_t row_bytes;
};

cudaError_t launch_attn_fwd(const CUtensorMap&, const CUtensorMap&, const CUtensorMap&, const CUtensorMap&,
                            const CUtensorMap&, const FwdParams&, int, cudaStream_t);
cudaError_t launch_attn_combine(const CombineParams&, int, int, cudaStream_t);
cudaError_t launch_impact(const CUtensorMap&, const CUtensorMap&, const CUtensorMap&, const ImpactParams&, int,
                          cudaStream_t);
cudaError_t launch_topk(const TopkParams&, int, int, cudaStream_t);
cudaError_t launch_simt_attn(const SimtParams&, int, cudaStream_t);
cudaError_t launch_simt_impact(const SimtParams&, int, int, cudaStream_t);
cudaError_t launch_pool_write(const PoolWriteParams&, int, cudaStream_t);

}  // namespace rag
