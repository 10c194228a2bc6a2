// Kernel parameter blocks shared by the host API and the kernel units, and
// the launchers each unit exports.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <mutex>
#include <utility>

#include "common.cuh"

namespace rag {

// Launch a kernel that may overlap the tail of the previous kernel in its
// stream (programmatic stream serialization). The kernel must call
// pdl_wait() before it reads anything the previous kernel writes, or writes
// anything the previous kernel reads. cluster > 1 also sets the cluster size.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                              int cluster, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  unsigned n = 1;
  if (cluster > 1) {
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = unsigned(cluster);
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    n = 2;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}
// cudaFuncSetAttribute acts on the current device's context only, so the
// largest dynamic shared-memory size set for a kernel is kept per device (and
// the record is shared by host threads under a mutex).
constexpr int kMaxDevices = 64;
struct SmemAttr {
  std::mutex mu;
  size_t bytes[kMaxDevices] = {};
};
template <typename Kernel>
inline cudaError_t ensure_smem_attr(Kernel kernel, SmemAttr& rec, size_t bytes) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(rec.mu);
  if (bytes > rec.bytes[dev]) {
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(bytes));
    if (e != cudaSuccess) return e;
    rec.bytes[dev] = bytes;
  }
  return cudaSuccess;
}

// The last CUDA error a library call met (reported by rag_last_cuda_error).
void note_cuda_error(cudaError_t e);

// Ordinary launch (waits for the previous kernel to complete) that returns
// this launch's own error rather than a stale one from an earlier call.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_plain(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                                Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.attrs = nullptr;
  cfg.numAttrs = 0;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

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
  const float2* rope;             // per chunk-list entry, 64 (cos, sin) pairs; null: keys used as stored
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
  const float2* rope;             // as FwdParams::rope
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
  int32_t v_to_f16;   // bf16 pool: V is stored as fp16 (its bf16 value, saturated beyond 65504)
};

// Selective recompute. The plan buffer (int32 words, each region 64-word
// aligned) that the plan kernel writes and the copy and GEMM kernels read:
//   header   16 words: n_tok, n_cow, n_needed, error bits
//   x_row    [max_tok]  hidden-state row of selected token t (-1: skipped)
//   dst      [max_tok]  private page * 16 + slot of token t (slot only, before the pages are known)
//   ref      [max_tok]  page reference of token t (-1: skipped)
//   cow_src  [max_cow]  page copied from
//   cow_dst  [max_cow]  private page copied to
//   cow_mask [max_cow]  selected slots of that page (bit s: slot s), which the copy leaves alone
//   flags    [page_refs] selected-slot mask per page reference
// max_tok = B * k_cap, max_cow = page_refs.
struct RcPlanLayout {
  int64_t x_row, dst, ref, cow_src, cow_dst, cow_mask, flags, words;
};
__host__ __device__ inline int64_t align64w(int64_t x) { return (x + 63) & ~int64_t(63); }
__host__ __device__ inline RcPlanLayout rc_plan_layout(int64_t max_tok, int64_t page_refs) {
  RcPlanLayout l;
  int64_t at = 64;
  l.x_row = at; at = align64w(at + max_tok);
  l.dst = at; at = align64w(at + max_tok);
  l.ref = at; at = align64w(at + max_tok);
  l.cow_src = at; at = align64w(at + page_refs);
  l.cow_dst = at; at = align64w(at + page_refs);
  l.cow_mask = at; at = align64w(at + page_refs);
  l.flags = at; at = align64w(at + page_refs);
  l.words = at;
  return l;
}
enum : int32_t { kRcHdrTok = 0, kRcHdrCow = 1, kRcHdrNeeded = 2, kRcHdrErr = 3, kRcHdrBySel = 4 };
enum : int32_t { kRcErrNoFree = 16 };   // error bit beyond the device error bits: too few free pages

struct RcPlanParams {
  BatchDev batch;
  const int32_t* topk_idx;
  const int32_t* k;
  const int32_t* free_pages;
  int32_t* page_ids_out;
  int32_t* plan;
  RcPlanLayout lay;
  int32_t k_cap, n_free, by_selection;
};
struct RcCopyParams {
  uint8_t* pool_k;
  uint8_t* pool_v;
  int32_t* plan;
  RcPlanLayout lay;
  int32_t layer, num_pages, num_kv_heads;
};
struct RcGemmParams {
  __nv_bfloat16* pool_k;
  __nv_bfloat16* pool_v;
  int32_t* plan;
  RcPlanLayout lay;
  int32_t layer, num_pages, num_kv_heads, d_model;
  int32_t x_rows;
  int32_t heads_per_tile;          // output heads per tile: 2 when num_kv_heads is even, else 1
  int64_t max_tok;
};

struct KvDecodeParams {
  __nv_bfloat16* pool_k;
  __nv_bfloat16* pool_v;
  const int32_t* chunk_tok_off;    // [n_chunks + 1]
  const int32_t* chunk_page_off;   // [n_chunks + 1]
  const int32_t* page_ids;         // [total pages]
  const uint8_t* codes_k;
  const uint8_t* codes_v;
  const float* scale_k;
  const float* offset_k;
  const float* scale_v;
  const float* offset_v;
  int32_t* err;
  int32_t layer, num_pages, num_kv_heads, n_chunks, bits;
};
cudaError_t launch_kv_decode(const KvDecodeParams&, int total_pages, cudaStream_t);

cudaError_t launch_rc_plan(const RcPlanParams&, cudaStream_t);
cudaError_t launch_rc_copy(const RcCopyParams&, int grid, cudaStream_t);
cudaError_t launch_rc_gemm(const CUtensorMap&, const CUtensorMap&, const CUtensorMap&, const CUtensorMap&,
                           const RcGemmParams&, int grid, cudaStream_t);

cudaError_t launch_attn_fwd(const CUtensorMap&, const CUtensorMap&, const CUtensorMap&, const CUtensorMap&,
                            const CUtensorMap&, const FwdParams&, int, cudaStream_t);
// max_block_rows: rows of the longest 256-row block of any request (max_q * G, at most 256)
cudaError_t launch_attn_combine(const CombineParams&, int max_rb, int max_block_rows, int num_requests,
                                cudaStream_t);
cudaError_t launch_rope_table(const BatchDev&, double base, float2* table, cudaStream_t);
// attention for query blocks of at most 16 rows (tq: a Q map whose box is those 16 rows)
cudaError_t launch_decode_attn(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                               const CUtensorMap& tkq, const CUtensorMap& tvq, const FwdParams& p, int grid,
                               cudaStream_t stream);
cudaError_t launch_impact(const CUtensorMap&, const CUtensorMap&, const CUtensorMap&, const ImpactParams&, int,
                          cudaStream_t);
cudaError_t launch_topk(const TopkParams&, int, int, cudaStream_t);
cudaError_t launch_simt_attn(const SimtParams&, int, cudaStream_t);
cudaError_t launch_simt_impact(const SimtParams&, int, int, cudaStream_t);
cudaError_t launch_pool_write(const PoolWriteParams&, int, cudaStream_t);

}  // namespace rag
