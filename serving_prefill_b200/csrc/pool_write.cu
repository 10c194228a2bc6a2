// Pool write: the on-device end of the offline precompute (TurboRAG page,
// "Technical Details": each chunk's per-layer K^(j), V^(j) are computed once
// and stored; the `precompute_kv_cache` listing keeps them per layer along
// the sequence axis). A chunk's dense [n_tokens][H_kv][d] K and V go to its
// pages of the pool [layers][pages][H_kv][16][d]: token t to page
// page_ids[t / 16], slot t % 16. The slots of the last page past the chunk's
// end are zeroed, so that a gathered tile holds only finite values.
//
// In a bf16 pool V is stored as fp16, the type in which it enters the product
// with the normalised weights: each bf16 value is rounded to the nearest fp16
// value (exact for magnitudes in [2^-14, 65280]); magnitudes from 65536 up,
// inf and nan saturate (nan stays nan) and raise kDevErrRange.
//
// One CTA per (page, kv head); each thread moves one 16-byte vector, so a
// 4 KB bf16 page row block is one fully coalesced read and write.
#include <cuda_runtime.h>

#include "params.cuh"

namespace rag {


__global__ void __launch_bounds__(256) pool_write_kernel(const PoolWriteParams p) {
  const int pi = blockIdx.x;           // page index within the chunk
  const int g = blockIdx.y;
  const int page = p.page_ids[pi];
  if (page < 0 || page >= p.num_pages) {
    if (threadIdx.x == 0 && p.err) atomicOr(p.err, kDevErrPage);
    return;
  }
  const int vec_per_row = p.row_bytes / 16;
  const int nvec = kPage * vec_per_row;
  const size_t dst_base =
      ((size_t(p.layer) * p.num_pages + page) * p.num_kv_heads + g) * kPage * size_t(p.row_bytes);
  uint32_t range = 0;
  for (int v = threadIdx.x; v < nvec; v += blockDim.x) {
    const int slot = v / vec_per_row;
    const int off = (v % vec_per_row) * 16;
    const int t = pi * kPage + slot;
    uint4 a = make_uint4(0, 0, 0, 0), c = make_uint4(0, 0, 0, 0);
    if (t < p.n_tokens) {
      const size_t src = (size_t(t) * p.num_kv_heads + g) * p.row_bytes + off;
      a = *reinterpret_cast<const uint4*>(p.k + src);
      c = *reinterpret_cast<const uint4*>(p.v + src);
    }
    if (p.v_to_f16) c = bf16x8_to_f16x8(c, range);
    const size_t dst = dst_base + size_t(slot) * p.row_bytes + off;
    *reinterpret_cast<uint4*>(p.pool_k + dst) = a;
    *reinterpret_cast<uint4*>(p.pool_v + dst) = c;
  }
  if (range_exceeded(range) && p.err) atomicOr(p.err, kDevErrRange);
}

cudaError_t launch_pool_write(const PoolWriteParams& p, int n_pages, cudaStream_t stream) {
  return launch_plain(pool_write_kernel, dim3(n_pages, p.num_kv_heads), dim3(256), 0, stream, p);
}

}  // namespace rag
