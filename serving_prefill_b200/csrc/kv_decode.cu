// Decode quantized chunk KV caches straight into the paged pool (CacheGen
// page, "How the technology works": a chunk's cache travels as a compact
// stream and is decoded on the GPU into a KV cache before generation; its
// glossary: quantization with different compression levels for different
// parts of the cache).
//
// Stream of one chunk, one layer: per token and KV head, head_dim codes of b
// bits (b = 8: one byte per channel; b = 4: two channels per byte, the even
// channel in the low nibble), with one fp32 (scale, offset) per KV head and
// channel. Value = fp32 fma(code, scale, offset), stored as bf16 in slot
// t % 16 of page page_ids[t / 16]; slots past the chunk's end are zeroed.
//
// One CTA per page of the batch: 16 slots x H_kv heads x 128 channels for K
// and for V; a thread makes 8 channels (one 16-byte store) at a time. The
// work is a stream from codes to pages, bound by HBM.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "params.cuh"

namespace rag {

constexpr int kDecThreads = 256;

__global__ void __launch_bounds__(kDecThreads) kv_decode_kernel(const KvDecodeParams p) {
  pdl_launch_dependents();
  const int gp = blockIdx.x;   // page of the batch
  // chunk of this page: last c with chunk_page_off[c] <= gp
  int lo = 0, hi = p.n_chunks - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldg(p.chunk_page_off + mid) <= gp) lo = mid; else hi = mid - 1;
  }
  const int c = lo;
  const int pg0 = __ldg(p.chunk_page_off + c), pg1 = __ldg(p.chunk_page_off + c + 1);
  const int t0 = __ldg(p.chunk_tok_off + c), t1 = __ldg(p.chunk_tok_off + c + 1);
  const int n_tok = t1 - t0;
  const int page = __ldg(p.page_ids + gp);
  pdl_wait();   // the pages may still be read or written by the kernel before this one
  if (gp < pg0 || gp >= pg1 || n_tok < 0 || (n_tok + kPage - 1) / kPage != pg1 - pg0) {
    if (threadIdx.x == 0 && p.err) atomicOr(p.err, kDevErrGeometry);
    return;
  }
  if (page < 0 || page >= p.num_pages) {
    if (threadIdx.x == 0 && p.err) atomicOr(p.err, kDevErrPage);
    return;
  }
  const int hk = p.num_kv_heads;
  const int code_row = kHeadDim * p.bits / 8;                  // bytes of one token and head
  const int units = 2 * kPage * hk * (kHeadDim / 8);            // 8-channel groups, K and V
  const int64_t page_base = (int64_t(p.layer) * p.num_pages + page) * hk * kPage * kHeadDim;
  for (int u = threadIdx.x; u < units; u += kDecThreads) {
    const int tensor = u / (units / 2);
    const int r = u % (units / 2);
    const int grp = r % (kHeadDim / 8);                         // channels 8 grp .. 8 grp + 7
    const int h = (r / (kHeadDim / 8)) % hk;
    const int slot = r / (kHeadDim / 8) / hk;
    const int t = (gp - pg0) * kPage + slot;                    // token of the chunk
    uint4 out = make_uint4(0u, 0u, 0u, 0u);
    if (t < n_tok) {
      const uint8_t* codes = (tensor ? p.codes_v : p.codes_k) + (int64_t(t0 + t) * hk + h) * code_row;
      uint32_t q[8];
      if (p.bits == 8) {
        const uint2 w = __ldg(reinterpret_cast<const uint2*>(codes + grp * 8));
#pragma unroll
        for (int j = 0; j < 4; ++j) { q[j] = (w.x >> (8 * j)) & 0xffu; q[4 + j] = (w.y >> (8 * j)) & 0xffu; }
      } else {
        const uint32_t w = __ldg(reinterpret_cast<const uint32_t*>(codes + grp * 4));
#pragma unroll
        for (int j = 0; j < 8; ++j) q[j] = (w >> (4 * j)) & 0xfu;
      }
      const int64_t sc = (int64_t(c) * hk + h) * kHeadDim + grp * 8;
      const float* scale = (tensor ? p.scale_v : p.scale_k) + sc;
      const float* offset = (tensor ? p.offset_v : p.offset_k) + sc;
      const float4 s0 = __ldg(reinterpret_cast<const float4*>(scale));
      const float4 s1 = __ldg(reinterpret_cast<const float4*>(scale) + 1);
      const float4 o0 = __ldg(reinterpret_cast<const float4*>(offset));
      const float4 o1 = __ldg(reinterpret_cast<const float4*>(offset) + 1);
      out.x = pack_bf16x2(__fmaf_rn(float(q[0]), s0.x, o0.x), __fmaf_rn(float(q[1]), s0.y, o0.y));
      out.y = pack_bf16x2(__fmaf_rn(float(q[2]), s0.z, o0.z), __fmaf_rn(float(q[3]), s0.w, o0.w));
      out.z = pack_bf16x2(__fmaf_rn(float(q[4]), s1.x, o1.x), __fmaf_rn(float(q[5]), s1.y, o1.y));
      out.w = pack_bf16x2(__fmaf_rn(float(q[6]), s1.z, o1.z), __fmaf_rn(float(q[7]), s1.w, o1.w));
    }
    __nv_bfloat16* pool = tensor ? p.pool_v : p.pool_k;
    reinterpret_cast<uint4*>(pool + page_base + (int64_t(h) * kPage + slot) * kHeadDim)[grp] = out;
  }
}

cudaError_t launch_kv_decode(const KvDecodeParams& p, int total_pages, cudaStream_t stream) {
  return launch_pdl(kv_decode_kernel, dim3(total_pages), dim3(kDecThreads), 0, stream, 1, p);
}

}  // namespace rag
