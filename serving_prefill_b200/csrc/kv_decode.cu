// Decode quantized chunk KV caches straight into the paged pool (CacheGen
// page, "How the technology works": a chunk's cache travels as a compact
// stream and is decoded on the GPU into a KV cache before generation; its
// glossary: quantization with different compression levels for different
// parts of the cache).
//
// Stream of one chunk, one layer: per token and KV head, head_dim codes of b
// bits (b = 8: one byte per channel; b = 4: two channels per byte, the even
// channel in the low nibble), with one fp32 (scale, offset) per KV head and
// channel. Value = fp32 fma(code, scale, offset), rounded once to the type the
// pool stores it in (K bf16, V fp16: nearest even, V saturated beyond 65504
// with kDevErrRange raised) and stored in slot t % 16 of page page_ids[t / 16];
// slots past the chunk's end are zeroed.
//
// One CTA per page of the batch: 16 slots x H_kv heads x 128 channels for K
// and for V; a thread makes 8 channels of one head (16-byte stores) for all 16
// slots. The work is a stream from codes to pages, bound by HBM.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "params.cuh"

namespace rag {

constexpr int kDecThreads = 256;

// 8 channels of one KV head for the 16 slots of a page: codes -> fp32 value
// fma(code, scale, offset) -> the stored type, rounded once (K: bf16; V:
// fp16, saturated). A decoded value is linear in its code and rounding is
// monotonic, so a group whose two end values (code 0 and code 2^b - 1) are
// within the fp16 range has no V value to check one by one (a nan scale or
// offset fails that test).
template <bool kV>
__device__ __forceinline__ void decode_unit(const KvDecodeParams& p, const uint8_t* codes, int64_t token_stride,
                                            int grp, int n_valid, const float* scale_p, const float* offset_p,
                                            uint4* out, bool& over) {
  const float4 s0 = __ldg(reinterpret_cast<const float4*>(scale_p));
  const float4 s1 = __ldg(reinterpret_cast<const float4*>(scale_p) + 1);
  const float4 o0 = __ldg(reinterpret_cast<const float4*>(offset_p));
  const float4 o1 = __ldg(reinterpret_cast<const float4*>(offset_p) + 1);
  bool check = false;
  if (kV) {
    const float top = float((1 << p.bits) - 1);
    check = beyond_f16(o0.x) || beyond_f16(o0.y) || beyond_f16(o0.z) || beyond_f16(o0.w) ||
            beyond_f16(o1.x) || beyond_f16(o1.y) || beyond_f16(o1.z) || beyond_f16(o1.w) ||
            beyond_f16(__fmaf_rn(top, s0.x, o0.x)) || beyond_f16(__fmaf_rn(top, s0.y, o0.y)) ||
            beyond_f16(__fmaf_rn(top, s0.z, o0.z)) || beyond_f16(__fmaf_rn(top, s0.w, o0.w)) ||
            beyond_f16(__fmaf_rn(top, s1.x, o1.x)) || beyond_f16(__fmaf_rn(top, s1.y, o1.y)) ||
            beyond_f16(__fmaf_rn(top, s1.z, o1.z)) || beyond_f16(__fmaf_rn(top, s1.w, o1.w));
  }
  uint2 cw[kPage];
#pragma unroll
  for (int slot = 0; slot < kPage; ++slot) {
    cw[slot] = make_uint2(0u, 0u);
    if (slot >= n_valid) continue;
    const uint8_t* cs = codes + slot * token_stride;
    if (p.bits == 8) cw[slot] = __ldg(reinterpret_cast<const uint2*>(cs + grp * 8));
    else cw[slot].x = __ldg(reinterpret_cast<const uint32_t*>(cs + grp * 4));
  }
#pragma unroll
  for (int slot = 0; slot < kPage; ++slot) {
    uint4 v = make_uint4(0u, 0u, 0u, 0u);   // slots past the chunk's end are zeroed
    if (slot < n_valid) {
      float q[8];
      if (p.bits == 8) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          q[i] = float((cw[slot].x >> (8 * i)) & 0xffu);
          q[4 + i] = float((cw[slot].y >> (8 * i)) & 0xffu);
        }
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) q[i] = float((cw[slot].x >> (4 * i)) & 0xfu);
      }
      const float y0 = __fmaf_rn(q[0], s0.x, o0.x), y1 = __fmaf_rn(q[1], s0.y, o0.y);
      const float y2 = __fmaf_rn(q[2], s0.z, o0.z), y3 = __fmaf_rn(q[3], s0.w, o0.w);
      const float y4 = __fmaf_rn(q[4], s1.x, o1.x), y5 = __fmaf_rn(q[5], s1.y, o1.y);
      const float y6 = __fmaf_rn(q[6], s1.z, o1.z), y7 = __fmaf_rn(q[7], s1.w, o1.w);
      if (kV) {
        if (check)
          over |= beyond_f16(y0) || beyond_f16(y1) || beyond_f16(y2) || beyond_f16(y3) || beyond_f16(y4) ||
                  beyond_f16(y5) || beyond_f16(y6) || beyond_f16(y7);
        v = make_uint4(pack_f16x2_sat(y0, y1), pack_f16x2_sat(y2, y3), pack_f16x2_sat(y4, y5),
                       pack_f16x2_sat(y6, y7));
      } else {
        v = make_uint4(pack_bf16x2(y0, y1), pack_bf16x2(y2, y3), pack_bf16x2(y4, y5), pack_bf16x2(y6, y7));
      }
    }
    out[slot * (kHeadDim / 8)] = v;
  }
}

__global__ void __launch_bounds__(kDecThreads, 3) kv_decode_kernel(const KvDecodeParams p) {
  // no early release: the attention kernel reads pool pages before its own
  // wait, so it must start only once every page written here is complete
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
  const int64_t page_base = (int64_t(p.layer) * p.num_pages + page) * hk * kPage * kHeadDim;
  const int n_valid = min(kPage, n_tok - (gp - pg0) * kPage);   // slots of this page holding tokens
  const int t_first = t0 + (gp - pg0) * kPage;
  // A thread owns one (tensor, KV head, 8-channel group): its scale and offset
  // are loaded once, then the codes of all 16 slots are loaded before the
  // first value is computed (16 loads in flight), and 16 stores follow.
  bool over = false;   // a V value saturated
  for (int u = threadIdx.x; u < 2 * hk * (kHeadDim / 8); u += kDecThreads) {
    const int tensor = u / (hk * (kHeadDim / 8));
    const int h = (u / (kHeadDim / 8)) % hk;
    const int grp = u % (kHeadDim / 8);                        // channels 8 grp .. 8 grp + 7
    const int64_t so = (int64_t(c) * hk + h) * kHeadDim + grp * 8;
    const uint8_t* codes = (tensor ? p.codes_v : p.codes_k) + (int64_t(t_first) * hk + h) * code_row;
    uint4* out = reinterpret_cast<uint4*>((tensor ? p.pool_v : p.pool_k) + page_base) + h * kPage * (kHeadDim / 8) + grp;
    if (tensor)
      decode_unit<true>(p, codes, hk * code_row, grp, n_valid, p.scale_v + so, p.offset_v + so, out, over);
    else
      decode_unit<false>(p, codes, hk * code_row, grp, n_valid, p.scale_k + so, p.offset_k + so, out, over);
  }
  if (over && p.err) atomicOr(p.err, kDevErrRange);
}

cudaError_t launch_kv_decode(const KvDecodeParams& p, int total_pages, cudaStream_t stream) {
  return launch_pdl(kv_decode_kernel, dim3(total_pages), dim3(kDecThreads), 0, stream, 1, p);
}

}  // namespace rag
