// Split-KV combine of the attention pass (TurboRAG page, "Technical Details":
// one softmax over the whole concatenated key sequence). When the attention
// kernel splits a unit's key tiles over several work items, each item leaves
// its own softmax average O_s/l_s (fp16), reference max m_s and sum l_s per
// row; this kernel merges them into the row's output and statistics.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "params.cuh"

namespace rag {

// Merge the split partials (O, m, l) of every row:
//   m = max_s m_s, l = sum_s l_s 2^(m_s - m), O = sum_s O_s 2^(m_s - m) / l.
// grid: x = (kv head * max row blocks + row block) * groups + group of 8 rows,
// y = request, with groups = 8-row groups of the longest row block of the
// batch (at most 32); one warp per row, each lane owns 4 of the 128 columns.
// The blocks start while the forward kernel runs; after its completion a row
// of the batch's first request costs one round of loads (the statistics and
// the O slice of up to 16 splits, all requested before any is used), a row of
// a later request one more (its first item's offset).
constexpr int kCombineRowsPerBlock = 8;
constexpr int kCombineBatch = 16;        // splits whose loads are in flight together

__global__ void __launch_bounds__(256, 4) attn_combine_kernel(const CombineParams p, int max_rb, int groups) {
  pdl_launch_dependents();
  // everything up to the partial loads depends on the batch descriptors only,
  // so it runs while the forward kernel finishes
  const int b = blockIdx.y;
  const int unit = blockIdx.x / groups;
  const int g = unit / max_rb;
  const int rb = unit % max_rb;
  const ReqInfo req = load_req(p.batch, b);
  const FwdShape sh = fwd_shape(p.batch, req, p.group, p.tiles_per_split);
  if (rb >= sh.n_rt || g >= p.num_kv_heads) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = p.group;
  const int rr = (blockIdx.x % groups) * kCombineRowsPerBlock + warp;   // row within the 256-row block
  const int pr = rb * kFwdRows + rr;
  const int tok = pr / G;
  if (tok >= req.n_q) return;   // uniform over the warp (one row per warp)
  const int head = g * G + pr % G;
  pdl_wait();   // partials and item offsets come from the forward kernel
  // first item of request b (the first request's is 0, no load needed)
  const int base = b == 0 ? 0 : __ldcg(p.item_prefix + b);
  const size_t first = size_t(base) + size_t(g) * sh.n_split * sh.n_rt + rb;
  if (first + size_t(sh.n_split - 1) * sh.n_rt >= size_t(p.max_items)) return;
  // split s weighs its own average O_s/l_s by l_s * 2^(m_s - m); lane j
  // holds the statistics of split s0 + j, every lane its 4 columns of each
  // split's O. Past the first 16 splits the running sums are rescaled to the
  // new maximum.
  const float* row0 = p.part + (first * kFwdRows + rr) * kPartStride;
  const size_t split_stride = size_t(sh.n_rt) * kFwdRows * kPartStride;
  constexpr int kStatOff = kHeadDim / 2;   // 32-bit word of m (then l) in a row
  float m = -INFINITY, l = 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int s0 = 0; s0 < sh.n_split; s0 += kCombineBatch) {
    const float2 ml = (lane < kCombineBatch && s0 + lane < sh.n_split)
                          ? __ldcg(reinterpret_cast<const float2*>(row0 + (s0 + lane) * split_stride + kStatOff))
                          : make_float2(-INFINITY, 0.f);
    uint2 v[kCombineBatch];
#pragma unroll
    for (int j = 0; j < kCombineBatch; ++j)
      v[j] = s0 + j < sh.n_split ? __ldcg(reinterpret_cast<const uint2*>(row0 + (s0 + j) * split_stride) + lane)
                                 : make_uint2(0u, 0u);
    float mb = fmaxf(m, ml.x);
    for (int o = 16; o > 0; o >>= 1) mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, o));
    const float mu = (mb == -INFINITY) ? 0.f : mb;
    if (s0 > 0) {
      const float sc = (m == -INFINITY) ? 0.f : ex2(m - mu);
      l *= sc;
      acc.x *= sc; acc.y *= sc; acc.z *= sc; acc.w *= sc;
    }
    m = mb;
    const float wl = (ml.x == -INFINITY) ? 0.f : ml.y * ex2(ml.x - mu);
#pragma unroll
    for (int j = 0; j < kCombineBatch; ++j) {
      const float wgt = __shfl_sync(0xffffffffu, wl, j);
      const float2 lo = __half22float2(*reinterpret_cast<const __half2*>(&v[j].x));
      const float2 hi = __half22float2(*reinterpret_cast<const __half2*>(&v[j].y));
      l += wgt;
      acc.x += lo.x * wgt; acc.y += lo.y * wgt; acc.z += hi.x * wgt; acc.w += hi.y * wgt;
    }
  }
  const float m_use = (m == -INFINITY) ? 0.f : m;
  const float inv = l > 0.f ? 1.f / l : 0.f;
  const int64_t orow = int64_t(req.q0 + tok) * p.num_q_heads + head;
  uint2 out;
  out.x = pack_bf16x2(acc.x * inv, acc.y * inv);
  out.y = pack_bf16x2(acc.z * inv, acc.w * inv);
  reinterpret_cast<uint2*>(p.o + orow * kHeadDim)[lane] = out;
  if (lane == 0) {
    p.row_m2[orow] = m_use;
    p.row_il[orow] = l > 0.f ? 1.f / (l * float(p.num_q_heads)) : 0.f;
    if (p.row_lse) p.row_lse[orow] = (m_use + __log2f(l)) * 0.69314718055994531f;
  }
}

cudaError_t launch_attn_combine(const CombineParams& p, int max_rb, int max_block_rows, int num_requests,
                                cudaStream_t stream) {
  const int rows = max_block_rows < 1 ? 1 : (max_block_rows > kFwdRows ? kFwdRows : max_block_rows);
  const int groups = (rows + kCombineRowsPerBlock - 1) / kCombineRowsPerBlock;
  dim3 grid(p.num_kv_heads * max_rb * groups, num_requests);
  return launch_pdl(attn_combine_kernel, grid, dim3(256), 0, stream, 1, p, max_rb, groups);
}

}  // namespace rag
