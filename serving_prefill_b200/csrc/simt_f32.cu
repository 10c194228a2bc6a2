// fp32 path (pool stored in fp32): plain CUDA-core kernels for the same
// gather -> masked attention -> Impact steps. The tensor cores have no fp32
// input format that meets a 1e-5 relative bound (TF32 keeps 10 mantissa
// bits), so this path uses FFMA. It serves small fp32 problems: every
// request's n_doc + q must fit the kSimtMaxKeys score buffer.
#include <cuda_runtime.h>

#include "params.cuh"

namespace rag {

constexpr int kSimtThreads = 128;
constexpr int kSimtMaxKeys = 8192;


__device__ __forceinline__ int request_of_token(const BatchDev& B, int tok) {
  int lo = 0, hi = B.num_requests - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (__ldg(B.q_off + mid) <= tok) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// Address of key/value i (logical position in [K_1;...;K_m;K_q]) of kv head g.
// Doc keys go through the page table; returns -1 for an invalid page.
__device__ __forceinline__ int64_t simt_key_row(const SimtParams& p, const ReqInfo& r, int g, int i,
                                                bool* is_query) {
  if (i >= r.n_doc) {
    *is_query = true;
    return (int64_t(r.q0 + i - r.n_doc) * p.num_kv_heads + g) * p.head_dim;
  }
  *is_query = false;
  const int pos = r.doc0 + i;
  int lo = r.c0, hi = r.c1 - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (__ldg(p.batch.chunk_doc_off + mid) <= pos) lo = mid; else hi = mid - 1;
  }
  const int t = pos - __ldg(p.batch.chunk_doc_off + lo);
  const int ref = __ldg(p.batch.chunk_page_off + lo) + t / kPage;
  if (ref >= __ldg(p.batch.chunk_page_off + lo + 1)) {
    atomicOr(p.err, kDevErrGeometry);
    return -1;
  }
  const int page = __ldg(p.batch.page_ids + ref);
  if (page < 0 || page >= p.num_pages) {
    atomicOr(p.err, kDevErrPage);
    return -1;
  }
  return ((int64_t(p.layer) * p.num_pages + page) * p.num_kv_heads * kPage + int64_t(g) * kPage + t % kPage) *
         p.head_dim;
}

__device__ __forceinline__ float block_reduce(float v, float* red, bool is_max) {
  for (int o = 16; o > 0; o >>= 1) {
    const float w = __shfl_xor_sync(0xffffffffu, v, o);
    v = is_max ? fmaxf(v, w) : v + w;
  }
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  v = red[0];
  for (int w = 1; w < kSimtThreads / 32; ++w) v = is_max ? fmaxf(v, red[w]) : v + red[w];
  return v;
}

// grid (total_q, H_q): one row (query token, head) per CTA
__global__ void __launch_bounds__(kSimtThreads) simt_attn_kernel(const SimtParams p) {
  extern __shared__ float sm[];
  float* sq = sm;                                  // [d]
  float* sp = sq + p.head_dim;                     // [kSimtMaxKeys] scores, then weights
  int64_t* srow = reinterpret_cast<int64_t*>(sp + kSimtMaxKeys);  // [kSimtMaxKeys] key rows
  __shared__ float red[kSimtThreads / 32];
  const int tok = blockIdx.x, h = blockIdx.y, tid = threadIdx.x, d = p.head_dim;
  const int b = request_of_token(p.batch, tok);
  const ReqInfo r = load_req(p.batch, b);
  if (!req_ok(p.batch, r)) {
    if (threadIdx.x == 0) atomicOr(p.err, kDevErrGeometry);
    return;
  }
  const int j = tok - r.q0;
  const int g = h / p.group;
  const int nvis = r.n_doc + j + 1;               // keys 0 .. n_doc + j
  const int64_t qrow = (int64_t(tok) * p.num_q_heads + h) * d;
  for (int x = tid; x < d; x += kSimtThreads) sq[x] = p.q[qrow + x];
  __syncthreads();
  float mx = -INFINITY;
  for (int i = tid; i < nvis; i += kSimtThreads) {
    bool isq;
    const int64_t row = simt_key_row(p, r, g, i, &isq);
    srow[i] = isq ? -(row + 1) : row;
    float s = -INFINITY;
    if (row >= 0) {
      const float* kp = isq ? p.kq + row : p.pool_k + row;
      float acc = 0.f;
      for (int x = 0; x < d; ++x) acc = fmaf(sq[x], kp[x], acc);
      s = acc * p.scale;
    }
    sp[i] = s;
    mx = fmaxf(mx, s);
  }
  const float m = block_reduce(mx, red, true);
  float ls = 0.f;
  for (int i = tid; i < nvis; i += kSimtThreads) {
    const float e = expf(sp[i] - m);
    sp[i] = e;
    ls += e;
  }
  const float l = block_reduce(ls, red, false);
  __syncthreads();
  const float inv = 1.f / l;
  for (int x = tid; x < d; x += kSimtThreads) {
    float acc = 0.f;
    for (int i = 0; i < nvis; ++i) {
      const int64_t row = srow[i];
      const float* vp = row >= 0 ? p.pool_v + row : p.vq + (-row - 1);
      acc = fmaf(sp[i], vp[x], acc);
    }
    p.o[qrow + x] = acc * inv;
  }
  if (tid == 0) {
    const int64_t ri = int64_t(tok) * p.num_q_heads + h;
    p.row_m[ri] = m;
    p.row_l[ri] = l;
    if (p.row_lse) p.row_lse[ri] = m + logf(l);
  }
}

// grid (max keys per request, B): Impact of one key, summed over every
// (head, query token) row that sees it, divided by H_q.
__global__ void __launch_bounds__(kSimtThreads) simt_impact_kernel(const SimtParams p) {
  extern __shared__ float sk[];   // [d]
  __shared__ float red[kSimtThreads / 32];
  const int i = blockIdx.x, b = blockIdx.y, tid = threadIdx.x, d = p.head_dim;
  const ReqInfo r = load_req(p.batch, b);
  if (!req_ok(p.batch, r) || i >= r.n_doc + r.n_q) return;
  float acc = 0.f;
  for (int g = 0; g < p.num_kv_heads; ++g) {
    bool isq;
    const int64_t row = simt_key_row(p, r, g, i, &isq);
    __syncthreads();
    for (int x = tid; x < d; x += kSimtThreads) sk[x] = row >= 0 ? (isq ? p.kq[row + x] : p.pool_k[row + x]) : 0.f;
    __syncthreads();
    if (row < 0) continue;
    const int j0 = i >= r.n_doc ? i - r.n_doc : 0;   // first query token that sees key i
    const int nrows = p.group * (r.n_q - j0);
    for (int e = tid; e < nrows; e += kSimtThreads) {
      const int j = j0 + e / p.group;
      const int h = g * p.group + e % p.group;
      const int64_t ri = int64_t(r.q0 + j) * p.num_q_heads + h;
      const float* qp = p.q + ri * d;
      float s = 0.f;
      for (int x = 0; x < d; ++x) s = fmaf(qp[x], sk[x], s);
      acc += expf(s * p.scale - p.row_m[ri]) / p.row_l[ri];
    }
  }
  const float tot = block_reduce(acc, red, false);
  if (tid == 0) p.impact[r.doc0 + r.q0 + i] = tot / float(p.num_q_heads);
}

cudaError_t launch_simt_attn(const SimtParams& p, int total_q, cudaStream_t stream) {
  const size_t smem = sizeof(float) * (p.head_dim + kSimtMaxKeys) + sizeof(int64_t) * kSimtMaxKeys;
  static SmemAttr attr;
  cudaError_t e = ensure_smem_attr(simt_attn_kernel, attr, smem);
  if (e != cudaSuccess) return e;
  return launch_plain(simt_attn_kernel, dim3(total_q, p.num_q_heads), dim3(kSimtThreads), smem, stream, p);
}

cudaError_t launch_simt_impact(const SimtParams& p, int max_keys, int num_requests, cudaStream_t stream) {
  return launch_plain(simt_impact_kernel, dim3(max_keys, num_requests), dim3(kSimtThreads), sizeof(float) * p.head_dim,
                      stream, p);
}

}  // namespace rag
