// Recompute selection (CacheBlend page, "Recompute ratio trade-off": the
// number of recomputed tokens is r times the total doc length; the listing
// takes max(1, int(doc_token_count * ratio)) and torch.topk over the doc slice
// of the impact vector).
//
// One CTA per request: an exact 4-pass radix select (8 bits per pass) over
// the fp32 impact bits finds the k-th largest value T; the CTA then keeps
// every doc token above T and the lowest-index tokens equal to T, and sorts
// the k survivors by (impact descending, position ascending) with a bitonic
// network in shared memory. Impacts are >= 0, so their IEEE bit patterns
// order like the values.
#include <cuda_runtime.h>

#include "params.cuh"

namespace rag {

constexpr int kTopkThreads = 1024;
constexpr int kTopkBins = 4096;


__device__ __forceinline__ uint32_t impact_key(float v) {
  const uint32_t u = __float_as_uint(v);
  return (u >> 31) ? 0u : u;   // -0 and negatives (never produced) sort as 0
}

// inclusive block scan of one int per thread (1024 threads)
__device__ __forceinline__ int block_scan_incl(int v, int* warp_sums) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_sums[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int s = warp_sums[lane];
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    warp_sums[lane] = s;
  }
  __syncthreads();
  const int add = warp > 0 ? warp_sums[warp - 1] : 0;
  __syncthreads();
  return x + add;
}

// Bitonic sort of kp (power of two) composite keys in shared memory, ascending.
__device__ __forceinline__ void bitonic_sort(uint64_t* a, int kp) {
  for (int size = 2; size <= kp; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = threadIdx.x; i < (kp >> 1); i += kTopkThreads) {
        const int lo = 2 * i - (i & (stride - 1));
        const int hi = lo + stride;
        const bool asc = (lo & size) == 0;
        const uint64_t x = a[lo], y = a[hi];
        if ((x > y) == asc) { a[lo] = y; a[hi] = x; }
      }
      __syncthreads();
    }
  }
}

// Composite sort key: ascending order = impact descending, position ascending.
__device__ __forceinline__ uint64_t composite(uint32_t key, int i) { return (uint64_t(~key) << 32) | uint32_t(i); }

__global__ void __launch_bounds__(kTopkThreads) topk_kernel(const TopkParams p) {
  extern __shared__ uint64_t sort_buf[];
  __shared__ uint32_t hist[kTopkBins];
  __shared__ uint32_t s_sel[2];
  __shared__ int warp_sums[32];
  const int b = blockIdx.x;
  const int tid = threadIdx.x;
  const ReqInfo req = load_req(p.batch, b);
  const bool ok = req_ok(p.batch, req);
  const int n = ok ? req.n_doc : 0;
  const float* keys = p.impact + (req.doc0 + req.q0);
  int k = n > 0 ? max(1, int(double(n) * p.r)) : 0;
  k = min(min(k, n), min(p.k_cap, p.k_max));
  int32_t* out_idx = p.topk_idx + int64_t(b) * p.k_cap;
  float* out_val = p.topk_val ? p.topk_val + int64_t(b) * p.k_cap : nullptr;
  if (p.k_out && tid == 0) p.k_out[b] = k;
  for (int i = k + tid; i < p.k_cap; i += kTopkThreads) {
    out_idx[i] = -1;
    if (out_val) out_val[i] = 0.f;
  }
  if (k == 0) return;

  int kp = 1;
  if (n <= p.sort_cap) {
    // ---- small request: sort every doc token
    while (kp < n) kp <<= 1;
    for (int i = tid; i < kp; i += kTopkThreads) sort_buf[i] = i < n ? composite(impact_key(keys[i]), i) : ~0ull;
    __syncthreads();
  } else {
    // ---- radix select over 12 + 12 + 8 bits: the k-th largest key T and the
    // number of keys equal to T that belong to the top k
    uint32_t prefix = 0, mask = 0, kr = uint32_t(k);
    const int lane = tid & 31;
    for (int pass = 0; pass < 3; ++pass) {
      const int shift = pass == 0 ? 20 : (pass == 1 ? 8 : 0);
      const int bits = pass < 2 ? 12 : 8;
      const int nbins = 1 << bits;
      for (int i = tid; i < nbins; i += kTopkThreads) hist[i] = 0;
      __syncthreads();
      for (int base = 0; base < n; base += kTopkThreads) {
        const int i = base + tid;
        uint32_t u = i < n ? impact_key(keys[i]) : 0u;
        const bool in = i < n && (u & mask) == prefix;
        const uint32_t dig = (u >> shift) & uint32_t(nbins - 1);
        // warp-aggregated increment: one atomic per distinct digit in the warp
        const uint32_t act = __ballot_sync(0xffffffffu, in);
        if (in) {
          const uint32_t same = __match_any_sync(act, dig);
          if ((__ffs(same) - 1) == lane) atomicAdd(&hist[dig], uint32_t(__popc(same)));
        }
      }
      __syncthreads();
      // bins per thread, scanned from the largest digit down
      const int per = nbins / kTopkThreads > 0 ? nbins / kTopkThreads : 1;
      const int hi_bin = nbins - 1 - tid * per;          // this thread's bins: hi_bin .. hi_bin - per + 1
      uint32_t mine = 0;
      if (tid * per < nbins)
        for (int j = 0; j < per; ++j) mine += hist[hi_bin - j];
      const int incl = block_scan_incl(int(mine), warp_sums);
      const uint32_t before = uint32_t(incl) - mine;
      if (tid * per < nbins && before < kr && uint32_t(incl) >= kr) {
        uint32_t cum = before;
        for (int j = 0; j < per; ++j) {
          const uint32_t h = hist[hi_bin - j];
          if (cum + h >= kr) { s_sel[0] = uint32_t(hi_bin - j); s_sel[1] = kr - cum; break; }
          cum += h;
        }
      }
      __syncthreads();
      prefix |= s_sel[0] << shift;
      mask |= uint32_t(nbins - 1) << shift;
      kr = s_sel[1];
      __syncthreads();
    }
    const uint32_t T = prefix;
    const int n_gt = k - int(kr);
    // ---- compaction in index order: all keys > T, the first kr keys == T
    const int per = (n + kTopkThreads - 1) / kTopkThreads;
    const int i0 = min(n, tid * per), i1 = min(n, i0 + per);
    int c_gt = 0, c_eq = 0;
    for (int i = i0; i < i1; ++i) {
      const uint32_t u = impact_key(keys[i]);
      c_gt += u > T;
      c_eq += u == T;
    }
    const int gt_incl = block_scan_incl(c_gt, warp_sums);
    const int eq_incl = block_scan_incl(c_eq, warp_sums);
    int pos_gt = gt_incl - c_gt, pos_eq = eq_incl - c_eq;
    for (int i = i0; i < i1; ++i) {
      const uint32_t u = impact_key(keys[i]);
      if (u > T) {
        sort_buf[pos_gt++] = composite(u, i);
      } else if (u == T) {
        if (pos_eq < int(kr)) sort_buf[n_gt + pos_eq] = composite(u, i);
        ++pos_eq;
      }
    }
    while (kp < k) kp <<= 1;
    for (int i = k + tid; i < kp; i += kTopkThreads) sort_buf[i] = ~0ull;
    __syncthreads();
  }
  bitonic_sort(sort_buf, kp);
  for (int i = tid; i < k; i += kTopkThreads) {
    const uint64_t comp = sort_buf[i];
    out_idx[i] = int32_t(comp & 0xffffffffu);
    if (out_val) out_val[i] = __uint_as_float(~uint32_t(comp >> 32));
  }
}

cudaError_t launch_topk(const TopkParams& p, int num_requests, int max_k, cudaStream_t stream) {
  // the buffer holds either all doc tokens of a request (up to sort_cap) or its k survivors
  int kp = 1;
  while (kp < max_k || kp < p.sort_cap) kp <<= 1;
  const size_t smem = sizeof(uint64_t) * size_t(kp);
  static size_t attr_set = 0;   // largest dynamic smem size configured so far
  if (smem > attr_set) {
    cudaError_t e = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    if (e != cudaSuccess) return e;
    attr_set = smem;
  }
  topk_kernel<<<num_requests, kTopkThreads, smem, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace rag
