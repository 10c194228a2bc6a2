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
constexpr int kBatch = 8;    // keys in flight per thread per radix pass
constexpr int kTopkMaxSort = 8192;   // requests up to this many doc tokens are sorted whole
constexpr int kTopkCand = 8192;      // candidates of the k-th key's bucket kept in shared memory


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

// Histogram of one digit of every key that matches (prefix, mask), read from
// global memory in coalesced batches; warp-aggregated shared-memory atomics.
__device__ __forceinline__ void digit_histogram(const float* keys, int n, uint32_t prefix, uint32_t mask,
                                                int shift, int nbins, uint32_t* hist) {
  const int tid = threadIdx.x, lane = tid & 31;
  for (int i = tid; i < nbins; i += kTopkThreads) hist[i] = 0;
  __syncthreads();
  for (int base = 0; base < n; base += kTopkThreads * kBatch) {
    uint32_t u[kBatch];
#pragma unroll
    for (int j = 0; j < kBatch; ++j) {
      const int i = base + j * kTopkThreads + tid;
      u[j] = i < n ? impact_key(__ldg(keys + i)) : 0u;
    }
#pragma unroll
    for (int j = 0; j < kBatch; ++j) {
      const int i = base + j * kTopkThreads + tid;
      const bool in = i < n && (u[j] & mask) == prefix;
      const uint32_t dig = (u[j] >> shift) & uint32_t(nbins - 1);
      const uint32_t act = __ballot_sync(0xffffffffu, in);
      if (in) {
        const uint32_t same = __match_any_sync(act, dig);
        if ((__ffs(same) - 1) == lane) atomicAdd(&hist[dig], uint32_t(__popc(same)));
      }
    }
  }
  __syncthreads();
}

// The digit holding the kr-th largest key (counting from the top bin down):
// sel[0] = digit, sel[1] = rank of the wanted key inside that digit's bin.
__device__ __forceinline__ void select_digit(const uint32_t* hist, int nbins, uint32_t kr, uint32_t* sel,
                                             int* warp_sums) {
  const int tid = threadIdx.x;
  const int per = nbins / kTopkThreads > 0 ? nbins / kTopkThreads : 1;
  const int hi_bin = nbins - 1 - tid * per;     // this thread's bins: hi_bin .. hi_bin - per + 1
  uint32_t mine = 0;
  if (tid * per < nbins)
    for (int j = 0; j < per; ++j) mine += hist[hi_bin - j];
  const int incl = block_scan_incl(int(mine), warp_sums);
  const uint32_t before = uint32_t(incl) - mine;
  if (tid * per < nbins && before < kr && uint32_t(incl) >= kr) {
    uint32_t cum = before;
    for (int j = 0; j < per; ++j) {
      const uint32_t h = hist[hi_bin - j];
      if (cum + h >= kr) { sel[0] = uint32_t(hi_bin - j); sel[1] = kr - cum; break; }
      cum += h;
    }
  }
  __syncthreads();
}

__global__ void __launch_bounds__(kTopkThreads) topk_kernel(const TopkParams p) {
  extern __shared__ uint64_t smem_topk[];
  uint64_t* sort_buf = smem_topk;                  // [kTopkMaxSort]
  uint64_t* cand = smem_topk + kTopkMaxSort;       // [kTopkCand]
  __shared__ uint32_t hist[kTopkBins];
  __shared__ uint32_t s_sel[2];
  __shared__ uint32_t s_cnt[2];
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
  if (n <= kTopkMaxSort) {
    // ---- short request: sort every doc token
    while (kp < n) kp <<= 1;
    for (int i = tid; i < kp; i += kTopkThreads) sort_buf[i] = i < n ? composite(impact_key(keys[i]), i) : ~0ull;
    __syncthreads();
    bitonic_sort(sort_buf, kp);
  } else {
    // ---- long request. Pass 1: the 12-bit bucket (sign, exponent, 3 mantissa
    // bits) that holds the k-th largest key, and how many keys lie above it.
    digit_histogram(keys, n, 0u, 0u, 20, kTopkBins, hist);
    select_digit(hist, kTopkBins, uint32_t(k), s_sel, warp_sums);
    const uint32_t d1 = s_sel[0];
    const int kr1 = int(s_sel[1]);
    const int n_gt1 = k - kr1;
    if (tid == 0) { s_cnt[0] = 0; s_cnt[1] = 0; }
    __syncthreads();
    // Pass 2: keys above the bucket go straight to the output buffer; keys in
    // it are gathered as candidates.
    for (int base = 0; base < n; base += kTopkThreads * kBatch) {
      uint32_t u[kBatch];
#pragma unroll
      for (int j = 0; j < kBatch; ++j) {
        const int i = base + j * kTopkThreads + tid;
        u[j] = i < n ? impact_key(__ldg(keys + i)) : 0u;
      }
#pragma unroll
      for (int j = 0; j < kBatch; ++j) {
        const int i = base + j * kTopkThreads + tid;
        if (i >= n) continue;
        const uint32_t dig = u[j] >> 20;
        if (dig > d1) {
          sort_buf[atomicAdd(&s_cnt[0], 1u)] = composite(u[j], i);
        } else if (dig == d1) {
          const uint32_t c = atomicAdd(&s_cnt[1], 1u);
          if (c < uint32_t(kTopkCand)) cand[c] = composite(u[j], i);
        }
      }
    }
    __syncthreads();
    const int nc = int(s_cnt[1]);
    if (nc <= kTopkCand) {
      // Sort the candidates (ties by position) and keep the best kr1.
      int cp = 1;
      while (cp < nc) cp <<= 1;
      for (int i = nc + tid; i < cp; i += kTopkThreads) cand[i] = ~0ull;
      __syncthreads();
      bitonic_sort(cand, cp);
      for (int i = tid; i < kr1; i += kTopkThreads) sort_buf[n_gt1 + i] = cand[i];
    } else {
      // Too many keys share the bucket: exact radix select on the low 20 bits
      // over global memory, then index-ordered compaction.
      uint32_t prefix = d1 << 20, mask = 0xfff00000u, kr = uint32_t(kr1);
      for (int pass = 0; pass < 2; ++pass) {
        const int shift = pass == 0 ? 8 : 0;
        const int bits = pass == 0 ? 12 : 8;
        const int nbins = 1 << bits;
        digit_histogram(keys, n, prefix, mask, shift, nbins, hist);
        select_digit(hist, nbins, kr, s_sel, warp_sums);
        prefix |= s_sel[0] << shift;
        mask |= uint32_t(nbins - 1) << shift;
        kr = s_sel[1];
        __syncthreads();
      }
      const uint32_t T = prefix;
      const int n_gt = k - int(kr);
      if (tid == 0) { s_sel[0] = uint32_t(n_gt1); s_sel[1] = 0; }   // keys > T already placed: those above d1
      __syncthreads();
      for (int base = 0; base < n; base += kTopkThreads) {
        const int i = base + tid;
        const uint32_t u = i < n ? impact_key(__ldg(keys + i)) : 0u;
        const bool in_bucket = i < n && (u >> 20) == d1;
        const bool gt = in_bucket && u > T;
        const bool eq = in_bucket && u == T;
        if (gt) sort_buf[atomicAdd(&s_sel[0], 1u)] = composite(u, i);
        const int eq_incl = block_scan_incl(eq ? 1 : 0, warp_sums);
        const uint32_t seen = s_sel[1];
        const uint32_t rank = seen + uint32_t(eq_incl) - (eq ? 1u : 0u);
        if (eq && rank < kr) sort_buf[n_gt + rank] = composite(u, i);
        __syncthreads();
        if (tid == kTopkThreads - 1) s_sel[1] = seen + uint32_t(eq_incl);
        __syncthreads();
        if (s_sel[1] >= kr && s_sel[0] >= uint32_t(n_gt)) break;
      }
    }
    while (kp < k) kp <<= 1;
    for (int i = k + tid; i < kp; i += kTopkThreads) sort_buf[i] = ~0ull;
    __syncthreads();
    bitonic_sort(sort_buf, kp);
  }
  for (int i = tid; i < k; i += kTopkThreads) {
    const uint64_t comp = sort_buf[i];
    out_idx[i] = int32_t(comp & 0xffffffffu);
    if (out_val) out_val[i] = __uint_as_float(~uint32_t(comp >> 32));
  }
}

cudaError_t launch_topk(const TopkParams& p, int num_requests, int max_k, cudaStream_t stream) {
  (void)max_k;
  const size_t smem = sizeof(uint64_t) * size_t(kTopkMaxSort + kTopkCand);
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
