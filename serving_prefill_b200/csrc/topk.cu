// Recompute selection (CacheBlend page, "Recompute ratio trade-off": the
// number of recomputed tokens is r times the total doc length; the listing
// takes max(1, int(doc_token_count * ratio)) and torch.topk over the doc slice
// of the impact vector).
//
// One CTA per request. A histogram of the top 12 bits of the fp32 impacts
// (impacts are >= 0, so their bit patterns order like the values) finds the
// bucket holding the k-th largest value; keys above it are scattered into
// their buckets' ranges in descending bucket order, and the keys inside it
// become candidates. Candidates and each bucket's keys are then ordered by
// counting ranks of the composite key (impact descending, position
// ascending); a bitonic network in shared memory takes over for long runs,
// and an exact radix select handles a bucket too full to stage.
#include <cuda_runtime.h>

#include "params.cuh"

namespace rag {

constexpr int kTopkThreads = 1024;
constexpr int kTopkBins = 4096;
constexpr int kBatch = 8;    // keys in flight per thread per radix pass
constexpr int kTopkMaxSort = 8192;   // requests up to this many doc tokens are sorted whole
constexpr int kTopkCand = 8192;      // candidates of the k-th key's bucket kept in shared memory
constexpr int kTopkRankMax = 512;    // runs up to this long are ordered by counting ranks


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
// When `start` is given it receives, per bin, the number of keys in the bins
// above it (where that bin's keys begin in descending order).
__device__ __forceinline__ void select_digit(const uint32_t* hist, int nbins, uint32_t kr, uint32_t* sel,
                                             int* warp_sums, uint32_t* start) {
  const int tid = threadIdx.x;
  const int per = nbins / kTopkThreads > 0 ? nbins / kTopkThreads : 1;
  const int hi_bin = nbins - 1 - tid * per;     // this thread's bins: hi_bin .. hi_bin - per + 1
  uint32_t mine = 0;
  if (tid * per < nbins)
    for (int j = 0; j < per; ++j) mine += hist[hi_bin - j];
  const int incl = block_scan_incl(int(mine), warp_sums);
  const uint32_t before = uint32_t(incl) - mine;
  if (tid * per < nbins) {
    uint32_t cum = before;
    bool found = !(before < kr && uint32_t(incl) >= kr);
    for (int j = 0; j < per; ++j) {
      const uint32_t h = hist[hi_bin - j];
      if (start) start[hi_bin - j] = cum;
      if (!found && cum + h >= kr) { sel[0] = uint32_t(hi_bin - j); sel[1] = kr - cum; found = true; }
      cum += h;
    }
  }
  __syncthreads();
}

// Position of composite key c among the sorted run a[s, e) of distinct keys.
__device__ __forceinline__ int rank_in(const uint64_t* a, int s, int e, uint64_t c) {
  int r = 0;
  for (int j = s; j < e; ++j) r += a[j] < c;
  return r;
}

__global__ void __launch_bounds__(kTopkThreads, 1) topk_kernel(const TopkParams p) {
  extern __shared__ uint64_t smem_topk[];
  uint64_t* sel_buf = smem_topk;                   // [kTopkMaxSort] selected keys, grouped by bucket
  uint64_t* cand = smem_topk + kTopkMaxSort;       // [kTopkCand] keys of the k-th key's bucket
  __shared__ uint32_t hist[kTopkBins];
  __shared__ uint32_t pos[kTopkBins];
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

  // Pass 1: histogram of the 12-bit buckets (sign, exponent, 3 mantissa bits);
  // d1 is the bucket of the k-th largest key, kr1 its rank inside it, and
  // pos[d] where bucket d's keys start in descending order.
  digit_histogram(keys, n, 0u, 0u, 20, kTopkBins, hist);
  select_digit(hist, kTopkBins, uint32_t(k), s_sel, warp_sums, pos);
  const uint32_t d1 = s_sel[0];
  const int kr1 = int(s_sel[1]);
  const int n_gt1 = k - kr1;
  if (tid == 0) { s_cnt[0] = 0; s_cnt[1] = 0; }
  __syncthreads();
  // Pass 2: keys above bucket d1 go to their bucket's range of sel_buf; keys
  // in d1 are gathered as candidates.
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
        sel_buf[atomicAdd(&pos[dig], 1u)] = composite(u[j], i);
      } else if (dig == d1) {
        const uint32_t c = atomicAdd(&s_cnt[1], 1u);
        if (c < uint32_t(kTopkCand)) cand[c] = composite(u[j], i);
      }
    }
  }
  __syncthreads();
  const int nc = int(s_cnt[1]);

  if (nc <= kTopkCand) {
    // the best kr1 candidates, in order, after the keys of the buckets above
    if (nc <= kTopkRankMax) {
      for (int i = tid; i < nc; i += kTopkThreads) {
        const uint64_t c = cand[i];
        const int r = rank_in(cand, 0, nc, c);
        if (r < kr1) sel_buf[n_gt1 + r] = c;
      }
    } else {
      int cp = 1;
      while (cp < nc) cp <<= 1;
      for (int i = nc + tid; i < cp; i += kTopkThreads) cand[i] = ~0ull;
      __syncthreads();
      bitonic_sort(cand, cp);
      for (int i = tid; i < kr1; i += kTopkThreads) sel_buf[n_gt1 + i] = cand[i];
    }
    __syncthreads();
    // keys above d1: each lands at its bucket's start plus its rank in the bucket
    bool small_buckets = true;
    for (int d = tid; d < kTopkBins; d += kTopkThreads)
      if (d > int(d1) && hist[d] > uint32_t(kTopkRankMax)) small_buckets = false;
    if (__syncthreads_and(small_buckets ? 1 : 0)) {
      for (int i = tid; i < k; i += kTopkThreads) {
        const uint64_t c = sel_buf[i];
        int at = i;
        if (i < n_gt1) {
          const uint32_t d = (~uint32_t(c >> 32)) >> 20;
          const int e = int(pos[d]);
          const int s0 = e - int(hist[d]);
          at = s0 + rank_in(sel_buf, s0, e, c);
        }
        out_idx[at] = int32_t(c & 0xffffffffu);
        if (out_val) out_val[at] = __uint_as_float(~uint32_t(c >> 32));
      }
      return;
    }
    int kp = 1;
    while (kp < k) kp <<= 1;
    for (int i = k + tid; i < kp; i += kTopkThreads) sel_buf[i] = ~0ull;
    __syncthreads();
    bitonic_sort(sel_buf, kp);
  } else {
    // Too many keys share bucket d1: exact radix select on its low 20 bits over
    // global memory, then index-ordered compaction and a full sort.
    uint32_t prefix = d1 << 20, mask = 0xfff00000u, kr = uint32_t(kr1);
    for (int pass = 0; pass < 2; ++pass) {
      const int shift = pass == 0 ? 8 : 0;
      const int bits = pass == 0 ? 12 : 8;
      const int nbins = 1 << bits;
      digit_histogram(keys, n, prefix, mask, shift, nbins, hist);
      select_digit(hist, nbins, kr, s_sel, warp_sums, nullptr);
      prefix |= s_sel[0] << shift;
      mask |= uint32_t(nbins - 1) << shift;
      kr = s_sel[1];
      __syncthreads();
    }
    const uint32_t T = prefix;
    const int n_gt = k - int(kr);
    if (tid == 0) { s_sel[0] = uint32_t(n_gt1); s_sel[1] = 0; }   // keys above d1 are already placed
    __syncthreads();
    for (int base = 0; base < n; base += kTopkThreads) {
      const int i = base + tid;
      const uint32_t u = i < n ? impact_key(__ldg(keys + i)) : 0u;
      const bool in_bucket = i < n && (u >> 20) == d1;
      const bool gt = in_bucket && u > T;
      const bool eq = in_bucket && u == T;
      if (gt) sel_buf[atomicAdd(&s_sel[0], 1u)] = composite(u, i);
      const int eq_incl = block_scan_incl(eq ? 1 : 0, warp_sums);
      const uint32_t seen = s_sel[1];
      const uint32_t rank = seen + uint32_t(eq_incl) - (eq ? 1u : 0u);
      if (eq && rank < kr) sel_buf[n_gt + rank] = composite(u, i);
      __syncthreads();
      if (tid == kTopkThreads - 1) s_sel[1] = seen + uint32_t(eq_incl);
      __syncthreads();
      if (s_sel[1] >= kr && s_sel[0] >= uint32_t(n_gt)) break;
    }
    int kp = 1;
    while (kp < k) kp <<= 1;
    for (int i = k + tid; i < kp; i += kTopkThreads) sel_buf[i] = ~0ull;
    __syncthreads();
    bitonic_sort(sel_buf, kp);
  }
  for (int i = tid; i < k; i += kTopkThreads) {
    const uint64_t comp = sel_buf[i];
    out_idx[i] = int32_t(comp & 0xffffffffu);
    if (out_val) out_val[i] = __uint_as_float(~uint32_t(comp >> 32));
  }
}

cudaError_t launch_topk(const TopkParams& p, int num_requests, int max_k, cudaStream_t stream) {
  (void)max_k;
  const size_t smem = sizeof(uint64_t) * size_t(kTopkMaxSort + kTopkCand);   // + 32 KB static
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
