// Recompute selection (CacheBlend page, "Recompute ratio trade-off": the
// number of recomputed tokens is r times the total doc length; the listing
// takes max(1, int(doc_token_count * ratio)) and torch.topk over the doc slice
// of the impact vector).
//
// A cluster of C CTAs per request (C grows with the longest request, up to
// 8). Each CTA histograms the top 12 bits of its slice of the fp32 impacts
// (impacts are >= 0, so their bit patterns order like the values); the
// cluster's histograms, read over distributed shared memory, give the bucket
// d1 holding the k-th largest value and every bucket's place in descending
// order. Each CTA then writes the composite keys (impact descending, position
// ascending) of its keys above d1, and of the candidates inside d1, into CTA
// 0's shared memory, bucket by bucket. CTA 0 sorts every bucket on its own
// (a warp per bucket, the whole CTA for a bucket of more than 1,024 keys);
// the first k keys are then the answer in order. When the keys above d1 and
// d1's candidates together exceed the 20,480 that shared memory stages, CTA 0
// finds the k-th key by an exact radix select on the remaining 20 bits
// instead and sorts the k keys. k is at most 16,384.
// A request served by one CTA (at most 8,192 doc tokens) takes a shorter
// path first: its keys stay in registers, one histogram gives the k-th key's
// bucket and where each bucket starts in descending order, and when at most
// 1,024 keys lie in that bucket or above and ordering them by counting
// inside their buckets takes at most 131,072 comparisons (the sum of the
// squared bucket lengths), the keys are staged bucket by bucket and each
// finds its place by counting the keys of its own bucket before it;
// otherwise it continues on the path above.
#include <cooperative_groups.h>
#include <cuda_runtime.h>

#include "params.cuh"

namespace rag {

namespace cg = cooperative_groups;

constexpr int kTopkThreads = 1024;
constexpr int kTopkWarps = kTopkThreads / 32;
constexpr int kTopkBins = 4096;
constexpr int kBatch = 8;            // keys in flight per thread per pass
constexpr int kTopkMaxK = 16384;     // largest k (the host rejects more)
constexpr int kTopkSortMax = 20480;  // staged keys: those above the k-th key's bucket, then its candidates
static_assert(kTopkMaxK <= kTopkSortMax, "the k selected keys must fit the staging array");
constexpr int kTopkMaxCluster = 8;
constexpr int kTopkSlice = 8192;     // doc tokens per CTA before the cluster grows
constexpr int kRankMax = 256;        // longest bucket ordered by counting ranks (longer: sorted)
constexpr int kLeanKeys = kTopkSlice / kTopkThreads;   // keys per thread on the one-CTA path
constexpr int kLeanRank = 1024;      // most keys the one-CTA path orders by counting
constexpr uint32_t kLeanWork = 131072;   // most comparisons (sum of squared bucket lengths) it makes
static_assert(kLeanKeys * kTopkThreads == kTopkSlice, "one-CTA path: whole keys per thread");

struct TopkSmem {
  uint64_t staged[kTopkSortMax];     // composite keys of the buckets this CTA orders, at their final bucket ranges
  uint32_t hist[kTopkBins];          // this CTA's slice histogram; later its list of buckets to order
  uint32_t ghist[kTopkBins];         // the request's histogram; later the key offsets of that list
  uint32_t cursor[kTopkBins];        // next staging position for this CTA's keys of each bucket
  uint8_t owner[kTopkBins];          // CTA of the cluster that orders each bucket
  uint32_t sel[2];
  uint32_t cnt[4];
  int warp_sums[32];
};

__host__ __device__ constexpr size_t topk_smem_bytes() { return sizeof(TopkSmem); }

__device__ __forceinline__ uint32_t impact_key(float v) {
  const uint32_t u = __float_as_uint(v);
  return (u >> 31) ? 0u : u;   // -0 and negatives (never produced) sort as 0
}

// Composite sort key: ascending order = impact descending, position ascending.
__device__ __forceinline__ uint64_t composite(uint32_t key, int i) { return (uint64_t(~key) << 32) | uint32_t(i); }

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

// Histogram of one digit of every key that matches (prefix, mask), read from
// global memory kBatch keys per thread at a time.
__device__ __forceinline__ void digit_histogram(const float* keys, int n, uint32_t prefix, uint32_t mask,
                                                int shift, int nbins, uint32_t* hist) {
  const int tid = threadIdx.x;
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
      if (i < n && (u[j] & mask) == prefix) atomicAdd(&hist[(u[j] >> shift) & uint32_t(nbins - 1)], 1u);
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

constexpr uint64_t kKeyInf = ~0ull;   // sorts after every real composite key

__device__ __forceinline__ uint64_t shfl_xor64(uint64_t v, int m) {
  const uint32_t lo = __shfl_xor_sync(0xffffffffu, uint32_t(v), m);
  const uint32_t hi = __shfl_xor_sync(0xffffffffu, uint32_t(v >> 32), m);
  return (uint64_t(hi) << 32) | lo;
}
__device__ __forceinline__ void cmpswap(uint64_t& x, uint64_t& y) {
  const uint64_t lo = x < y ? x : y, hi = x < y ? y : x;
  x = lo;
  y = hi;
}

// The sorting networks below are bitonic in the all-ascending form: merging
// two sorted halves of a block of `size` positions first compares position i
// with its mirror image i ^ (size - 1), then runs half-cleaners (i against
// i ^ stride); the lower position always keeps the smaller key. Positions at
// or past the run's length act as +infinity, which this form never moves, so
// they are neither stored nor read. A thread holds E consecutive positions.

// In-thread steps: sizes 2 .. E (whole blocks inside one thread).
template <int E>
__device__ __forceinline__ void sort_in_thread(uint64_t (&r)[E]) {
#pragma unroll
  for (int lg = 1; (1 << lg) <= E; ++lg) {
#pragma unroll
    for (int s = 0; s < E; ++s) {
      const int t = s ^ ((1 << lg) - 1);
      if (s < t) cmpswap(r[s], r[t]);
    }
#pragma unroll
    for (int ls = lg - 2; ls >= 0; --ls) {
#pragma unroll
      for (int s = 0; s < E; ++s) {
        const int t = s ^ (1 << ls);
        if (s < t) cmpswap(r[s], r[t]);
      }
    }
  }
}

// Mirror step of a block of `size` > E positions whose partner is in the same
// warp (size / E <= 32).
template <int E>
__device__ __forceinline__ void mirror_shfl(uint64_t (&r)[E], int size, int lane) {
  const int m = size / E - 1;
  const bool lower = (lane & ((m + 1) >> 1)) == 0;
  if (E == 1) {
    const uint64_t y = shfl_xor64(r[0], m);
    r[0] = lower ? (r[0] < y ? r[0] : y) : (r[0] < y ? y : r[0]);
    return;
  }
#pragma unroll
  for (int s = 0; s < E / 2; ++s) {   // slots s and E-1-s trade places with the partner
    const uint64_t ya = shfl_xor64(r[E - 1 - s], m);
    const uint64_t yb = shfl_xor64(r[s], m);
    r[s] = lower ? (r[s] < ya ? r[s] : ya) : (r[s] < ya ? ya : r[s]);
    r[E - 1 - s] = lower ? (r[E - 1 - s] < yb ? r[E - 1 - s] : yb) : (r[E - 1 - s] < yb ? yb : r[E - 1 - s]);
  }
}

// Half-cleaners from stride st down to 1, st < 32 * E (partners in the warp).
template <int E>
__device__ __forceinline__ void cleaners_in_warp(uint64_t (&r)[E], int st, int lane) {
  for (; st >= E; st >>= 1) {
    const int m = st / E;
    const bool lower = (lane & m) == 0;
#pragma unroll
    for (int s = 0; s < E; ++s) {
      const uint64_t y = shfl_xor64(r[s], m);
      r[s] = lower ? (r[s] < y ? r[s] : y) : (r[s] < y ? y : r[s]);
    }
  }
#pragma unroll
  for (int ls = 0; (1 << ls) < E; ++ls) {
    const int stv = (E >> 1) >> ls;   // E/2, E/4, ..., 1
#pragma unroll
    for (int s = 0; s < E; ++s) {
      const int t = s ^ stv;
      if (s < t) cmpswap(r[s], r[t]);
    }
  }
}

// Place of each of a[0, m): the keys are grouped by 12-bit bucket in
// descending bucket order, bucket d ending at end[d] and holding len[d]
// keys; a key's place is its bucket's start plus the keys of its bucket
// that sort before it, counted by P threads per key. Keys placed below k are
// written out.
__device__ __forceinline__ void rank_in_buckets(const uint64_t* a, int m, const uint32_t* end,
                                                const uint32_t* len, int k, int32_t* out_idx, float* out_val) {
  const int tid = threadIdx.x;
  int P = 32;
  while (P > 1 && m * P > kTopkThreads) P >>= 1;
  const int per_pass = kTopkThreads / P;
  const int p_lane = tid & (P - 1);
  for (int f0 = 0; f0 < m; f0 += per_pass) {
    const int f = f0 + tid / P;
    uint64_t me = 0ull;
    int first = 0, n_b = 0;
    if (f < m) {
      me = a[f];
      const uint32_t d = (~uint32_t(me >> 32)) >> 20;
      n_b = int(len[d]);
      first = int(end[d]) - n_b;
    }
    const uint64_t* run = a + first;
    int c[4] = {0, 0, 0, 0};
    int j = p_lane;
    for (; j + 3 * P < n_b; j += 4 * P) {   // four independent loads in flight per step
      uint64_t v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) v[u] = run[j + u * P];
#pragma unroll
      for (int u = 0; u < 4; ++u) c[u] += v[u] < me ? 1 : 0;
    }
    for (; j < n_b; j += P) c[0] += run[j] < me ? 1 : 0;
    int cnt = (c[0] + c[1]) + (c[2] + c[3]);
    for (int o = 1; o < P; o <<= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
    const int place = first + cnt;
    if (f < m && p_lane == 0 && place < k) {
      out_idx[place] = int32_t(me & 0xffffffffu);
      if (out_val) out_val[place] = __uint_as_float(~uint32_t(me >> 32));
    }
  }
}

// The whole CTA sorts a[0, len), len <= 1024 * E; steps whose partners are
// in another warp go through shared memory between block barriers.
template <int E>
__device__ void block_sort(uint64_t* a, int len) {
  const int tid = threadIdx.x, lane = tid & 31;
  int sp = 32 * E;
  while (sp < len) sp <<= 1;
  const bool holds = tid < sp / E;   // whole warps
  const int i0 = tid * E;
  uint64_t r[E];
#pragma unroll
  for (int s = 0; s < E; ++s) r[s] = (holds && i0 + s < len) ? a[i0 + s] : kKeyInf;
  if (holds) sort_in_thread<E>(r);
  for (int size = 2 * E; size <= sp; size <<= 1) {
    int st = size >> 2;
    if (size / E > 32) {
      __syncthreads();
      if (holds) {
#pragma unroll
        for (int s = 0; s < E; ++s)
          if (i0 + s < len) a[i0 + s] = r[s];
      }
      __syncthreads();
      const int half = size >> 1, lg_half = __ffs(half) - 1;
      for (int q = tid; q < (sp >> 1); q += kTopkThreads) {
        const int base = (q >> lg_half) * size, off = q & (half - 1);
        const int i = base + off, j = base + size - 1 - off;
        if (j < len) cmpswap(a[i], a[j]);
      }
      __syncthreads();
      for (; st >= 32 * E; st >>= 1) {
        for (int q = tid; q < (sp >> 1); q += kTopkThreads) {
          const int i = 2 * q - (q & (st - 1)), j = i + st;
          if (j < len) cmpswap(a[i], a[j]);
        }
        __syncthreads();
      }
      if (holds) {
#pragma unroll
        for (int s = 0; s < E; ++s) r[s] = i0 + s < len ? a[i0 + s] : kKeyInf;
      }
    } else if (holds) {
      mirror_shfl<E>(r, size, lane);
    }
    if (holds) cleaners_in_warp<E>(r, st, lane);
  }
  __syncthreads();
  if (holds) {
#pragma unroll
    for (int s = 0; s < E; ++s)
      if (i0 + s < len) a[i0 + s] = r[s];
  }
  __syncthreads();
}

// The same network with every step in shared memory (runs longer than the
// register forms hold: more than 8,192 keys).
__device__ void block_sort_smem(uint64_t* a, int len) {
  const int tid = threadIdx.x;
  int sp = 2;
  while (sp < len) sp <<= 1;
  __syncthreads();
  for (int size = 2; size <= sp; size <<= 1) {
    const int half = size >> 1, lg_half = __ffs(half) - 1;
    for (int q = tid; q < (sp >> 1); q += kTopkThreads) {
      const int base = (q >> lg_half) * size, off = q & (half - 1);
      const int i = base + off, j = base + size - 1 - off;
      if (j < len) cmpswap(a[i], a[j]);
    }
    __syncthreads();
    for (int st = size >> 2; st >= 1; st >>= 1) {
      for (int q = tid; q < (sp >> 1); q += kTopkThreads) {
        const int i = 2 * q - (q & (st - 1)), j = i + st;
        if (j < len) cmpswap(a[i], a[j]);
      }
      __syncthreads();
    }
  }
}

__device__ void block_sort_any(uint64_t* a, int len) {
  if (len <= 64 * kTopkWarps) block_sort<2>(a, len);
  else if (len <= 128 * kTopkWarps) block_sort<4>(a, len);
  else if (len <= 256 * kTopkWarps) block_sort<8>(a, len);
  else block_sort_smem(a, len);
}

__global__ void __launch_bounds__(kTopkThreads, 1) topk_kernel(const TopkParams p) {
  extern __shared__ __align__(16) uint8_t topk_raw[];
  TopkSmem& S = *reinterpret_cast<TopkSmem*>(topk_raw);
  cg::cluster_group cluster = cg::this_cluster();
  const int csize = int(cluster.num_blocks());
  const int crank = int(cluster.block_rank());
  const int b = blockIdx.x / csize;
  const int tid = threadIdx.x;
  const ReqInfo req = load_req(p.batch, b);
  const bool ok = req_ok(p.batch, req);
  const int n = ok ? req.n_doc : 0;
  const float* keys = p.impact + (req.doc0 + req.q0);
  int k = n > 0 ? max(1, int(double(n) * p.r)) : 0;
  k = min(min(k, n), min(p.k_cap, p.k_max));
  int32_t* out_idx = p.topk_idx + int64_t(b) * p.k_cap;
  float* out_val = p.topk_val ? p.topk_val + int64_t(b) * p.k_cap : nullptr;
  pdl_wait();   // the impact vector comes from the kernel before this one; outputs are written after it
  if (crank == 0) {
    if (p.k_out && tid == 0) p.k_out[b] = k;
    for (int i = k + tid; i < p.k_cap; i += kTopkThreads) {
      out_idx[i] = -1;
      if (out_val) out_val[i] = 0.f;
    }
  }
  if (k == 0) return;   // the whole cluster leaves together

  if (csize == 1) {
    // One CTA: the request's keys (at most 8,192) in registers, one histogram
    // of the 12-bit buckets, the k-th key's bucket d1; the keys of d1 and of
    // the buckets above it, when there are at most 1,024, are ordered by
    // counting. Otherwise the general path below runs.
    uint32_t u[kLeanKeys];
#pragma unroll
    for (int j = 0; j < kLeanKeys; ++j) {
      const int i = j * kTopkThreads + tid;
      u[j] = i < n ? impact_key(__ldg(keys + i)) : 0u;
    }
    for (int i = tid; i < kTopkBins; i += kTopkThreads) S.hist[i] = 0;
    if (tid == 0) S.cnt[0] = 0;
    __syncthreads();
#pragma unroll
    for (int j = 0; j < kLeanKeys; ++j)
      if (j * kTopkThreads + tid < n) atomicAdd(&S.hist[u[j] >> 20], 1u);
    __syncthreads();
    // S.cursor[d]: keys in the buckets above d (where bucket d starts)
    select_digit(S.hist, kTopkBins, uint32_t(k), S.sel, S.warp_sums, S.cursor);
    const uint32_t d1 = S.sel[0];
    const int m = k - int(S.sel[1]) + int(S.hist[d1]);   // keys in d1 and above
    if (m <= kLeanRank) {
      // comparisons of the counting: the squared lengths of the buckets from d1 up
      uint32_t work = 0;
      for (int d = tid; d < kTopkBins; d += kTopkThreads)
        if (d >= int(d1)) work += S.hist[d] * S.hist[d];
      for (int o = 16; o > 0; o >>= 1) work += __shfl_xor_sync(0xffffffffu, work, o);
      if ((tid & 31) == 0 && work > 0) atomicAdd(&S.cnt[0], work);
    }
    __syncthreads();
    if (m <= kLeanRank && S.cnt[0] <= kLeanWork) {
      // stage bucket by bucket; afterwards S.cursor[d] is where bucket d ends
#pragma unroll
      for (int j = 0; j < kLeanKeys; ++j) {
        const int i = j * kTopkThreads + tid;
        if (i < n && (u[j] >> 20) >= d1) S.staged[atomicAdd(&S.cursor[u[j] >> 20], 1u)] = composite(u[j], i);
      }
      __syncthreads();
      rank_in_buckets(S.staged, m, S.cursor, S.hist, k, out_idx, out_val);
      return;
    }
    __syncthreads();   // every thread has read S.hist and S.sel before the general path rewrites them
  }


  // Pass 1: histogram of the 12-bit buckets (sign, exponent, 3 mantissa bits)
  // of this CTA's slice, then the request's histogram and, per bucket, how
  // many of its keys the lower-ranked CTAs hold.
  const int lo = int(int64_t(n) * crank / csize), hi = int(int64_t(n) * (crank + 1) / csize);
  digit_histogram(keys + lo, hi - lo, 0u, 0u, 20, kTopkBins, S.hist);
  cluster.sync();
  for (int d4 = tid; d4 < kTopkBins / 4; d4 += kTopkThreads) {
    uint4 tot = make_uint4(0, 0, 0, 0), bef = make_uint4(0, 0, 0, 0);
    uint4 h[kTopkMaxCluster];
#pragma unroll
    for (int r = 0; r < kTopkMaxCluster; ++r)   // all reads in flight before any is used
      h[r] = r < csize ? reinterpret_cast<const uint4*>(cluster.map_shared_rank(S.hist, r))[d4] : make_uint4(0, 0, 0, 0);
#pragma unroll
    for (int r = 0; r < kTopkMaxCluster; ++r) {
      tot.x += h[r].x; tot.y += h[r].y; tot.z += h[r].z; tot.w += h[r].w;
      if (r < crank) { bef.x += h[r].x; bef.y += h[r].y; bef.z += h[r].z; bef.w += h[r].w; }
    }
    reinterpret_cast<uint4*>(S.ghist)[d4] = tot;
    reinterpret_cast<uint4*>(S.cursor)[d4] = bef;
  }
  __syncthreads();
  // d1: bucket of the k-th largest key; kr1: keys taken from it
  select_digit(S.ghist, kTopkBins, uint32_t(k), S.sel, S.warp_sums, nullptr);
  const uint32_t d1 = S.sel[0];
  const int kr1 = int(S.sel[1]);
  const int n_gt1 = k - kr1;
  const int nc = int(S.ghist[d1]);
  const bool stage_cand = n_gt1 + nc <= kTopkSortMax;
  // Staging: the keys of the buckets above d1 in descending bucket order, then
  // the candidates. Every bucket from d1 up that holds keys is a segment;
  // segment g (in descending bucket order) is ordered by CTA g % C, and only
  // that CTA receives its keys. This CTA's keys of bucket d start at
  // start(d) + (keys of d in lower-ranked CTAs).
  constexpr int kPer = kTopkBins / kTopkThreads;
  const int hi_bin = kTopkBins - 1 - tid * kPer;   // this thread's bins, descending
  uint32_t seg_at[kPer], seg_len[kPer];
  int seg_g[kPer];
  {
    uint32_t keys_mine = 0, segs_mine = 0;
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      const int d = hi_bin - j;
      const uint32_t len = d > int(d1) ? S.ghist[d] : d == int(d1) ? uint32_t(nc) : 0u;
      if (d > int(d1)) keys_mine += len;
      if (len > 0) ++segs_mine;
    }
    // keys above d1 (< 2^14) in the low half, segments in the high half
    const uint32_t incl = uint32_t(block_scan_incl(int(keys_mine | (segs_mine << 16)), S.warp_sums));
    if (tid == kTopkThreads - 1) S.cnt[3] = incl >> 16;   // segments in all
    uint32_t at = (incl & 0xffffu) - keys_mine;
    int g = int(incl >> 16) - int(segs_mine);
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      const int d = hi_bin - j;
      const uint32_t len = d > int(d1) ? S.ghist[d] : d == int(d1) ? uint32_t(nc) : 0u;
      seg_len[j] = len;
      seg_at[j] = d == int(d1) ? uint32_t(n_gt1) : at;
      seg_g[j] = len > 0 ? g : -1;
      if (len > 0) ++g;
      if (d >= int(d1)) {
        S.cursor[d] += seg_at[j];
        S.owner[d] = uint8_t(stage_cand && len > 0 ? (seg_g[j] % csize) : 0);
      }
      if (d > int(d1)) at += len;
    }
  }
  __syncthreads();
  // Pass 2: this CTA's keys above d1, and in d1, to the CTA that orders them
  // (all to CTA 0 when d1 is too full to stage).
  for (int base = lo; base < hi; base += kTopkThreads * kBatch) {
    uint32_t u[kBatch];
#pragma unroll
    for (int j = 0; j < kBatch; ++j) {
      const int i = base + j * kTopkThreads + tid;
      u[j] = i < hi ? impact_key(__ldg(keys + i)) : 0u;
    }
#pragma unroll
    for (int j = 0; j < kBatch; ++j) {
      const int i = base + j * kTopkThreads + tid;
      if (i >= hi) continue;
      const uint32_t dig = u[j] >> 20;
      if (dig > d1 || (dig == d1 && stage_cand)) {
        const uint32_t at = atomicAdd(&S.cursor[dig], 1u);
        cluster.map_shared_rank(S.staged, int(S.owner[dig]))[at] = composite(u[j], i);
      }
    }
  }
  cluster.sync();   // every key is with its CTA; no CTA touches another's memory again

  if (stage_cand) {
    // This CTA's segments, in order: (first position, length) in S.hist, the
    // running count of keys of its short segments in S.ghist; long ones are
    // also listed from the back of S.hist.
    const int n_seg = int(S.cnt[3]);
    const int n_mine = n_seg > crank ? (n_seg - crank + csize - 1) / csize : 0;
    if (tid == 0) S.cnt[1] = 0;
    __syncthreads();
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      if (seg_g[j] < 0 || seg_g[j] % csize != crank) continue;
      const uint32_t e = seg_at[j] | (seg_len[j] << 16);
      S.hist[seg_g[j] / csize] = e;
      if (seg_len[j] > uint32_t(kRankMax)) S.hist[kTopkBins - 1 - atomicAdd(&S.cnt[1], 1u)] = e;
    }
    __syncthreads();
    {
      uint32_t mine = 0;
#pragma unroll
      for (int j = 0; j < kPer; ++j) {
        const int i = tid * kPer + j;
        const uint32_t len = i < n_mine ? (S.hist[i] >> 16) : 0u;
        mine += len <= uint32_t(kRankMax) ? len : 0u;
      }
      const uint32_t incl = uint32_t(block_scan_incl(int(mine), S.warp_sums));
      uint32_t run = incl - mine;
#pragma unroll
      for (int j = 0; j < kPer; ++j) {
        const int i = tid * kPer + j;
        S.ghist[i] = run;
        const uint32_t len = i < n_mine ? (S.hist[i] >> 16) : 0u;
        run += len <= uint32_t(kRankMax) ? len : 0u;
      }
      if (tid == kTopkThreads - 1) S.cnt[2] = incl;   // keys of the short segments
    }
    __syncthreads();
    const int n_big = int(S.cnt[1]);
    const int n_keys = int(S.cnt[2]);
    // long segments: sorted in place by the whole CTA
    for (int i = 0; i < n_big; ++i) {
      const uint32_t e = S.hist[kTopkBins - 1 - i];
      const int first = int(e & 0xffffu), len = int(e >> 16);
      block_sort_any(S.staged + first, len);
      const int take = first == n_gt1 ? kr1 : len;   // only d1's segment starts at n_gt1
      for (int j = tid; j < take; j += kTopkThreads) {
        const uint64_t comp = S.staged[first + j];
        out_idx[first + j] = int32_t(comp & 0xffffffffu);
        if (out_val) out_val[first + j] = __uint_as_float(~uint32_t(comp >> 32));
      }
    }
    // short segments: a key's place is the number of keys of its segment
    // that sort before it; P threads share each key's comparisons
    int P = 32;
    while (P > 1 && n_keys * P > kTopkThreads) P >>= 1;
    const int per_pass = kTopkThreads / P;
    const int p_lane = tid & (P - 1);
    for (int f0 = 0; f0 < n_keys; f0 += per_pass) {
      const int f = f0 + tid / P;
      int first = 0, len = 0, local = 0;
      uint64_t me = 0;
      if (f < n_keys) {
        int lo_s = 0, hi_s = n_mine - 1;   // last segment whose key offset is <= f
        while (lo_s < hi_s) {
          const int mid = (lo_s + hi_s + 1) >> 1;
          if (int(S.ghist[mid]) <= f) lo_s = mid; else hi_s = mid - 1;
        }
        const uint32_t e = S.hist[lo_s];
        first = int(e & 0xffffu);
        len = int(e >> 16);
        local = f - int(S.ghist[lo_s]);
        me = S.staged[first + local];
      }
      // eight independent loads in flight per step
      const uint64_t* run = S.staged + first;
      int c[8] = {0, 0, 0, 0, 0, 0, 0, 0};
      int j = p_lane;
      for (; j + 7 * P < len; j += 8 * P) {
        uint64_t v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) v[u] = run[j + u * P];
#pragma unroll
        for (int u = 0; u < 8; ++u) c[u] += v[u] < me ? 1 : 0;
      }
      for (; j < len; j += P) c[0] += run[j] < me ? 1 : 0;
      int cnt = ((c[0] + c[1]) + (c[2] + c[3])) + ((c[4] + c[5]) + (c[6] + c[7]));
      for (int o = 1; o < P; o <<= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
      if (f < n_keys && p_lane == 0 && (first != n_gt1 || cnt < kr1)) {
        out_idx[first + cnt] = int32_t(me & 0xffffffffu);
        if (out_val) out_val[first + cnt] = __uint_as_float(~uint32_t(me >> 32));
      }
    }
    return;
  } else {
    // Too many keys share bucket d1: CTA 0 alone runs an exact radix select on
    // its low 20 bits over the whole request, then an index-ordered compaction
    // and one sort of the k keys.
    if (crank != 0) return;
    uint32_t prefix = d1 << 20, mask = 0xfff00000u, kr = uint32_t(kr1);
    for (int pass = 0; pass < 2; ++pass) {
      const int shift = pass == 0 ? 8 : 0;
      const int bits = pass == 0 ? 12 : 8;
      const int nbins = 1 << bits;
      digit_histogram(keys, n, prefix, mask, shift, nbins, S.hist);
      select_digit(S.hist, nbins, kr, S.sel, S.warp_sums, nullptr);
      prefix |= S.sel[0] << shift;
      mask |= uint32_t(nbins - 1) << shift;
      kr = S.sel[1];
      __syncthreads();
    }
    const uint32_t T = prefix;
    const int n_gt = k - int(kr);
    if (tid == 0) { S.sel[0] = uint32_t(n_gt1); S.sel[1] = 0; }   // keys above d1 are already staged
    __syncthreads();
    for (int base = 0; base < n; base += kTopkThreads) {
      const int i = base + tid;
      const uint32_t u = i < n ? impact_key(__ldg(keys + i)) : 0u;
      const bool in_bucket = i < n && (u >> 20) == d1;
      const bool gt = in_bucket && u > T;
      const bool eq = in_bucket && u == T;
      if (gt) S.staged[atomicAdd(&S.sel[0], 1u)] = composite(u, i);
      const int eq_incl = block_scan_incl(eq ? 1 : 0, S.warp_sums);
      const uint32_t seen = S.sel[1];
      const uint32_t rank = seen + uint32_t(eq_incl) - (eq ? 1u : 0u);
      if (eq && rank < kr) S.staged[n_gt + rank] = composite(u, i);
      __syncthreads();
      if (tid == kTopkThreads - 1) S.sel[1] = seen + uint32_t(eq_incl);
      __syncthreads();
      if (S.sel[1] >= kr && S.sel[0] >= uint32_t(n_gt)) break;
    }
    block_sort_any(S.staged, k);
  }
  for (int i = tid; i < k; i += kTopkThreads) {
    const uint64_t comp = S.staged[i];
    out_idx[i] = int32_t(comp & 0xffffffffu);
    if (out_val) out_val[i] = __uint_as_float(~uint32_t(comp >> 32));
  }
}

int topk_cluster_size(int max_doc) {
  int c = 1;
  while (c < kTopkMaxCluster && int64_t(c) * kTopkSlice < max_doc) c <<= 1;
  return c;
}

cudaError_t launch_topk(const TopkParams& p, int num_requests, int max_k, cudaStream_t stream) {
  (void)max_k;
  const size_t smem = topk_smem_bytes();
  static SmemAttr attr;
  cudaError_t e = ensure_smem_attr(topk_kernel, attr, smem);
  if (e != cudaSuccess) return e;
  const int c = topk_cluster_size(p.batch.max_doc);
  return launch_pdl(topk_kernel, dim3(num_requests * c), dim3(kTopkThreads), smem, stream, c, p);
}

}  // namespace rag
