// Selective KV recompute into copy-on-write pages (CacheBlend page,
// "Contributions": only the tokens of high attention impact are recomputed
// when the cached KV are fused; "How it works": concatenate -> pick the
// high-Impact tokens -> recompute their KV -> generate).
//
// Three kernels, in stream order:
//   plan (one CTA)  : for every selected token (the top-k positions) its page
//                     reference and slot; every reference that holds a
//                     selected token gets a private page from the caller's
//                     free list (ascending reference order), the request's
//                     page table is rewritten, and the token's destination
//                     (private page, slot) and hidden-state row are listed
//   copy            : per private page and layer, every slot that is NOT
//                     selected is copied from the page it replaces (K and V,
//                     all KV heads); the selected slots are left to the GEMM,
//                     so the two never write the same bytes
//   GEMM (tcgen05)  : [K | V] rows = X_sel W^T. The A operand (128 selected
//                     tokens x 64 hidden features per stage) is loaded as one
//                     tiled TMA box when the hidden states are listed by
//                     selection rank, or gathered by TMA tile::gather4 from
//                     rows listed by doc position; the B operand (the rows of
//                     two KV heads of W_K or W_V, one when H_kv is odd) by a
//                     tiled TMA load; the accumulator lives in TMEM, and the
//                     epilogue rounds each row once to the type the pool
//                     stores it in (K bf16, V fp16: nearest even, V saturated
//                     beyond 65504 with kDevErrRange raised) and stores it
//                     into its slot of its private page.
// Every wait is bounded; a timeout raises a device error instead of hanging.
// None of these kernels releases its dependents early: they write page tables
// and pool pages, which the attention kernel reads before its own wait. (Running
// the copy beside the projection measured slower: the projection streams its
// operands from L2 at a high rate and the copy competes for it.)
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "params.cuh"

namespace rag {

// ---------------------------------------------------------------- plan

constexpr int kRcPlanThreads = 1024;

// exclusive block scan of one value per thread (1024 threads); returns the
// exclusive prefix and writes the block total to *total
__device__ __forceinline__ int rc_block_scan(int v, int* warp_sums, int* total) {
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
  const int before = (warp > 0 ? warp_sums[warp - 1] : 0) + x - v;
  *total = warp_sums[31];
  __syncthreads();
  return before;
}

__global__ void __launch_bounds__(kRcPlanThreads, 1) rc_plan_kernel(const RcPlanParams p) {
  __shared__ int32_t kpre[kMaxRequests + 1];
  __shared__ int warp_sums[32];
  __shared__ int32_t s_err;
  const int tid = threadIdx.x;
  const BatchDev& B = p.batch;
  const int nb = B.num_requests;
  const int n_refs = B.num_page_refs;
  int32_t* hdr = p.plan;
  int32_t* x_row = p.plan + p.lay.x_row;
  int32_t* dst = p.plan + p.lay.dst;
  int32_t* ref_of = p.plan + p.lay.ref;
  int32_t* cow_src = p.plan + p.lay.cow_src;
  int32_t* cow_dst = p.plan + p.lay.cow_dst;
  int32_t* cow_mask = p.plan + p.lay.cow_mask;
  uint32_t* flags = reinterpret_cast<uint32_t*>(p.plan + p.lay.flags);
  if (tid == 0) s_err = 0;
  pdl_wait();   // the selection comes from the kernel before this one

  // k_b of every request (clamped to [0, k_cap]) -> exclusive prefix
  constexpr int kPer = (kMaxRequests + kRcPlanThreads - 1) / kRcPlanThreads;
  int kv[kPer];
  int mine = 0;
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int b = tid * kPer + i;
    int kb = b < nb ? __ldg(p.k + b) : 0;
    kb = kb < 0 ? 0 : (kb > p.k_cap ? p.k_cap : kb);
    kv[i] = kb;
    mine += kb;
  }
  int n_tok = 0;
  int run = rc_block_scan(mine, warp_sums, &n_tok);
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int b = tid * kPer + i;
    if (b <= nb) kpre[b] = run;
    run += kv[i];
  }
  for (int r = tid; r < n_refs; r += kRcPlanThreads) flags[r] = 0u;
  __syncthreads();

  // every selected token: its page reference and slot; mark the reference
  for (int t = tid; t < n_tok; t += kRcPlanThreads) {
    int lo = 0, hi = nb - 1;   // last b with kpre[b] <= t
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (kpre[mid] <= t) lo = mid; else hi = mid - 1;
    }
    const int b = lo;
    const int pos = __ldg(p.topk_idx + int64_t(b) * p.k_cap + (t - kpre[b]));
    const ReqInfo r = load_req(B, b);
    ref_of[t] = -1;
    x_row[t] = -1;
    dst[t] = 0;
    if (!req_ok(B, r) || pos < 0 || pos >= r.n_doc) { atomicOr(&s_err, kDevErrGeometry); continue; }
    int clo = r.c0, chi = r.c1 - 1;   // last chunk-list entry starting at or before pos
    while (clo < chi) {
      const int mid = (clo + chi + 1) >> 1;
      if (__ldg(B.chunk_doc_off + mid) - r.doc0 <= pos) clo = mid; else chi = mid - 1;
    }
    const int tl = pos - (__ldg(B.chunk_doc_off + clo) - r.doc0);
    const int ref = __ldg(B.chunk_page_off + clo) + tl / kPage;
    if (ref >= __ldg(B.chunk_page_off + clo + 1) || ref >= n_refs) { atomicOr(&s_err, kDevErrGeometry); continue; }
    atomicOr(&flags[ref], 1u << (tl % kPage));
    ref_of[t] = ref;
    dst[t] = tl % kPage;
    x_row[t] = p.by_selection ? t : r.doc0 + pos;
  }
  __syncthreads();

  // references holding a selected token: how many private pages are needed
  int dirty = 0;
  for (int r = tid; r < n_refs; r += kRcPlanThreads) dirty += __ldcg(flags + r) != 0u ? 1 : 0;
  int n_needed = 0;
  rc_block_scan(dirty, warp_sums, &n_needed);
  const bool fits = n_needed <= p.n_free;

  // private pages in ascending reference order; the rewritten page table
  int carry = 0;
  for (int base = 0; base < n_refs; base += kRcPlanThreads * 4) {
    uint32_t f[4];
    int cnt = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = base + tid * 4 + i;
      f[i] = (r < n_refs && fits) ? __ldcg(flags + r) : 0u;
      cnt += f[i] != 0u ? 1 : 0;
    }
    int chunk_total = 0;
    int idx = carry + rc_block_scan(cnt, warp_sums, &chunk_total);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = base + tid * 4 + i;
      if (r >= n_refs) continue;
      const int32_t old = __ldg(B.page_ids + r);
      if (f[i] != 0u) {
        const int32_t np = __ldg(p.free_pages + idx);
        p.page_ids_out[r] = np;
        cow_src[idx] = old;
        cow_dst[idx] = np;
        cow_mask[idx] = int32_t(f[i]);
        ++idx;
      } else {
        p.page_ids_out[r] = old;
      }
    }
    carry += chunk_total;
  }
  __syncthreads();

  // destinations of the selected tokens in their private pages
  for (int t = tid; t < n_tok; t += kRcPlanThreads) {
    const int ref = ref_of[t];
    if (!fits || ref < 0) { x_row[t] = -1; continue; }
    dst[t] = p.page_ids_out[ref] * kPage + dst[t];
  }
  if (tid == 0) {
    hdr[kRcHdrTok] = fits ? n_tok : 0;
    hdr[kRcHdrCow] = fits ? n_needed : 0;
    hdr[kRcHdrNeeded] = n_needed;
    hdr[kRcHdrErr] = s_err | (fits ? 0 : kRcErrNoFree);
    hdr[kRcHdrBySel] = p.by_selection;   // rows t of the hidden states are consecutive
  }
}

// ---------------------------------------------------------------- copy

constexpr int kRcCopyThreads = 512;   // 16 warps: one per (tensor, KV head) block of a page, up to 8 heads

// One private page per block iteration: K and V of this layer, every KV head,
// every slot the selection does not overwrite. A warp copies one (tensor,
// head) block of 16 slots x 256 bytes: each lane moves eight 16-byte units,
// all eight loads in flight before the first store.
__global__ void __launch_bounds__(kRcCopyThreads, 2) rc_copy_kernel(const RcCopyParams p) {
  pdl_wait();   // the plan comes from the kernel before this one
  const int32_t* hdr = p.plan;
  const int n_cow = __ldcg(hdr + kRcHdrCow);
  const int hk = p.num_kv_heads;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int kUnits = kPage * kHeadDim * 2 / 16;            // 16-byte units of one (tensor, head) block
  const int64_t block_units = kUnits;
  const int64_t page_units = int64_t(hk) * kUnits;              // one page of one tensor, one layer
  const int64_t layer_base = int64_t(p.layer) * p.num_pages;
  for (int i = blockIdx.x; i < n_cow; i += gridDim.x) {
    const int src = __ldcg(p.plan + p.lay.cow_src + i);
    const int dstp = __ldcg(p.plan + p.lay.cow_dst + i);
    const uint32_t mask = uint32_t(__ldcg(p.plan + p.lay.cow_mask + i));
    if (src < 0 || src >= p.num_pages || dstp < 0 || dstp >= p.num_pages) {
      if (threadIdx.x == 0) atomicOr(p.plan + kRcHdrErr, kDevErrPage);
      continue;
    }
    for (int blk = warp; blk < 2 * hk; blk += kRcCopyThreads / 32) {
      const int tensor = blk / hk, h = blk % hk;
      const uint4* from = reinterpret_cast<const uint4*>(tensor ? p.pool_v : p.pool_k) +
                          (layer_base + src) * page_units + h * block_units;
      uint4* to = reinterpret_cast<uint4*>(tensor ? p.pool_v : p.pool_k) + (layer_base + dstp) * page_units +
                  h * block_units;
      uint4 v[kUnits / 32];
#pragma unroll
      for (int j = 0; j < kUnits / 32; ++j) {
        const int u = lane + 32 * j;                            // slot u / 16
        if (!(mask & (1u << (u >> 4)))) v[j] = __ldg(from + u);
      }
#pragma unroll
      for (int j = 0; j < kUnits / 32; ++j) {
        const int u = lane + 32 * j;
        if (!(mask & (1u << (u >> 4)))) to[u] = v[j];
      }
    }
  }
}

// ---------------------------------------------------------------- GEMM

constexpr int kRcBM = 128;            // selected tokens per tile (MMA M, TMEM lanes)
constexpr int kRcHead = 128;          // output columns of one KV head
constexpr int kRcBNMax = 2 * kRcHead; // output columns per tile: one or two heads of K or V
constexpr int kRcBK = 64;             // hidden features per stage (128 B rows, 128B swizzle)
constexpr int kRcStages = 4;
constexpr int kRcABytes = kRcBM * kRcBK * 2;
constexpr int kRcBBytesMax = kRcBNMax * kRcBK * 2;
constexpr int kRcStageBytes = kRcABytes + kRcBBytesMax;
constexpr int kRcThreads = 192;       // producer, MMA, 4 epilogue warps

struct RcCtrl {
  uint64_t full[kRcStages], empty[kRcStages];
  uint64_t acc_full[2], acc_empty[2];
  uint32_t tmem_base;
  int32_t abort;
};

__host__ size_t rc_gemm_smem_bytes() { return 1024 + size_t(kRcStages) * kRcStageBytes + sizeof(RcCtrl) + 64; }

__device__ __forceinline__ uint64_t rc_desc(uint32_t base, int kk) { return sdesc_sw128(base + kk * 32, 16, 1024); }

__device__ __forceinline__ void rc_abort(RcCtrl* c, int32_t* err) {
  if (!c->abort) {
    atomicOr(err, kDevErrTimeout);
    c->abort = 1;
  }
}

__global__ void __launch_bounds__(kRcThreads, 1)
rc_gemm_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_xt,
               const __grid_constant__ CUtensorMap tm_wk, const __grid_constant__ CUtensorMap tm_wv,
               const RcGemmParams p) {
  extern __shared__ uint8_t rc_smem_raw[];
  uint8_t* smem = rc_smem_raw + ((1024 - (smem_u32(rc_smem_raw) & 1023)) & 1023);
  RcCtrl* ctl = reinterpret_cast<RcCtrl*>(smem + kRcStages * kRcStageBytes);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int s = 0; s < kRcStages; ++s) { mbar_init(&ctl->full[s], 1); mbar_init(&ctl->empty[s], 1); }
    for (int b = 0; b < 2; ++b) { mbar_init(&ctl->acc_full[b], 1); mbar_init(&ctl->acc_empty[b], 128); }
    ctl->abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&ctl->tmem_base, 2 * kRcBNMax);   // two accumulators of up to 256 columns
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_x); tma_prefetch_desc(&tm_xt); tma_prefetch_desc(&tm_wk); tma_prefetch_desc(&tm_wv);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  pdl_wait();   // the plan and the page copies come from the kernels before this one

  int32_t* err = p.plan + kRcHdrErr;
  const int n_tok = __ldcg(p.plan + kRcHdrTok);
  const int hpt = p.heads_per_tile;            // 1 or 2: an output tile is hpt heads of K or of V
  const int bn = kRcHead * hpt;
  const int n_nt = 2 * p.num_kv_heads / hpt;
  const int n_tiles = ((n_tok + kRcBM - 1) / kRcBM) * n_nt;
  const int nk = p.d_model / kRcBK;
  const uint32_t tmem = ctl->tmem_base;
  volatile int* abort_flag = &ctl->abort;
  const int32_t* x_row = p.plan + p.lay.x_row;
  const int32_t* dst = p.plan + p.lay.dst;

  if (warp == 0) {
    // ---------------------------------------------------------- producer
    // Hidden states listed by selection rank are consecutive rows: one tiled
    // box of 128 rows per stage. Listed by doc position they are scattered:
    // 32 gather4 loads of four rows each (one per lane).
    const bool tiled = __ldcg(p.plan + kRcHdrBySel) != 0;
    uint32_t it = 0;
    int bad = 0;
    for (int tile = blockIdx.x; tile < n_tiles && !bad; tile += gridDim.x) {
      const int m0 = (tile / n_nt) * kRcBM;
      const int nt = tile % n_nt;
      int32_t r[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int t = m0 + 4 * lane + i;
        const int x = t < n_tok ? __ldcg(x_row + t) : -1;
        r[i] = (x < 0 || x >= p.x_rows) ? 0 : x;   // skipped rows read row 0; the epilogue stores nothing for them
      }
      const int h0 = nt * hpt;                 // first output head, over K heads then V heads
      const CUtensorMap* tb = h0 < p.num_kv_heads ? &tm_wk : &tm_wv;
      const int brow = (h0 % p.num_kv_heads) * kRcHead;
      for (int ks = 0; ks < nk; ++ks, ++it) {
        const int s = it % kRcStages;
        if (it >= uint32_t(kRcStages) && !mbar_wait(&ctl->empty[s], ((it / kRcStages) - 1) & 1, abort_flag)) {
          bad = 1;
          break;
        }
        uint8_t* sa = smem + s * kRcStageBytes;
        if (lane == 0) mbar_arrive_expect_tx(&ctl->full[s], kRcABytes + bn * kRcBK * 2);
        __syncwarp();
        if (tiled) {
          // rows past x_rows are filled with zeros; the epilogue stores nothing for them
          if (lane == 0) tma_load_2d(sa, &tm_xt, &ctl->full[s], ks * kRcBK, m0);
        } else {
          tma_gather4(sa + lane * 4 * 128, &tm_x, &ctl->full[s], ks * kRcBK, r[0], r[1], r[2], r[3]);
        }
        if (lane == 0) tma_load_2d(sa + kRcABytes, tb, &ctl->full[s], ks * kRcBK, brow);
      }
    }
    bad = __any_sync(0xffffffffu, bad);
    if (bad && lane == 0) rc_abort(ctl, err);
    // let every copy this warp issued land before the CTA exits
    if (lane == 0 && ctl->abort) {
      int zero = 0;
      const uint32_t first = it > uint32_t(kRcStages) ? it - kRcStages : 0;
      for (uint32_t t = first; t < it; ++t) mbar_wait(&ctl->full[t % kRcStages], (t / kRcStages) & 1, &zero);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(kRcBM, kRcHead * p.heads_per_tile, 0);
      uint32_t it = 0, tcount = 0;
      int bad = 0;
      for (int tile = blockIdx.x; tile < n_tiles && !bad; tile += gridDim.x, ++tcount) {
        const uint32_t buf = tcount & 1;
        if (tcount >= 2 && !mbar_wait(&ctl->acc_empty[buf], ((tcount - 2) >> 1) & 1, abort_flag)) { bad = 1; break; }
        tc_fence_after();
        const uint32_t d = tmem + buf * kRcBNMax;
        for (int ks = 0; ks < nk; ++ks, ++it) {
          const int s = it % kRcStages;
          if (!mbar_wait(&ctl->full[s], (it / kRcStages) & 1, abort_flag)) { bad = 1; break; }
          tc_fence_after();
          const uint32_t a = smem_u32(smem + s * kRcStageBytes);
          const uint32_t b = a + kRcABytes;
#pragma unroll
          for (int kk = 0; kk < kRcBK / 16; ++kk) mma_ss(d, rc_desc(a, kk), rc_desc(b, kk), idesc, (ks | kk) != 0);
          tc_commit(&ctl->empty[s]);
        }
        if (bad) break;
        tc_commit(&ctl->acc_full[buf]);
      }
      if (bad) rc_abort(ctl, err);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------- epilogue: thread = token row
    const int q = warp & 3;
    const int row = q * 32 + lane;
    const uint32_t lane_off = uint32_t(q * 32) << 16;
    uint32_t tcount = 0;
    int bad = 0;
    for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++tcount) {
      const uint32_t buf = tcount & 1;
      if (!mbar_wait(&ctl->acc_full[buf], (tcount >> 1) & 1, abort_flag)) { bad = 1; break; }
      tc_fence_after();
      const int m0 = (tile / n_nt) * kRcBM;
      const int nt = tile % n_nt;
      const int t = m0 + row;
      const int xr = t < n_tok ? __ldcg(x_row + t) : -1;
      const int dv = xr >= 0 ? __ldcg(dst + t) : 0;
      const int page = dv / kPage, slot = dv % kPage;
      const bool store = xr >= 0 && xr < p.x_rows && page >= 0 && page < p.num_pages;
      if (xr >= p.x_rows) atomicOr(err, kDevErrGeometry);
      else if (xr >= 0 && (page < 0 || page >= p.num_pages)) atomicOr(err, kDevErrPage);
      // one KV head (128 columns) at a time: read from TMEM, round, store
      for (int hh = 0; hh < hpt; ++hh) {
        float acc[kRcHead];
#pragma unroll
        for (int c = 0; c < kRcHead / 32; ++c) {
          uint32_t u[32];
          tmem_ld32(tmem + lane_off + buf * kRcBNMax + hh * kRcHead + 32 * c, u);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 32; ++j) acc[32 * c + j] = __uint_as_float(u[j]);
        }
        if (hh == hpt - 1) {
          tc_fence_before();
          mbar_arrive(&ctl->acc_empty[buf]);   // the accumulator is read: the next tile may overwrite it
        }
        if (store) {
          const int ho = nt * hpt + hh;       // output head over K heads then V heads
          const int head = ho % p.num_kv_heads;
          const bool is_v = ho >= p.num_kv_heads;
          __nv_bfloat16* pool = is_v ? p.pool_v : p.pool_k;
          bool over = false;
          const int64_t orow = ((int64_t(p.layer) * p.num_pages + page) * p.num_kv_heads + head) * kPage + slot;
          uint4* out = reinterpret_cast<uint4*>(pool + orow * kHeadDim);
#pragma unroll
          for (int c = 0; c < kRcHead / 8; ++c) {
            uint4 v;
            if (is_v) {
#pragma unroll
              for (int j = 0; j < 8; ++j) over |= beyond_f16(acc[8 * c + j]);
              v.x = pack_f16x2_sat(acc[8 * c + 0], acc[8 * c + 1]);
              v.y = pack_f16x2_sat(acc[8 * c + 2], acc[8 * c + 3]);
              v.z = pack_f16x2_sat(acc[8 * c + 4], acc[8 * c + 5]);
              v.w = pack_f16x2_sat(acc[8 * c + 6], acc[8 * c + 7]);
            } else {
              v.x = pack_bf16x2(acc[8 * c + 0], acc[8 * c + 1]);
              v.y = pack_bf16x2(acc[8 * c + 2], acc[8 * c + 3]);
              v.z = pack_bf16x2(acc[8 * c + 4], acc[8 * c + 5]);
              v.w = pack_bf16x2(acc[8 * c + 6], acc[8 * c + 7]);
            }
            out[c] = v;
          }
          if (over) atomicOr(err, kDevErrRange);
        }
      }
    }
    if (bad) rc_abort(ctl, err);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 2 * kRcBNMax);
  }
}

// ---------------------------------------------------------------- launchers

cudaError_t launch_rc_plan(const RcPlanParams& p, cudaStream_t stream) {
  return launch_pdl(rc_plan_kernel, dim3(1), dim3(kRcPlanThreads), 0, stream, 1, p);
}

cudaError_t launch_rc_copy(const RcCopyParams& p, int grid, cudaStream_t stream) {
  return launch_pdl(rc_copy_kernel, dim3(grid), dim3(kRcCopyThreads), 0, stream, 1, p);
}

cudaError_t launch_rc_gemm(const CUtensorMap& tx, const CUtensorMap& txt, const CUtensorMap& twk,
                           const CUtensorMap& twv, const RcGemmParams& p, int grid, cudaStream_t stream) {
  const size_t smem = rc_gemm_smem_bytes();
  static SmemAttr attr;
  cudaError_t e = ensure_smem_attr(rc_gemm_kernel, attr, smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(rc_gemm_kernel, dim3(grid), dim3(kRcThreads), smem, stream, 1, tx, txt, twk, twv, p);
}

}  // namespace rag
