// Attention pass of the fused prefill: the query block of each request
// attends over [K_1; ...; K_m; K_q] gathered from the paged pool
// (TurboRAG page, "Technical Details": Concat of the per-chunk caches and the
// query's own K/V; causal attention softmax(QK^T/sqrt(d_k) + M_causal) V).
//
// One persistent CTA per SM walks work items (request, kv head, 256-row
// block, split of the key tiles). Rows pack the G query heads of one KV head
// with the query tokens (row = token * G + head-in-group), so GQA groups share
// every K/V tile in the MMA M dimension. A block is two 128-row Q tiles that
// share each 128-key K/V tile:
//   K producer warp : Q tiles, then page table -> 8 TMA page boxes per K tile
//                     (or one box of K_q), and the tile's mask descriptor
//   V producer warp : the same for V
//   convert warp    : the tile of the query block's own V_q (a bf16 input)
//                     rounded to fp16 in place; with position re-basing, each
//                     K tile rotated in place to its concatenated positions
//   MMA warp        : S_i = Q_i K^T (tcgen05 smem x smem -> TMEM) for both Q
//                     tiles, then O_i += P_i V (P_i from TMEM, V from smem)
//   2 x 4 softmax warps: warpgroup i owns Q tile i; thread = row = TMEM lane;
//                     mask, online max/sum in the log2 domain, P_i (fp16)
//                     written over the columns of S_i, lazy O_i rescale
// The two softmax warpgroups alternate with the tensor core: while one
// computes exponentials the MMA warp runs the other Q tile's products.
// PV runs in fp16 (P and V): P keeps 3 more mantissa bits than bf16, and the
// pool of a bf16 cache stores V as fp16 already, so doc V tiles go from TMA
// to the tensor core untouched.
// Every exponential runs on MUFU: moving a share of them onto the FMA pipe
// as a polynomial measured slower on B200 (the softmax warps are bound by
// their issue rate, not by MUFU). Every wait is bounded; a timeout raises a
// device error instead of hanging.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "params.cuh"

namespace rag {

constexpr int kKStages = 2;
constexpr int kVStages = 2;
constexpr int kDescSlots = 4;
constexpr int kTileBytes = kBN * kHeadDim * 2;   // one K, V or Q tile, 16-bit
constexpr int kHalfBytes = kTileBytes / 2;       // 64 columns of d
constexpr int kFwdThreads = 384;                 // 8 softmax + K + V + MMA + convert warps
constexpr float kRescaleThreshold = 8.0f;        // log2 units: rescale O when the max grows by > 2^8

// TMEM columns: S_i (P_i aliased over its first 64 columns), O_i
__host__ __device__ constexpr uint32_t col_s(int qt) { return 128u * qt; }
__host__ __device__ constexpr uint32_t col_o(int qt) { return 256u + 128u * qt; }

struct TileDesc {
  int32_t kind;       // 0: doc tile from the pool, 1: query-key tile
  int32_t kbase;      // query tile: index of its first query key
  int32_t full;       // doc tile: every slot of the 8 pages is a real token
  uint8_t nvalid[kPagesPerTile];
};

struct FwdCtrl {
  uint64_t q_full, q_empty;
  uint64_t kfull[kKStages], kempty[kKStages], kconv[kKStages];
  uint64_t vfull[kVStages], vempty[kVStages], vconv[kVStages];
  int32_t kchunk[kKStages][kPagesPerTile];   // chunk-list entry per page of a K stage (-1: none)
  // s_full[b] / p_lo[b] / p_hi[b]: S buffer b (Q tile b's columns; with one Q
  // tile in the item, both buffers serve Q tile 0 in turn); P of keys 0-63 and
  // of keys 64-127 are published separately, so that PV over the first half
  // runs while the second half is exponentiated
  uint64_t s_full[kQTiles], p_lo[kQTiles], p_hi[kQTiles], pv_done[kQTiles], o_full[kQTiles], o_free[kQTiles];
  uint64_t teardown;
  uint64_t desc_full[kDescSlots], desc_empty[kDescSlots];
  TileDesc desc[kDescSlots];
  ChunkCache chunks[2];                 // one per producer warp
  uint32_t tmem_base;
  int32_t abort;
  int32_t total_items;
};

constexpr size_t kFwdSmemData = size_t(kQTiles + kKStages + kVStages) * kTileBytes;

__host__ size_t fwd_smem_bytes(int num_requests) {
  return 1024 + kFwdSmemData + sizeof(FwdCtrl) + sizeof(int32_t) * (num_requests + 1) + 64;
}

struct FwdItem {
  int b, g, rb, split;
  int n_qt;             // active Q tiles (1 or 2)
  int t_begin, t_end;   // tiles of the unit handled by this item
  int n_doc_tiles;
  ReqInfo req;
};

__device__ __forceinline__ FwdItem decode_fwd_item(const FwdParams& p, const int32_t* prefix, int w) {
  const int B = p.batch.num_requests;
  int lo = 0, hi = B - 1;
  while (lo < hi) {  // last b with prefix[b] <= w
    int mid = (lo + hi + 1) >> 1;
    if (prefix[mid] <= w) lo = mid; else hi = mid - 1;
  }
  FwdItem it;
  it.b = lo;
  it.req = load_req(p.batch, lo);
  const FwdShape sh = fwd_shape(p.batch, it.req, p.group, p.tiles_per_split);
  int local = w - prefix[lo];
  it.rb = local % sh.n_rt;
  local /= sh.n_rt;
  it.split = local % sh.n_split;
  it.g = local / sh.n_split;
  const int rows = it.req.n_q * p.group - it.rb * kFwdRows;
  it.n_qt = (rows > kBM && kFwdRows > kBM) ? 2 : 1;   // Q tiles holding rows of this block
  it.n_doc_tiles = doc_tiles(it.req);
  const int last_tok = min(it.req.n_q, (it.rb + 1) * kFwdRows / p.group) - 1;
  const int n_tiles = it.n_doc_tiles + query_tiles_upto(last_tok);
  it.t_begin = min(it.split * p.tiles_per_split, n_tiles);
  it.t_end = min(it.t_begin + p.tiles_per_split, n_tiles);
  return it;
}

__device__ __forceinline__ void raise_abort(FwdCtrl* c, int32_t* err) {
  if (!c->abort) {
    atomicOr(err, kDevErrTimeout);
    c->abort = 1;
  }
}

// Wait bounded by time only (teardown after an abort).
__device__ __forceinline__ void wait_quiet(uint64_t* bar, uint32_t parity) {
  int zero = 0;
  mbar_wait(bar, parity, &zero);
}

// K-major, 128B-swizzled tile of 128 rows x 128 16-bit values stored as two
// 64-column halves of 16 KB; k-step kk covers columns [16 kk, 16 kk + 16).
__device__ __forceinline__ uint64_t kmajor_desc(uint32_t base, int kk) {
  return sdesc_sw128(base + (kk >> 2) * kHalfBytes + (kk & 3) * 32, 16, 1024);
}
// V tile [128 keys][128 d] as the B operand with N = d contiguous (MN-major):
// k-step kk covers keys [16 kk, 16 kk + 16); the two 64-wide d halves are
// 16 KB apart (leading byte offset), 8-key groups 1 KB apart (stride).
__device__ __forceinline__ uint64_t v_desc(uint32_t base, int kk) {
  return sdesc_sw128(base + kk * 16 * 128, kHalfBytes, 1024);
}

__global__ void __launch_bounds__(kFwdThreads, 1)
attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_kq,
                const __grid_constant__ CUtensorMap tm_vq, const FwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + kQTiles * kTileBytes;
  uint8_t* sV = sK + kKStages * kTileBytes;
  FwdCtrl* ctl = reinterpret_cast<FwdCtrl*>(sV + kVStages * kTileBytes);
  int32_t* prefix = reinterpret_cast<int32_t*>(ctl + 1);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int B = p.batch.num_requests;
  const int G = p.group;

  // the kernels after this one (combine, impact) may start launching now;
  // they wait for this grid before they read what it writes
  pdl_launch_dependents();

  if (tid == 0) {
    mbar_init(&ctl->q_full, 1);
    mbar_init(&ctl->q_empty, 1);
    for (int s = 0; s < kKStages; ++s) {
      mbar_init(&ctl->kfull[s], 1);
      mbar_init(&ctl->kempty[s], 1);
      mbar_init(&ctl->kconv[s], 1);
    }
    for (int s = 0; s < kVStages; ++s) {
      mbar_init(&ctl->vfull[s], 1);
      mbar_init(&ctl->vempty[s], 1);
      mbar_init(&ctl->vconv[s], 1);
    }
    for (int q = 0; q < kQTiles; ++q) {
      mbar_init(&ctl->s_full[q], 1);
      mbar_init(&ctl->p_lo[q], 128);
      mbar_init(&ctl->p_hi[q], 128);
      mbar_init(&ctl->pv_done[q], 1);
      mbar_init(&ctl->o_full[q], 1);
      mbar_init(&ctl->o_free[q], 128);
    }
    mbar_init(&ctl->teardown, 1);
    for (int s = 0; s < kDescSlots; ++s) {
      mbar_init(&ctl->desc_full[s], 1);
      mbar_init(&ctl->desc_empty[s], 8);   // one arrival per softmax warp
    }
    ctl->abort = 0;
    fence_mbar_init();
  }
  if (warp == 10) {
    tmem_alloc(&ctl->tmem_base, 512);
    tmem_relinquish();
  }
  if (warp == 8 && lane == 0) {
    tma_prefetch_desc(&tm_q); tma_prefetch_desc(&tm_k); tma_prefetch_desc(&tm_kq);
  }
  if (warp == 9 && lane == 0) { tma_prefetch_desc(&tm_v); tma_prefetch_desc(&tm_vq); }

  // Reads and writes. The kernel reads only its inputs (the pool, the batch
  // descriptors, q, kq, vq), which no library kernel that releases its
  // dependents early writes, so producers, MMA and softmax start while the
  // previous kernel in the stream finishes; every thread that writes global
  // memory (the impact zeroing, the item offsets, the epilogue) first waits
  // for that kernel to complete (pdl_wait is free once it has).

  // zero the impact accumulator for the impact pass that follows
  if (p.impact_zero) {
    pdl_wait();
    for (int64_t i = int64_t(blockIdx.x) * blockDim.x + tid; i < p.impact_len;
         i += int64_t(gridDim.x) * blockDim.x)
      p.impact_zero[i] = 0.f;
  }

  // per-request item counts -> exclusive prefix (warp 0), total in ctl
  if (warp == 0) {
    int carry = 0;
    for (int base = 0; base < B; base += 32) {
      const int b = base + lane;
      int cnt = 0;
      if (b < B) {
        const ReqInfo r = load_req(p.batch, b);
        if (!req_ok(p.batch, r) && blockIdx.x == 0) atomicOr(p.err, kDevErrGeometry);
        const FwdShape sh = fwd_shape(p.batch, r, G, p.tiles_per_split);
        cnt = p.num_kv_heads * sh.n_split * sh.n_rt;
      }
      int incl = cnt;
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      if (b < B) prefix[b] = carry + incl - cnt;
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) {
      // more work than the workspace was sized for: descriptors disagree with
      // the host totals; report and do nothing
      if (carry > p.max_items) {
        if (blockIdx.x == 0) atomicOr(p.err, kDevErrGeometry);
        carry = 0;
        for (int b = 0; b < B; ++b) prefix[b] = 0;
      }
      prefix[B] = carry;
      ctl->total_items = carry;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (blockIdx.x == 0 && p.item_prefix) {
    pdl_wait();   // the previous call's combine may still read the offsets
    for (int b = tid; b <= B; b += blockDim.x) p.item_prefix[b] = prefix[b];
  }

  const int total_items = ctl->total_items;
  const uint32_t tmem = ctl->tmem_base;
  volatile int* abort_flag = &ctl->abort;

  // registers: the softmax warpgroups take 208 per thread, the four role warps 88
  if (warp < 8) {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 208;" ::: "memory");
    // ------------------------------------------------------------ softmax warpgroup qt
    const int qt = warp >> 2;
    const int r = tid & 127;
    const uint32_t lane_off = uint32_t((warp & 3) * 32) << 16;
    const uint32_t o_addr = tmem + lane_off + col_o(qt);
    uint32_t t_glob = 0;            // tiles seen by the CTA
    uint32_t n_sf0 = 0, n_sf1 = 0;  // completions of s_full[0] / s_full[1] consumed (one P written per completion)
    uint32_t n_pvq = 0;             // PVs into O_qt issued before the current step
    uint32_t n_of = 0;              // items whose O_qt has been read
    int bad = 0;
    for (int w = blockIdx.x; w < total_items && !bad; w += gridDim.x) {
      const FwdItem it = decode_fwd_item(p, prefix, w);
      const int n = it.t_end - it.t_begin;
      // One Q tile: warpgroup 0 alone, alternating between the two S buffers
      // so that S of the next tile is computed during this tile's softmax.
      const bool single = it.n_qt == 1;
      const bool active = qt < it.n_qt;
      const int pr = it.rb * kFwdRows + qt * kBM + r;
      const int tok = pr / G;
      const int head = it.g * G + (pr % G);
      const bool row_valid = active && tok < it.req.n_q;
      // A warp whose 32 rows are all past the query block (short queries,
      // decode steps) skips the softmax and the epilogue's loads and stores;
      // it still waits for every S and O and makes every arrival, so the
      // barrier phases stay in step with the warps that hold real rows.
      const bool warp_live = __any_sync(0xffffffffu, row_valid);
      float m_ref = -INFINITY, l_sum = 0.f;
      for (int i = 0; i < n; ++i) {
        const uint32_t t = t_glob + i;
        const uint32_t slot = t % kDescSlots;
        if (!mbar_wait(&ctl->desc_full[slot], (t / kDescSlots) & 1, abort_flag)) { bad = 1; break; }
        const TileDesc td = ctl->desc[slot];
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctl->desc_empty[slot]);
        if (!active) continue;
        const int sb = single ? (i & 1) : qt;   // S buffer of this step
        const uint32_t s_addr = tmem + lane_off + col_s(sb);
        if (!mbar_wait(&ctl->s_full[sb], (sb ? n_sf1 : n_sf0) & 1, abort_flag)) { bad = 1; break; }
        tc_fence_after();
        if (!warp_live) {
          mbar_arrive(&ctl->p_lo[sb]);
          mbar_arrive(&ctl->p_hi[sb]);
          if (sb) ++n_sf1; else ++n_sf0;
          ++n_pvq;
          continue;
        }
        float x[kBN];
        {
          // the whole row in one round trip: four loads, one wait
          uint32_t u0[32], u1[32], u2[32], u3[32];
          tmem_ld32(s_addr + 0, u0);
          tmem_ld32(s_addr + 32, u1);
          tmem_ld32(s_addr + 64, u2);
          tmem_ld32(s_addr + 96, u3);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            x[j] = __uint_as_float(u0[j]);
            x[32 + j] = __uint_as_float(u1[j]);
            x[64 + j] = __uint_as_float(u2[j]);
            x[96 + j] = __uint_as_float(u3[j]);
          }
        }
        // mask (only partial tiles), then the row max of the raw scores
        if (td.kind == 0) {
          if (!td.full) {
            const uint32_t nv_lo = *reinterpret_cast<const uint32_t*>(&td.nvalid[0]);
            const uint32_t nv_hi = *reinterpret_cast<const uint32_t*>(&td.nvalid[4]);
#pragma unroll
            for (int c = 0; c < kBN; ++c) {
              const int pg = c >> 4;
              const uint32_t nv = ((pg < 4 ? nv_lo >> (8 * pg) : nv_hi >> (8 * (pg - 4))) & 0xffu);
              if (uint32_t(c & 15) >= nv) x[c] = -INFINITY;
            }
          }
        } else {
          const int lim = tok - td.kbase;   // keys c <= lim are visible
          if (lim < kBN - 1) {
#pragma unroll
            for (int c = 0; c < kBN; ++c)
              if (c > lim) x[c] = -INFINITY;
          }
        }
        // row max: four independent 3-input max chains
        float mq[4] = {x[0], x[1], x[2], x[3]};
#pragma unroll
        for (int c = 4; c < kBN; c += 8) {
#pragma unroll
          for (int a = 0; a < 4; ++a) mq[a] = fmax3(mq[a], x[c + 2 * a], x[c + 2 * a + 1]);
        }
        float mx = fmax3(fmaxf(mq[0], mq[1]), mq[2], mq[3]);
        mx = mx * p.scale_log2;   // scale > 0: max of scaled = scaled max
        float alpha = 1.f;
        bool need = false;
        if (i == 0) {
          m_ref = mx;
        } else if (mx > m_ref + kRescaleThreshold) {
          alpha = ex2(m_ref - mx);
          need = true;
        }
        if (__any_sync(0xffffffffu, need)) {
          // O must hold the previous tile's PV before it is rescaled. The PV
          // before that is complete (it was issued ahead of this tile's QK,
          // whose result is here), so the parity names exactly PV(n_pvq - 1).
          if (!mbar_wait(&ctl->pv_done[qt], (n_pvq - 1) & 1, abort_flag)) { bad = 1; break; }
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t u[32];
            tmem_ld32(o_addr + 32 * c, u);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 32; ++j) u[j] = __float_as_uint(__uint_as_float(u[j]) * alpha);
            tmem_st32(o_addr + 32 * c, u);
          }
          tmem_wait_st();
          if (need) { l_sum *= alpha; m_ref = mx; }
        }
        const float neg_m = (m_ref == -INFINITY) ? 0.f : -m_ref;
        const float2 sc2 = make_float2(p.scale_log2, p.scale_log2);
        const float2 nm2 = make_float2(neg_m, neg_m);
        float2 ls[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                        make_float2(0.f, 0.f)};
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t pk[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const float2 y = ffma2(make_float2(x[64 * h + 2 * j], x[64 * h + 2 * j + 1]), sc2, nm2);
            const float2 e = make_float2(ex2(y.x), ex2(y.y));
            ls[j & 3] = fadd2(ls[j & 3], e);
            pk[j] = pack_f16x2(e.x, e.y);
          }
          tmem_st32(s_addr + 32 * h, pk);   // P over the first 64 columns of S
          // publish this half of P: PV over its 64 keys may start
          tmem_wait_st();
          tc_fence_before();
          mbar_arrive(h == 0 ? &ctl->p_lo[sb] : &ctl->p_hi[sb]);
        }
        const float2 ls01 = fadd2(ls[0], ls[1]), ls23 = fadd2(ls[2], ls[3]);
        l_sum += (ls01.x + ls01.y) + (ls23.x + ls23.y);
        if (sb) ++n_sf1; else ++n_sf0;
        ++n_pvq;
      }
      if (bad) break;
      t_glob += n;
      // completions of s_full[1] that the other warpgroup consumed: the odd
      // tiles of a one-Q-tile item (warpgroup 0's), every tile of a two-Q-tile
      // item (warpgroup 1's)
      if (single && qt == 1) n_sf1 += uint32_t(n) / 2;
      if (!single && qt == 0) n_sf1 += uint32_t(n);
      if (!active) continue;

      // ---- epilogue: O of this Q tile
      if (n > 0) {
        // the MMA warp commits o_full once per item after the item's last PV
        if (!mbar_wait(&ctl->o_full[qt], n_of & 1, abort_flag)) { bad = 1; break; }
        ++n_of;
        tc_fence_after();
      }
      if (!warp_live) {   // no row of this warp is read or written
        if (n > 0) {
          tc_fence_before();
          mbar_arrive(&ctl->o_free[qt]);
        }
        continue;
      }
      pdl_wait();   // outputs and partials may still be read by the previous kernel
      float o[kHeadDim];
      if (n > 0) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t u[32];
          tmem_ld32(o_addr + 32 * c, u);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 32; ++j) o[32 * c + j] = __uint_as_float(u[j]);
        }
        tc_fence_before();
        mbar_arrive(&ctl->o_free[qt]);
      } else {
#pragma unroll
        for (int j = 0; j < kHeadDim; ++j) o[j] = 0.f;
      }
      if (p.direct) {
        if (row_valid) {
          const float inv = l_sum > 0.f ? 1.f / l_sum : 0.f;
          const int64_t row = int64_t(it.req.q0 + tok) * p.num_q_heads + head;
          uint4* dst = reinterpret_cast<uint4*>(p.o + row * kHeadDim);
#pragma unroll
          for (int c = 0; c < kHeadDim / 8; ++c) {
            uint4 v;
            v.x = pack_bf16x2(o[8 * c + 0] * inv, o[8 * c + 1] * inv);
            v.y = pack_bf16x2(o[8 * c + 2] * inv, o[8 * c + 3] * inv);
            v.z = pack_bf16x2(o[8 * c + 4] * inv, o[8 * c + 5] * inv);
            v.w = pack_bf16x2(o[8 * c + 6] * inv, o[8 * c + 7] * inv);
            dst[c] = v;
          }
          const float m_use = (m_ref == -INFINITY) ? 0.f : m_ref;
          p.row_m2[row] = m_use;
          p.row_il[row] = l_sum > 0.f ? 1.f / (l_sum * float(p.num_q_heads)) : 0.f;
          if (p.row_lse) p.row_lse[row] = (m_use + __log2f(l_sum)) * 0.69314718055994531f;
        }
      } else {
        // partial row: this split's own softmax average O/l in fp16 (|O/l| is
        // bounded by max |V|), then its reference max m and sum l in fp32
        const float inv = l_sum > 0.f ? 1.f / l_sum : 0.f;
        uint4* dst = reinterpret_cast<uint4*>(p.part + (size_t(w) * kFwdRows + qt * kBM + r) * kPartStride);
#pragma unroll
        for (int c = 0; c < kHeadDim / 8; ++c) {
          uint4 v;
          v.x = pack_f16x2(o[8 * c + 0] * inv, o[8 * c + 1] * inv);
          v.y = pack_f16x2(o[8 * c + 2] * inv, o[8 * c + 3] * inv);
          v.z = pack_f16x2(o[8 * c + 4] * inv, o[8 * c + 5] * inv);
          v.w = pack_f16x2(o[8 * c + 6] * inv, o[8 * c + 7] * inv);
          dst[c] = v;
        }
        reinterpret_cast<float4*>(dst + kHeadDim / 8)[0] = make_float4(m_ref, l_sum, 0.f, 0.f);
      }
    }
    if (bad) raise_abort(ctl, p.err);
  } else {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 88;" ::: "memory");
    if (warp == 8 || warp == 9) {
    // ------------------------------------------------------------ producers
    const bool is_k = (warp == 8);
    const CUtensorMap* tm_pool = is_k ? &tm_k : &tm_v;
    const CUtensorMap* tm_qkv = is_k ? &tm_kq : &tm_vq;
    uint8_t* sbase = is_k ? sK : sV;
    const int nstages = is_k ? kKStages : kVStages;
    uint64_t* full = is_k ? ctl->kfull : ctl->vfull;
    uint64_t* empty = is_k ? ctl->kempty : ctl->vempty;
    uint32_t t_glob = 0, q_iter = 0;
    int bad = 0;
    for (int w = blockIdx.x; w < total_items && !bad; w += gridDim.x) {
      const FwdItem it = decode_fwd_item(p, prefix, w);
      const int n = it.t_end - it.t_begin;
      if (n == 0) continue;
      ChunkCache* cc = &ctl->chunks[is_k ? 0 : 1];
      load_chunk_cache(cc, p.batch, it.req, lane);
      int32_t next_page = (it.t_begin < it.n_doc_tiles && lane < kPagesPerTile)
                              ? load_page_id(p.batch, it.req, it.t_begin * kPagesPerTile + lane)
                              : -1;
      if (is_k) {
        if (q_iter > 0 && !mbar_wait(&ctl->q_empty, (q_iter - 1) & 1, abort_flag)) { bad = 1; break; }
        if (lane == 0) {
          mbar_arrive_expect_tx(&ctl->q_full, it.n_qt * kTileBytes);
          for (int q = 0; q < it.n_qt; ++q) {
            const int tok0 = it.req.q0 + (it.rb * kFwdRows + q * kBM) / G;
            tma_load_3d(sQ + q * kTileBytes, &tm_q, &ctl->q_full, 0, it.g * G, tok0);
            tma_load_3d(sQ + q * kTileBytes + kHalfBytes, &tm_q, &ctl->q_full, 64, it.g * G, tok0);
          }
          // warm L2 with the Q rows of this CTA's next item
          const int wn = w + int(gridDim.x);
          if (wn < total_items) {
            const FwdItem nx = decode_fwd_item(p, prefix, wn);
            for (int q = 0; q < nx.n_qt; ++q) {
              const int tok0 = nx.req.q0 + (nx.rb * kFwdRows + q * kBM) / G;
              tma_prefetch_3d(&tm_q, 0, nx.g * G, tok0);
              tma_prefetch_3d(&tm_q, 64, nx.g * G, tok0);
            }
          }
        }
        ++q_iter;
      }
      for (int i = 0; i < n; ++i) {
        const uint32_t t = t_glob + i;
        const int tile = it.t_begin + i;
        const bool doc = tile < it.n_doc_tiles;
        const int32_t page_id = next_page;
        next_page = (tile + 1 < it.n_doc_tiles && lane < kPagesPerTile)
                        ? load_page_id(p.batch, it.req, (tile + 1) * kPagesPerTile + lane)
                        : -1;
        PageRef pg;
        pg.page = -1; pg.nvalid = 0; pg.lstart = 0;
        if (doc && lane < kPagesPerTile)
          pg = page_ref_cached(cc, p.batch, it.req, tile * kPagesPerTile + lane, page_id, p.num_pages,
                               is_k ? p.err : nullptr);
        if (is_k) {
          const uint32_t slot = t % kDescSlots;
          if (t >= kDescSlots && !mbar_wait(&ctl->desc_empty[slot], ((t / kDescSlots) - 1) & 1, abort_flag)) {
            bad = 1;
            break;
          }
          TileDesc* d = &ctl->desc[slot];
          const unsigned full_pages = __ballot_sync(0xffffffffu, lane < kPagesPerTile && pg.nvalid == kPage);
          if (doc) {
            if (lane < kPagesPerTile) d->nvalid[lane] = uint8_t(pg.nvalid);
            if (lane == 0) { d->kind = 0; d->kbase = 0; d->full = (full_pages == 0xffu) ? 1 : 0; }
          } else if (lane == 0) {
            d->kind = 1;
            d->kbase = (tile - it.n_doc_tiles) * kBN;
            d->full = 0;
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(&ctl->desc_full[slot]);
        }
        const int s = t % nstages;
        if (t >= uint32_t(nstages) && !mbar_wait(&empty[s], ((t / nstages) - 1) & 1, abort_flag)) {
          bad = 1;
          break;
        }
        if (is_k && lane < kPagesPerTile) ctl->kchunk[s][lane] = (doc && pg.page >= 0) ? pg.chunk : -1;
        __syncwarp();
        if (lane == 0) mbar_arrive_expect_tx(&full[s], kTileBytes);
        __syncwarp();
        uint8_t* dst = sbase + s * kTileBytes;
        if (doc) {
          if (lane < kPagesPerTile) {
            const int row = pg.page >= 0
                                ? ((p.layer * p.num_pages + pg.page) * p.num_kv_heads + it.g) * kPage
                                : -kPage;   // fully out of range: the box is zero-filled
            tma_load_2d(dst + lane * kPage * 128, tm_pool, &full[s], 0, row);
            tma_load_2d(dst + kHalfBytes + lane * kPage * 128, tm_pool, &full[s], 64, row);
          }
        } else if (lane == 0) {
          const int kq0 = it.req.q0 + (tile - it.n_doc_tiles) * kBN;
          tma_load_3d(dst, tm_qkv, &full[s], 0, it.g, kq0);
          tma_load_3d(dst + kHalfBytes, tm_qkv, &full[s], 64, it.g, kq0);
        }
      }
      t_glob += n;
    }
    if (bad) raise_abort(ctl, p.err);
    // let every copy this warp issued land before the CTA exits
    if (lane == 0 && ctl->abort) {
      const uint32_t first = t_glob > uint32_t(nstages) ? t_glob - nstages : 0;
      for (uint32_t t = first; t < t_glob; ++t) wait_quiet(&full[t % nstages], (t / nstages) & 1);
      if (is_k && q_iter > 0) wait_quiet(&ctl->q_full, (q_iter - 1) & 1);
    }
    __syncwarp();
  } else if (warp == 11) {
    // ------------------------------------------------------------ convert warp
    // Per tile, in order: with position re-basing, the K tile is rotated in
    // place to the concatenated positions of its keys; then the V stage is
    // released to the MMA warp (vconv), after rounding it from bf16 to fp16 in
    // place when it holds the query block's own V_q (doc V tiles are fp16 in
    // the pool already). Every bf16 V_q value of magnitude in [2^-14, 65280]
    // is exact in fp16; magnitudes from 65536 up, inf and nan saturate and
    // raise kDevErrRange. Rows past the request's query block are zeroed (a
    // masked key must still hold a finite value). The 128B swizzle is
    // unchanged by an elementwise rewrite.
    uint32_t t_glob = 0;
    int bad = 0;
    uint32_t range = 0;
    for (int w = blockIdx.x; w < total_items && !bad; w += gridDim.x) {
      const FwdItem it = decode_fwd_item(p, prefix, w);
      const int n = it.t_end - it.t_begin;
      for (int i = 0; i < n; ++i) {
        const uint32_t t = t_glob + i;
        const int tile = it.t_begin + i;
        if (p.rope) {
          const int sk = t % kKStages;
          if (!mbar_wait(&ctl->kfull[sk], (t / kKStages) & 1, abort_flag)) { bad = 1; break; }
          rope_rotate_tile(sK + sk * kTileBytes, ctl->kchunk[sk], p.rope, lane);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(&ctl->kconv[sk]);
        }
        const int s = t % kVStages;
        if (!mbar_wait(&ctl->vfull[s], (t / kVStages) & 1, abort_flag)) { bad = 1; break; }
        if (tile >= it.n_doc_tiles) {
          const int rows = min(kBN, it.req.n_q - (tile - it.n_doc_tiles) * kBN);
          uint8_t* base = sV + s * kTileBytes;
#pragma unroll 4
          for (int u = lane; u < kBN * (kHeadDim / 8); u += 32) {
            const int r = u >> 4, c = u & 15;   // row, 16-byte chunk of the row
            uint4* at = reinterpret_cast<uint4*>(base + (c >> 3) * kHalfBytes + r * 128 + ((c & 7) << 4));
            *at = r < rows ? bf16x8_to_f16x8(*at, range) : make_uint4(0u, 0u, 0u, 0u);
          }
          fence_proxy_async_smem();
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctl->vconv[s]);
      }
      t_glob += n;
    }
    if (bad) raise_abort(ctl, p.err);
    if (range_exceeded(range)) atomicOr(p.err, kDevErrRange);
    __syncwarp();
  } else {
    // ------------------------------------------------------------ MMA issuer (warp 10)
    if (lane == 0) {
      const uint32_t idesc_qk = idesc_bf16_f32(kBM, kBN, 0);
      const uint32_t idesc_pv = idesc_f16_f32(kBM, kHeadDim, 1);
      const uint32_t q_base = smem_u32(sQ);
      uint32_t t_glob = 0, q_iter = 0;
      uint32_t n_pf0 = 0, n_pf1 = 0;       // completions of p_lo/p_hi[0] and [1] consumed
      uint32_t n_item[kQTiles] = {0, 0};   // items begun, per Q tile
      int bad = 0;
      for (int w = blockIdx.x; w < total_items && !bad; w += gridDim.x) {
        const FwdItem it = decode_fwd_item(p, prefix, w);
        const int n = it.t_end - it.t_begin;
        if (n == 0) continue;
        if (!mbar_wait(&ctl->q_full, q_iter & 1, abort_flag)) { bad = 1; break; }
        tc_fence_after();
        if (it.n_qt == 1) {
          // One Q tile, two S buffers: QK of tiles 0 and 1 first, then per tile
          // i, PV(i) as soon as its P is written and QK(i + 2) into the buffer
          // PV(i) has just read (issue order keeps them apart).
          auto qk = [&](int j) {
            const uint32_t t = t_glob + j;
            const int s = t % kKStages;
            if (!mbar_wait(p.rope ? &ctl->kconv[s] : &ctl->kfull[s], (t / kKStages) & 1, abort_flag)) return false;
            const uint32_t k_base = smem_u32(sK + s * kTileBytes);
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < kHeadDim / 16; ++kk)
              mma_ss(tmem + col_s(j & 1), kmajor_desc(q_base, kk), kmajor_desc(k_base, kk), idesc_qk, kk > 0);
            tc_commit(&ctl->s_full[j & 1]);
            tc_commit(&ctl->kempty[s]);
            if (j == n - 1) tc_commit(&ctl->q_empty);   // the rest of the item reads no Q
            return true;
          };
          for (int j = 0; j < n && j < 2 && !bad; ++j)
            if (!qk(j)) bad = 1;
          for (int i = 0; i < n && !bad; ++i) {
            const uint32_t t = t_glob + i;
            const int sv = t % kVStages;
            const int b = i & 1;
            // doc V tiles straight from TMA; the V_q tile once it is fp16
            const bool v_doc = it.t_begin + i < it.n_doc_tiles;
            if (!mbar_wait(v_doc ? &ctl->vfull[sv] : &ctl->vconv[sv], (t / kVStages) & 1, abort_flag)) {
              bad = 1;
              break;
            }
            if (i == 0) {
              if (n_item[0] > 0 && !mbar_wait(&ctl->o_free[0], (n_item[0] - 1) & 1, abort_flag)) { bad = 1; break; }
              ++n_item[0];
            }
            uint32_t& npf = b ? n_pf1 : n_pf0;
            const uint32_t v_base = smem_u32(sV + sv * kTileBytes);
            bool ok = true;
            for (int hh = 0; hh < 2 && ok; ++hh) {
              if (!mbar_wait(hh == 0 ? &ctl->p_lo[b] : &ctl->p_hi[b], npf & 1, abort_flag)) { ok = false; break; }
              tc_fence_after();
#pragma unroll
              for (int kk = 4 * hh; kk < 4 * hh + 4; ++kk)
                mma_ts(tmem + col_o(0), tmem + col_s(b) + kk * 8, v_desc(v_base, kk), idesc_pv, (i > 0) || (kk > 0));
            }
            if (!ok) { bad = 1; break; }
            ++npf;
            tc_commit(&ctl->pv_done[0]);
            if (i == n - 1) tc_commit(&ctl->o_full[0]);
            tc_commit(&ctl->vempty[sv]);
            if (i + 2 < n && !qk(i + 2)) { bad = 1; break; }
          }
          if (bad) break;
          t_glob += n;
          ++q_iter;
          continue;
        }
        // Tensor-core order per step: PV_0(t-1), QK_0(t), PV_1(t-1), QK_1(t), so
        // that softmax 0 of tile t runs while the pipe does PV_1 and QK_1.
        for (int i = 0; i <= n && !bad; ++i) {
          const uint32_t t = t_glob + i;          // tile of the QK products of this step
          const uint32_t tp = t - 1;              // tile of the PV products of this step
          const int s = t % kKStages;
          const int sv = tp % kVStages;
          uint32_t v_base = 0;
          const uint32_t k_base = smem_u32(sK + s * kTileBytes);
          if (i >= 1) {
            const bool v_doc = it.t_begin + i - 1 < it.n_doc_tiles;
            if (!mbar_wait(v_doc ? &ctl->vfull[sv] : &ctl->vconv[sv], (tp / kVStages) & 1, abort_flag)) {
              bad = 1;
              break;
            }
            v_base = smem_u32(sV + sv * kTileBytes);
          }
          for (int q = 0; q < it.n_qt && !bad; ++q) {
            if (i >= 1) {
              // O_q += P_q V for the previous tile
              if (i == 1) {
                if (n_item[q] > 0 && !mbar_wait(&ctl->o_free[q], (n_item[q] - 1) & 1, abort_flag)) {
                  bad = 1;
                  break;
                }
                ++n_item[q];
              }
              uint32_t& npf = q ? n_pf1 : n_pf0;
              bool ok = true;
              for (int hh = 0; hh < 2 && ok; ++hh) {
                if (!mbar_wait(hh == 0 ? &ctl->p_lo[q] : &ctl->p_hi[q], npf & 1, abort_flag)) { ok = false; break; }
                tc_fence_after();
#pragma unroll
                for (int kk = 4 * hh; kk < 4 * hh + 4; ++kk)
                  mma_ts(tmem + col_o(q), tmem + col_s(q) + kk * 8, v_desc(v_base, kk), idesc_pv,
                         (i > 1) || (kk > 0));
              }
              if (!ok) { bad = 1; break; }
              ++npf;
              tc_commit(&ctl->pv_done[q]);
              if (i == n) tc_commit(&ctl->o_full[q]);   // O_q of this item is complete
              if (q == it.n_qt - 1) tc_commit(&ctl->vempty[sv]);   // the last read of this V stage
            }
            if (i < n) {
              // K of this tile is waited for only here, so that PV_0 of the
              // previous tile never waits on the next tile's load
              if (q == 0 &&
                  !mbar_wait(p.rope ? &ctl->kconv[s] : &ctl->kfull[s], (t / kKStages) & 1, abort_flag)) {
                bad = 1;
                break;
              }
              // S_q = Q_q K^T for this tile. It overwrites P_q (aliased over S_q),
              // which PV_q of the previous tile reads: tcgen05.mma operations of
              // one CTA execute in issue order, so no completion wait is needed.
              tc_fence_after();
              const uint32_t qb = q_base + q * kTileBytes;
#pragma unroll
              for (int kk = 0; kk < kHeadDim / 16; ++kk)
                mma_ss(tmem + col_s(q), kmajor_desc(qb, kk), kmajor_desc(k_base, kk), idesc_qk, kk > 0);
              tc_commit(&ctl->s_full[q]);
            }
          }
          if (bad) break;
          if (i < n) tc_commit(&ctl->kempty[s]);
          // the drain step reads no Q: the next item's Q may load now
          if (i == n - 1) tc_commit(&ctl->q_empty);
        }
        if (bad) break;
        t_glob += n;
        ++q_iter;
      }
      if (bad) raise_abort(ctl, p.err);
      // every MMA issued so far completes before TMEM is released
      tc_commit(&ctl->teardown);
      wait_quiet(&ctl->teardown, 0);
    }
    __syncwarp();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 10) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------- RoPE table

// Per chunk-list entry e of request b, the re-basing angle of every rotary
// pair: offset o_e (doc tokens of the request before the entry) times
// theta_i = base^(-2 i / 128), as (cos, sin), computed in fp64 and stored in
// fp32. One block per request.
__global__ void __launch_bounds__(256) rope_table_kernel(const BatchDev B, double base, float2* table) {
  // no early release: the attention kernel reads the table before its own
  // wait, so it must start only once the table is complete
  const ReqInfo r = load_req(B, blockIdx.x);
  if (!req_ok(B, r)) return;
  pdl_wait();   // the kernel before this one may still read the table of the previous call
  const int n = (r.c1 - r.c0) * 64;
  for (int idx = threadIdx.x; idx < n; idx += blockDim.x) {
    const int e = r.c0 + idx / 64, i = idx % 64;
    const double o = double(__ldg(B.chunk_doc_off + e) - r.doc0);
    const double theta = pow(base, -2.0 * double(i) / double(kHeadDim));
    double sn, cn;
    sincos(o * theta, &sn, &cn);
    table[int64_t(e) * 64 + i] = make_float2(float(cn), float(sn));
  }
}

// ---------------------------------------------------------------- launchers

cudaError_t launch_rope_table(const BatchDev& b, double base, float2* table, cudaStream_t stream) {
  return launch_pdl(rope_table_kernel, dim3(b.num_requests), dim3(256), 0, stream, 1, b, base, table);
}

cudaError_t launch_attn_fwd(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const CUtensorMap& tkq, const CUtensorMap& tvq, const FwdParams& p, int grid,
                            cudaStream_t stream) {
  const size_t smem = fwd_smem_bytes(p.batch.num_requests);
  static SmemAttr attr;
  cudaError_t e = ensure_smem_attr(attn_fwd_kernel, attr, smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(attn_fwd_kernel, dim3(grid), dim3(kFwdThreads), smem, stream, 1, tq, tk, tv, tkq, tvq, p);
}

}  // namespace rag
