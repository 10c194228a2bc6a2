// Impact pass (CacheBlend page, "Mathematical formulation": Impact(i) is the
// sum of the normalised attention weights alpha_{j,i} that tokens outside
// doc(i) give to token i; the `select_tokens_for_recompute` listing sums the
// query rows of the softmax over each column).
//
// alpha_{j,i} = exp(s_{j,i} - m_j) / l_j needs each row's final max and sum,
// which the attention pass leaves in (row_m2, row_il). This pass recomputes
// the scores in transposed form, S^T = K Q^T, so that a TMEM lane is a key:
// each thread sums its key's weights over up to 256 query rows with no
// cross-thread reduction, then adds the total into impact[] with one atomic.
//
//   producer warp : Q rows of the block (TMA, once per item) and K tiles
//                   gathered through the page table (TMA page boxes)
//   MMA warp      : S^T (128 keys x N rows) = K (smem) x Q^T (smem) -> TMEM,
//                   two S buffers ahead of the epilogue
//   8 epilogue warps: two per TMEM lane quarter, each over half of the rows;
//                   per key 2^(s c + b_row), with the row's normaliser folded
//                   into the bias b_row = log2(1 / (l H_q)) - m2, summed on
//                   MUFU exp2 with packed fp32 pair arithmetic; each half
//                   adds its column sum with one atomicAdd per key (16 warps,
//                   four per quarter, measured slower)
// The producer and MMA warps start while the kernels before this one finish
// (programmatic dependent launch); the epilogue waits for their row
// statistics.
// Impact is averaged over the H_q query heads (1/H_q is folded into row_il),
// so the impacts of all N_doc + q columns of a request add up to q.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "params.cuh"

namespace rag {

constexpr int kIKStages = 4;
constexpr int kIDescSlots = 6;
constexpr int kITileBytes = kBN * kHeadDim * 2;     // K tile
constexpr int kIHalf = kITileBytes / 2;
constexpr int kIQHalf = kImpactRows * 128;          // 256 rows x 64 d (bf16) per d-half
constexpr int kIQBytes = 2 * kIQHalf;
constexpr int kImpEpiWarps = 8;              // two per TMEM lane quarter, each over half of the rows
constexpr int kImpParts = kImpEpiWarps / 4;  // row parts per TMEM lane quarter
constexpr int kImpEpiThreads = kImpEpiWarps * 32;
constexpr int kWarpProducer = kImpEpiWarps, kWarpMma = kImpEpiWarps + 1, kWarpRope = kImpEpiWarps + 2;
constexpr int kImpThreads = (kImpEpiWarps + 3) * 32;   // epilogue + producer + MMA + RoPE warps

struct ImpDesc {
  int32_t kind;      // 0 doc tile, 1 query-key tile
  int32_t kbase;
  uint8_t nvalid[kPagesPerTile];
  int32_t lstart[kPagesPerTile];
};


struct ImpCtrl {
  uint64_t q_full, q_empty;
  uint64_t kfull[kIKStages], kempty[kIKStages], kconv[kIKStages];
  int32_t kchunk[kIKStages][kPagesPerTile];   // chunk-list entry per page of a K stage (-1: none)
  uint64_t s_full[2], s_free[2];
  uint64_t teardown;
  uint64_t desc_full[kIDescSlots], desc_empty[kIDescSlots];
  ImpDesc desc[kIDescSlots];
  ChunkCache chunks;
  alignas(16) float neg_m2[kImpactRows];   // per row: log2(1 / (l * H_q)) - m (log2 units; -inf: no row)
  uint32_t tmem_base;
  int32_t abort;
  int32_t total_items;
};

__host__ size_t impact_smem_bytes(int num_requests) {
  return 1024 + kIQBytes + size_t(kIKStages) * kITileBytes + sizeof(ImpCtrl) +
         sizeof(int32_t) * (num_requests + 1) + 64;
}

struct ImpItem {
  int b, g, rb, split, t_begin, t_end, n_doc_tiles, nrows, N;
  ReqInfo req;
};

__device__ __forceinline__ ImpItem decode_imp_item(const ImpactParams& p, const int32_t* prefix, int w) {
  const int B = p.batch.num_requests;
  int lo = 0, hi = B - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (prefix[mid] <= w) lo = mid; else hi = mid - 1;
  }
  ImpItem it;
  it.b = lo;
  it.req = load_req(p.batch, lo);
  const FwdShape sh = impact_shape(p.batch, it.req, p.group, p.tiles_per_split);
  int local = w - prefix[lo];
  it.rb = local % sh.n_rt;
  local /= sh.n_rt;
  it.split = local % sh.n_split;
  it.g = local / sh.n_split;
  it.n_doc_tiles = doc_tiles(it.req);
  const int G = p.group;
  const int last_tok = min(it.req.n_q, (it.rb + 1) * kImpactRows / G) - 1;
  const int n_tiles = it.n_doc_tiles + query_tiles_upto(last_tok);
  it.t_begin = min(it.split * p.tiles_per_split, n_tiles);
  it.t_end = min(it.t_begin + p.tiles_per_split, n_tiles);
  it.nrows = min(kImpactRows, it.req.n_q * G - it.rb * kImpactRows);
  it.N = (it.nrows + 32 * kImpParts - 1) / (32 * kImpParts) * (32 * kImpParts);   // parts of whole 32-column loads
  return it;
}

__device__ __forceinline__ uint64_t imp_kdesc(uint32_t base, int kk) {
  return sdesc_sw128(base + (kk >> 2) * kIHalf + (kk & 3) * 32, 16, 1024);
}
__device__ __forceinline__ uint64_t imp_qdesc(uint32_t base, int kk) {
  return sdesc_sw128(base + (kk >> 2) * kIQHalf + (kk & 3) * 32, 16, 1024);
}

__device__ __forceinline__ void imp_abort(ImpCtrl* c, int32_t* err) {
  if (!c->abort) {
    atomicOr(err, kDevErrTimeout);
    c->abort = 1;
  }
}

// The launch bounds let ptxas bound the registers by what one SM
// sub-partition's 16,384-register file holds for its share of the warps.
__global__ void __launch_bounds__(kImpThreads, 1)
impact_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
              const __grid_constant__ CUtensorMap tm_kq, const ImpactParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint8_t* sQ = smem;
  uint8_t* sK = smem + kIQBytes;
  ImpCtrl* ctl = reinterpret_cast<ImpCtrl*>(sK + kIKStages * kITileBytes);
  int32_t* prefix = reinterpret_cast<int32_t*>(ctl + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int B = p.batch.num_requests;
  const int G = p.group;
  pdl_launch_dependents();

  if (tid == 0) {
    mbar_init(&ctl->q_full, 1);
    mbar_init(&ctl->q_empty, 1);
    for (int s = 0; s < kIKStages; ++s) {
      mbar_init(&ctl->kfull[s], 1);
      mbar_init(&ctl->kempty[s], 1);
      mbar_init(&ctl->kconv[s], 1);
    }
    for (int s = 0; s < 2; ++s) { mbar_init(&ctl->s_full[s], 1); mbar_init(&ctl->s_free[s], kImpEpiThreads); }
    mbar_init(&ctl->teardown, 1);
    for (int s = 0; s < kIDescSlots; ++s) { mbar_init(&ctl->desc_full[s], 1); mbar_init(&ctl->desc_empty[s], kImpEpiWarps); }
    ctl->abort = 0;
    fence_mbar_init();
  }
  if (warp == kWarpMma) {
    tmem_alloc(&ctl->tmem_base, 512);
    tmem_relinquish();
  }
  if (warp == kWarpProducer && lane == 0) {
    tma_prefetch_desc(&tm_q); tma_prefetch_desc(&tm_k); tma_prefetch_desc(&tm_kq);
  }
  if (warp == 0) {
    int carry = 0;
    for (int base = 0; base < B; base += 32) {
      const int b = base + lane;
      int cnt = 0;
      if (b < B) {
        const ReqInfo r = load_req(p.batch, b);
        if (!req_ok(p.batch, r) && blockIdx.x == 0) atomicOr(p.err, kDevErrGeometry);
        const FwdShape sh = impact_shape(p.batch, r, G, p.tiles_per_split);
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
    if (lane == 0) { prefix[B] = carry; ctl->total_items = carry; }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  const int total_items = ctl->total_items;
  const uint32_t tmem = ctl->tmem_base;
  volatile int* abort_flag = &ctl->abort;

  if (warp < kImpEpiWarps) {
    // ------------------------------------------------------------ epilogue: thread = key
    // kImpParts warps per TMEM lane quarter: warps w, w + 4, ... share 32 keys
    // and take one part of the block's rows each; every warp adds its own
    // column sums (no barrier between the parts).
    const int part = warp >> 2;
    const int k = (warp & 3) * 32 + lane;
    const uint32_t lane_off = uint32_t((warp & 3) * 32) << 16;
    uint32_t t_glob = 0;
    int bad = 0;
    // The row statistics, and the zeroed impact vector, come from the kernels
    // before this one; the producer and MMA warps only read inputs and start
    // on the first tiles while those finish.
    pdl_wait();
    for (int w = blockIdx.x; w < total_items && !bad; w += gridDim.x) {
      const ImpItem it = decode_imp_item(p, prefix, w);
      const int n = it.t_end - it.t_begin;
      if (n == 0) continue;
      named_bar_sync(1, kImpEpiThreads);
      if (tid < kImpactRows) {
        const int r = tid;   // one row each
        // per row: -m + log2(1 / (l * H_q)), so that 2^(s*c + bias) is the
        // row's normalised weight already divided by H_q (-inf: no row)
        float bias = -INFINITY;
        if (r < it.nrows) {
          const int pr = it.rb * kImpactRows + r;
          const int64_t row = int64_t(it.req.q0 + pr / G) * p.num_q_heads + it.g * G + pr % G;
          const float il = p.row_il[row];
          bias = il > 0.f ? __log2f(il) - p.row_m2[row] : -INFINITY;
        }
        ctl->neg_m2[r] = bias;
      }
      named_bar_sync(1, kImpEpiThreads);
      float* seg = p.impact + (it.req.doc0 + it.req.q0);
      const int cols = it.N / kImpParts;   // rows of this part (a multiple of 32)
      const int c0 = part * cols;
      for (int i = 0; i < n; ++i) {
        const uint32_t t = t_glob + i;
        const uint32_t buf = t & 1;
        const uint32_t slot = t % kIDescSlots;
        if (!mbar_wait(&ctl->desc_full[slot], (t / kIDescSlots) & 1, abort_flag)) { bad = 1; break; }
        const ImpDesc* d = &ctl->desc[slot];
        const int kind = d->kind;
        bool valid;
        int lpos, rlim = 0;
        if (kind == 0) {
          const int pg = k >> 4, sl = k & 15;
          valid = sl < int(d->nvalid[pg]);
          lpos = d->lstart[pg] + sl;
        } else {
          const int kq = d->kbase + k;
          valid = kq < it.req.n_q;
          lpos = it.req.n_doc + kq;
          rlim = kq * G - it.rb * kImpactRows;   // rows r >= rlim see this key
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctl->desc_empty[slot]);
        if (!mbar_wait(&ctl->s_full[buf], (t >> 1) & 1, abort_flag)) { bad = 1; break; }
        tc_fence_after();
        const uint32_t col = tmem + lane_off + (buf ? 256u : 0u) + c0;
        // 32-column chunks with the next chunk's TMEM load in flight while the
        // current one is reduced; per score one packed FMA (scale and the
        // row's bias) per pair, one exp2 on MUFU, one packed add per pair
        const float2 sc2 = make_float2(p.scale_log2, p.scale_log2);
        float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                         make_float2(0.f, 0.f)};
        // doc tiles: every row sees every key, no mask
        auto chunk_doc = [&](const uint32_t (&u)[32], int cbase) {
#pragma unroll
          for (int j = 0; j < 32; j += 4) {
            const float4 b = *reinterpret_cast<const float4*>(&ctl->neg_m2[c0 + cbase + j]);
            const float2 e0 = ffma2(make_float2(__uint_as_float(u[j]), __uint_as_float(u[j + 1])), sc2,
                                    make_float2(b.x, b.y));
            const float2 e1 = ffma2(make_float2(__uint_as_float(u[j + 2]), __uint_as_float(u[j + 3])), sc2,
                                    make_float2(b.z, b.w));
            const int a = (j >> 1) & 2;
            acc[a] = fadd2(acc[a], make_float2(ex2(e0.x), ex2(e0.y)));
            acc[a + 1] = fadd2(acc[a + 1], make_float2(ex2(e1.x), ex2(e1.y)));
          }
        };
        // query-key tiles: row r sees this key from r >= rlim on (causal)
        auto chunk_query = [&](const uint32_t (&u)[32], int cbase) {
#pragma unroll
          for (int j = 0; j < 32; j += 4) {
            const int r0 = c0 + cbase + j;
            const float4 b = *reinterpret_cast<const float4*>(&ctl->neg_m2[r0]);
            const float2 e0 = ffma2(make_float2(__uint_as_float(u[j]), __uint_as_float(u[j + 1])), sc2,
                                    make_float2(b.x, b.y));
            const float2 e1 = ffma2(make_float2(__uint_as_float(u[j + 2]), __uint_as_float(u[j + 3])), sc2,
                                    make_float2(b.z, b.w));
            float v0 = ex2(e0.x), v1 = ex2(e0.y), v2 = ex2(e1.x), v3 = ex2(e1.y);
            if (r0 < rlim) v0 = 0.f;
            if (r0 + 1 < rlim) v1 = 0.f;
            if (r0 + 2 < rlim) v2 = 0.f;
            if (r0 + 3 < rlim) v3 = 0.f;
            const int a = (j >> 1) & 2;
            acc[a] = fadd2(acc[a], make_float2(v0, v1));
            acc[a + 1] = fadd2(acc[a + 1], make_float2(v2, v3));
          }
        };
        uint32_t ua[32], ub[32];
        tmem_ld32(col, ua);
        tmem_wait_ld();
        for (int c = 0; c < cols; c += 64) {
          const bool more_b = c + 32 < cols;
          if (more_b) tmem_ld32(col + c + 32, ub);
          if (kind == 0) chunk_doc(ua, c); else chunk_query(ua, c);
          tmem_wait_ld();
          if (!more_b) break;
          const bool more_a = c + 64 < cols;
          if (more_a) tmem_ld32(col + c + 64, ua);
          if (kind == 0) chunk_doc(ub, c + 32); else chunk_query(ub, c + 32);
          tmem_wait_ld();
        }
        tc_fence_before();
        mbar_arrive(&ctl->s_free[buf]);
        // each part adds its own column sum: no barrier between them
        const float2 a01 = fadd2(acc[0], acc[1]), a23 = fadd2(acc[2], acc[3]);
        const float total = (a01.x + a01.y) + (a23.x + a23.y);
        if (valid) atomicAdd(seg + lpos, total);
      }
      t_glob += n;
    }
    if (bad) imp_abort(ctl, p.err);
  } else if (warp == kWarpProducer) {
    // ------------------------------------------------------------ producer
    uint32_t t_glob = 0, q_iter = 0;
    int bad = 0;
    for (int w = blockIdx.x; w < total_items && !bad; w += gridDim.x) {
      const ImpItem it = decode_imp_item(p, prefix, w);
      const int n = it.t_end - it.t_begin;
      if (n == 0) continue;
      load_chunk_cache(&ctl->chunks, p.batch, it.req, lane);
      int32_t next_page = (it.t_begin < it.n_doc_tiles && lane < kPagesPerTile)
                              ? load_page_id(p.batch, it.req, it.t_begin * kPagesPerTile + lane)
                              : -1;
      if (q_iter > 0 && !mbar_wait(&ctl->q_empty, (q_iter - 1) & 1, abort_flag)) { bad = 1; break; }
      if (lane == 0) {
        const int nbox = (it.N + kBM - 1) / kBM;
        mbar_arrive_expect_tx(&ctl->q_full, nbox * 2 * (kBM * 128));
        for (int bi = 0; bi < nbox; ++bi) {
          const int tok0 = it.req.q0 + (it.rb * kImpactRows + bi * kBM) / G;
          tma_load_3d(sQ + bi * (kBM * 128), &tm_q, &ctl->q_full, 0, it.g * G, tok0);
          tma_load_3d(sQ + kIQHalf + bi * (kBM * 128), &tm_q, &ctl->q_full, 64, it.g * G, tok0);
        }
      }
      ++q_iter;
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
          pg = page_ref_cached(&ctl->chunks, p.batch, it.req, tile * kPagesPerTile + lane, page_id, p.num_pages,
                               p.err);
        const uint32_t slot = t % kIDescSlots;
        if (t >= kIDescSlots && !mbar_wait(&ctl->desc_empty[slot], ((t / kIDescSlots) - 1) & 1, abort_flag)) {
          bad = 1;
          break;
        }
        ImpDesc* d = &ctl->desc[slot];
        if (doc) {
          if (lane < kPagesPerTile) { d->nvalid[lane] = uint8_t(pg.nvalid); d->lstart[lane] = pg.lstart; }
          if (lane == 0) { d->kind = 0; d->kbase = 0; }
        } else if (lane == 0) {
          d->kind = 1;
          d->kbase = (tile - it.n_doc_tiles) * kBN;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctl->desc_full[slot]);
        const int s = t % kIKStages;
        if (t >= uint32_t(kIKStages) && !mbar_wait(&ctl->kempty[s], ((t / kIKStages) - 1) & 1, abort_flag)) {
          bad = 1;
          break;
        }
        if (lane < kPagesPerTile) ctl->kchunk[s][lane] = (doc && pg.page >= 0) ? pg.chunk : -1;
        __syncwarp();
        if (lane == 0) mbar_arrive_expect_tx(&ctl->kfull[s], kITileBytes);
        __syncwarp();
        uint8_t* dst = sK + s * kITileBytes;
        if (doc) {
          if (lane < kPagesPerTile) {
            const int row = pg.page >= 0 ? ((p.layer * p.num_pages + pg.page) * p.num_kv_heads + it.g) * kPage
                                         : -kPage;
            tma_load_2d(dst + lane * kPage * 128, &tm_k, &ctl->kfull[s], 0, row);
            tma_load_2d(dst + kIHalf + lane * kPage * 128, &tm_k, &ctl->kfull[s], 64, row);
          }
        } else if (lane == 0) {
          const int kq0 = it.req.q0 + (tile - it.n_doc_tiles) * kBN;
          tma_load_3d(dst, &tm_kq, &ctl->kfull[s], 0, it.g, kq0);
          tma_load_3d(dst + kIHalf, &tm_kq, &ctl->kfull[s], 64, it.g, kq0);
        }
      }
      t_glob += n;
    }
    if (bad) imp_abort(ctl, p.err);
    if (lane == 0 && ctl->abort) {
      int zero = 0;
      const uint32_t first = t_glob > uint32_t(kIKStages) ? t_glob - kIKStages : 0;
      for (uint32_t t = first; t < t_glob; ++t) mbar_wait(&ctl->kfull[t % kIKStages], (t / kIKStages) & 1, &zero);
      if (q_iter > 0) mbar_wait(&ctl->q_full, (q_iter - 1) & 1, &zero);
    }
    __syncwarp();
  } else if (warp == kWarpRope) {
    // ------------------------------------------------------------ RoPE re-basing of the K tiles
    if (p.rope) {
      uint32_t t_glob = 0;
      int bad = 0;
      for (int w = blockIdx.x; w < total_items && !bad; w += gridDim.x) {
        const ImpItem it = decode_imp_item(p, prefix, w);
        const int n = it.t_end - it.t_begin;
        for (int i = 0; i < n; ++i) {
          const uint32_t t = t_glob + i;
          const int s = t % kIKStages;
          if (!mbar_wait(&ctl->kfull[s], (t / kIKStages) & 1, abort_flag)) { bad = 1; break; }
          rope_rotate_tile(sK + s * kITileBytes, ctl->kchunk[s], p.rope, lane);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(&ctl->kconv[s]);
        }
        t_glob += n;
      }
      if (bad && lane == 0) imp_abort(ctl, p.err);
      __syncwarp();
    }
  } else {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t q_base = smem_u32(sQ);
      uint32_t t_glob = 0, q_iter = 0;
      int bad = 0;
      for (int w = blockIdx.x; w < total_items && !bad; w += gridDim.x) {
        const ImpItem it = decode_imp_item(p, prefix, w);
        const int n = it.t_end - it.t_begin;
        if (n == 0) continue;
        const uint32_t idesc = idesc_bf16_f32(kBN, it.N, 0);
        if (!mbar_wait(&ctl->q_full, q_iter & 1, abort_flag)) { bad = 1; break; }
        tc_fence_after();
        for (int i = 0; i < n; ++i) {
          const uint32_t t = t_glob + i;
          const int s = t % kIKStages;
          if (!mbar_wait(p.rope ? &ctl->kconv[s] : &ctl->kfull[s], (t / kIKStages) & 1, abort_flag)) {
            bad = 1;
            break;
          }
          if (t >= 2 && !mbar_wait(&ctl->s_free[t & 1], ((t - 2) >> 1) & 1, abort_flag)) { bad = 1; break; }
          tc_fence_after();
          const uint32_t k_base = smem_u32(sK + s * kITileBytes);
          const uint32_t d_s = tmem + ((t & 1) ? 256u : 0u);
#pragma unroll
          for (int kk = 0; kk < kHeadDim / 16; ++kk)
            mma_ss(d_s, imp_kdesc(k_base, kk), imp_qdesc(q_base, kk), idesc, kk > 0);
          tc_commit(&ctl->s_full[t & 1]);
          tc_commit(&ctl->kempty[s]);
        }
        if (bad) break;
        tc_commit(&ctl->q_empty);
        t_glob += n;
        ++q_iter;
      }
      if (bad) imp_abort(ctl, p.err);
      tc_commit(&ctl->teardown);
      int zero = 0;
      mbar_wait(&ctl->teardown, 0, &zero);
    }
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

cudaError_t launch_impact(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tkq,
                          const ImpactParams& p, int grid, cudaStream_t stream) {
  const size_t smem = impact_smem_bytes(p.batch.num_requests);
  static SmemAttr attr;
  cudaError_t e = ensure_smem_attr(impact_kernel, attr, smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(impact_kernel, dim3(grid), dim3(kImpThreads), smem, stream, 1, tq, tk, tkq, p);
}

}  // namespace rag
