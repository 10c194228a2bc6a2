// Attention pass for short query blocks: at most 16 rows (query tokens x the
// query heads of one KV head) per unit, as in a decode step (one new token
// attending over the request's chunks and its own context; TurboRAG page,
// "Technical Details": the same softmax(QK^T/sqrt(d_k) + M_causal) V over the
// concatenated cache).
//
// With so few rows the prefill kernel's softmax, a row per thread, leaves one
// warp computing 128 exponentials per row. Here the products are transposed
// so that a thread owns a key instead of a row:
//   S^T = K Q^T   (tcgen05, A = K tile [128 keys x 128 d], B = Q [16 rows])
//   per row: max over the 128 keys by warp shuffles and a shared exchange
//   between the four key warps, one exponential per row and thread, the rows
//   padded to R = 4, 8 or 16 (compiled for each; a decode step with G = 4
//   has 4), P^T (fp16, [16 rows x 128 keys]) written to shared memory,
//   O^T += V^T P^T (A = the V tile read as [d x keys], B = P^T)
// O^T sits in TMEM with d on the lanes; the epilogue writes the same partial
// rows (O/l in fp16, m, l) or output rows as the prefill kernel, so the split
// combine and the Impact pass are shared. The K, V and Q copies, the
// page-table gather and the V_q conversion are the prefill kernel's.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <type_traits>

#include "params.cuh"

namespace rag {
namespace dec {

constexpr int kRows = 16;                          // query rows of a unit
constexpr int kKSt = 3, kVSt = 3;                  // K and V stages
constexpr int kThreads = 256;                      // 4 key warps + K, V, MMA, convert warps
constexpr int kTile = kBN * kHeadDim * 2;          // K or V tile, 16-bit: 32 KB
constexpr int kHalf = kTile / 2;                   // 64 columns of d
constexpr int kQBytes = kRows * kHeadDim * 2;      // Q: two 64-column halves of 16 rows x 128 B
constexpr int kQHalf = kQBytes / 2;
constexpr int kPBytes = kRows * kBN * 2;           // P^T: 16 rows x 128 keys, fp16, two 64-key halves
constexpr int kPHalf = kPBytes / 2;
constexpr int kDescSlots = 4;
constexpr float kRescale = 8.0f;                   // log2 units: rescale O when a row max grows by > 2^8
constexpr uint32_t kColS = 0;                      // S^T buffers: columns [0, 16) and [16, 32)
constexpr uint32_t kColO = 32;                     // O^T: columns [32, 48)
constexpr uint32_t kTmemCols = 64;

struct TileDesc {
  int32_t kind;       // 0: doc tile from the pool, 1: query-key tile
  int32_t kbase;      // query tile: index of its first query key
  int32_t full;
  uint8_t nvalid[kPagesPerTile];
};

struct Ctrl {
  uint64_t q_full, q_empty;
  uint64_t kfull[kKSt], kempty[kKSt];
  uint64_t vfull[kVSt], vempty[kVSt], vconv[kVSt];
  uint64_t s_full[2], p_full[2], pv_done[2], o_full, o_free;
  uint64_t teardown;
  uint64_t desc_full[kDescSlots], desc_empty[kDescSlots];
  TileDesc desc[kDescSlots];
  ChunkCache chunks[2];
  float red[2][4][kRows];   // per-tile row maxima of the four key warps, by tile parity
  float lsum[4][kRows];     // per-item row sums of the four key warps
  uint32_t tmem_base;
  int32_t abort;
  int32_t total_items;
};

constexpr size_t kSmemData = size_t(kQBytes) + 2 * kPBytes + size_t(kKSt) * kTile + size_t(kVSt) * kTile;

struct Item {
  int b, g, split;
  int t_begin, t_end;
  int n_doc_tiles;
  ReqInfo req;
};

// Work items in the prefill kernel's order (request, KV head, split, one row
// block), so that the split combine finds the partial rows where it expects.
__device__ __forceinline__ Item decode_item(const FwdParams& p, const int32_t* prefix, int w) {
  const int B = p.batch.num_requests;
  int lo = 0, hi = B - 1;
  while (lo < hi) {   // last b with prefix[b] <= w
    const int mid = (lo + hi + 1) >> 1;
    if (prefix[mid] <= w) lo = mid; else hi = mid - 1;
  }
  Item it;
  it.b = lo;
  it.req = load_req(p.batch, lo);
  const FwdShape sh = fwd_shape(p.batch, it.req, p.group, p.tiles_per_split);
  int local = w - prefix[lo];
  local /= sh.n_rt;   // one row block
  it.split = local % sh.n_split;
  it.g = local / sh.n_split;
  it.n_doc_tiles = doc_tiles(it.req);
  const int n_tiles = it.n_doc_tiles + query_tiles_upto(it.req.n_q - 1);
  it.t_begin = min(it.split * p.tiles_per_split, n_tiles);
  it.t_end = min(it.t_begin + p.tiles_per_split, n_tiles);
  return it;
}

__device__ __forceinline__ void raise_abort(Ctrl* c, int32_t* err) {
  if (!c->abort) {
    atomicOr(err, kDevErrTimeout);
    c->abort = 1;
  }
}

__device__ __forceinline__ void wait_quiet(uint64_t* bar, uint32_t parity) {
  int zero = 0;
  mbar_wait(bar, parity, &zero);
}

// 32 lanes x 16 columns of 32-bit: thread i of the warp gets lane (base + i).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}

// K-major, 128B-swizzled operand of rows of 128 B stored as two 64-column
// halves `half` bytes apart; k-step kk covers columns [16 kk, 16 kk + 16).
__device__ __forceinline__ uint64_t kmajor(uint32_t base, int kk, uint32_t half) {
  return sdesc_sw128(base + (kk >> 2) * half + (kk & 3) * 32, 16, 1024);
}
// A V tile [128 keys][128 d] (d contiguous, two 64-wide halves 16 KB apart) read
// as the MN-major A operand V^T (M = d): k-step kk covers keys [16 kk, 16 kk + 16).
__device__ __forceinline__ uint64_t vt_desc(uint32_t base, int kk) {
  return sdesc_sw128(base + kk * 16 * 128, kHalf, 1024);
}
// Byte offset of P^T[r][k] in its buffer: K-major rows of 64 keys (128 B) in
// 8-row atoms of 1 KB, the 16-byte chunk index XORed with the row in the atom
// (the 128-byte swizzle the tensor core reads), the two 64-key halves 2 KB apart.
__device__ __forceinline__ uint32_t p_offset(int r, int k) {
  const int half = k >> 6, kk = k & 63, chunk = kk >> 3, e = kk & 7;
  return uint32_t(half * kPHalf + (r >> 3) * 1024 + (r & 7) * 128 + ((chunk ^ (r & 7)) << 4) + (e << 1));
}

// Instruction descriptors: S^T = K Q^T (bf16, M = 128 keys, N = 16 rows, both
// K-major); O^T += V^T P^T (fp16, M = 128 d, N = 16 rows, A MN-major, B K-major).
constexpr uint32_t kIdescQK = idesc_bf16_f32(kBN, kRows, 0);
constexpr uint32_t kIdescPV = (1u << 4) | (1u << 15) | (uint32_t(kRows >> 3) << 17) | (uint32_t(kHeadDim >> 4) << 24);

}  // namespace dec

using namespace dec;

__global__ void __launch_bounds__(dec::kThreads, 1)
decode_attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_kq,
                   const __grid_constant__ CUtensorMap tm_vq, const FwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint8_t* sQ = smem;
  uint8_t* sP = sQ + kQBytes;
  uint8_t* sK = sP + 2 * kPBytes;
  uint8_t* sV = sK + kKSt * kTile;
  Ctrl* ctl = reinterpret_cast<Ctrl*>(sV + kVSt * kTile);
  int32_t* prefix = reinterpret_cast<int32_t*>(ctl + 1);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int B = p.batch.num_requests;
  const int G = p.group;

  pdl_launch_dependents();

  if (tid == 0) {
    mbar_init(&ctl->q_full, 1);
    mbar_init(&ctl->q_empty, 1);
    for (int s = 0; s < kKSt; ++s) { mbar_init(&ctl->kfull[s], 1); mbar_init(&ctl->kempty[s], 1); }
    for (int s = 0; s < kVSt; ++s) {
      mbar_init(&ctl->vfull[s], 1);
      mbar_init(&ctl->vempty[s], 1);
      mbar_init(&ctl->vconv[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&ctl->s_full[b], 1);
      mbar_init(&ctl->p_full[b], 128);
      mbar_init(&ctl->pv_done[b], 1);
    }
    mbar_init(&ctl->o_full, 1);
    mbar_init(&ctl->o_free, 128);
    mbar_init(&ctl->teardown, 1);
    for (int s = 0; s < kDescSlots; ++s) {
      mbar_init(&ctl->desc_full[s], 1);
      mbar_init(&ctl->desc_empty[s], 4);   // one arrival per key warp
    }
    ctl->abort = 0;
    fence_mbar_init();
  }
  if (warp == 6) {
    tmem_alloc(&ctl->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  if (warp == 4 && lane == 0) { tma_prefetch_desc(&tm_q); tma_prefetch_desc(&tm_k); tma_prefetch_desc(&tm_kq); }
  if (warp == 5 && lane == 0) { tma_prefetch_desc(&tm_v); tma_prefetch_desc(&tm_vq); }

  // zero the impact accumulator for the impact pass that follows
  if (p.impact_zero) {
    pdl_wait();
    for (int64_t i = int64_t(blockIdx.x) * blockDim.x + tid; i < p.impact_len; i += int64_t(gridDim.x) * blockDim.x)
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

  if (warp < 4) {
    // ------------------------------------------------------------ key warps: thread = key of the tile
    const int k = tid;
    const uint32_t lane_off = uint32_t(warp * 32) << 16;
    uint32_t t_glob = 0, n_items = 0;
    int bad = 0;
    // One item with the rows padded to R (4, 8 or 16: the item's rows are
    // n_q * G <= 16); returns false when a wait gave up.
    auto run_item = [&](auto Rc, const Item& it, int w, int n) -> bool {
      constexpr int R = decltype(Rc)::value;
      const int rows = it.req.n_q * G;
      float m_ref[R], ls[R];
#pragma unroll
      for (int r = 0; r < R; ++r) { m_ref[r] = -INFINITY; ls[r] = 0.f; }
      for (int i = 0; i < n; ++i) {
        const uint32_t t = t_glob + i;
        const uint32_t slot = t % kDescSlots;
        const int bsel = int(t & 1u);
        if (!mbar_wait(&ctl->desc_full[slot], (t / kDescSlots) & 1, abort_flag)) return false;
        const int kind = ctl->desc[slot].kind;
        const int kbase = ctl->desc[slot].kbase;
        const int nv = ctl->desc[slot].nvalid[k >> 4];
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctl->desc_empty[slot]);
        if (!mbar_wait(&ctl->s_full[bsel], (t >> 1) & 1, abort_flag)) return false;
        tc_fence_after();
        uint32_t u[kRows];
        tmem_ld16(tmem + lane_off + kColS + 16u * bsel, u);
        tmem_wait_ld();
        // the key of this thread: a pool slot (valid while inside its page's
        // tokens) or a query key (valid inside the query block, visible to the
        // rows of its own and later tokens)
        bool kvalid;
        int kq = 0;
        if (kind == 0) {
          kvalid = (k & 15) < nv;
        } else {
          kq = kbase + k;
          kvalid = kq < it.req.n_q;
        }
        float y[R], mt[R];
#pragma unroll
        for (int r = 0; r < R; ++r) {
          const bool vis = kvalid && r < rows && (kind == 0 || kq <= r / G);
          y[r] = vis ? __uint_as_float(u[r]) * p.scale_log2 : -INFINITY;
          mt[r] = y[r];
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
#pragma unroll
          for (int r = 0; r < R; ++r) mt[r] = fmaxf(mt[r], __shfl_xor_sync(0xffffffffu, mt[r], o));
        }
        if (lane == 0) {
#pragma unroll
          for (int r = 0; r < R; ++r) ctl->red[bsel][warp][r] = mt[r];
        }
        named_bar_sync(1, 128);
        float alpha[R];
        bool need = false;
#pragma unroll
        for (int r = 0; r < R; ++r) {
          const float mtile = fmaxf(fmaxf(ctl->red[bsel][0][r], ctl->red[bsel][1][r]),
                                    fmaxf(ctl->red[bsel][2][r], ctl->red[bsel][3][r]));
          alpha[r] = 1.f;
          if (mtile != -INFINITY) {
            if (m_ref[r] == -INFINITY) {
              m_ref[r] = mtile;   // the row's first visible key: O^T holds zeros for it so far
            } else if (mtile > m_ref[r] + kRescale) {
              alpha[r] = ex2(m_ref[r] - mtile);
              m_ref[r] = mtile;
              need = true;
            }
          }
        }
        if (need) {   // the same decision in every key thread (the maxima are shared)
          // O^T must hold PV of the previous tile before it is rescaled
          if (!mbar_wait(&ctl->pv_done[(t - 1) & 1], ((t - 1) >> 1) & 1, abort_flag)) return false;
          tc_fence_after();
          uint32_t ov[kRows];
          tmem_ld16(tmem + lane_off + kColO, ov);
          tmem_wait_ld();
#pragma unroll
          for (int r = 0; r < R; ++r) ov[r] = __float_as_uint(__uint_as_float(ov[r]) * alpha[r]);
          tmem_st16(tmem + lane_off + kColO, ov);
          tmem_wait_st();
#pragma unroll
          for (int r = 0; r < R; ++r) ls[r] *= alpha[r];
        }
        float pr[R];
#pragma unroll
        for (int r = 0; r < R; ++r) {
          pr[r] = (y[r] != -INFINITY) ? ex2(y[r] - m_ref[r]) : 0.f;
          ls[r] += pr[r];
        }
        // this P^T buffer was last read by the PV of tile t - 2; rows past R
        // are left as they are: an output column reads only its own P^T row
        if (t >= 2 && !mbar_wait(&ctl->pv_done[bsel], ((t >> 1) + 1) & 1, abort_flag)) return false;
        uint8_t* pb = sP + bsel * kPBytes;
#pragma unroll
        for (int r = 0; r < R; ++r) *reinterpret_cast<__half*>(pb + p_offset(r, k)) = __float2half_rn(pr[r]);
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&ctl->p_full[bsel]);
      }
      t_glob += n;
      // ---- epilogue: O^T of this item, the row sums over the 128 keys
      if (!mbar_wait(&ctl->o_full, n_items & 1, abort_flag)) return false;
      ++n_items;
      tc_fence_after();
      uint32_t ov[kRows];
      tmem_ld16(tmem + lane_off + kColO, ov);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(&ctl->o_free);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
#pragma unroll
        for (int r = 0; r < R; ++r) ls[r] += __shfl_xor_sync(0xffffffffu, ls[r], o);
      }
      if (lane == 0) {
#pragma unroll
        for (int r = 0; r < R; ++r) ctl->lsum[warp][r] = ls[r];
      }
      named_bar_sync(1, 128);
      pdl_wait();   // outputs and partials may still be read by the previous kernel
      const int d = k;   // this thread's TMEM lane of O^T is column d of the output rows
#pragma unroll
      for (int r = 0; r < R; ++r) {
        if (r >= rows) continue;
        const float l = (ctl->lsum[0][r] + ctl->lsum[1][r]) + (ctl->lsum[2][r] + ctl->lsum[3][r]);
        const float inv = l > 0.f ? 1.f / l : 0.f;
        const float ov_r = __uint_as_float(ov[r]) * inv;
        const int tok = r / G;
        const int head = it.g * G + r % G;
        const float m_use = (m_ref[r] == -INFINITY) ? 0.f : m_ref[r];
        if (p.direct) {
          const int64_t row = int64_t(it.req.q0 + tok) * p.num_q_heads + head;
          p.o[row * kHeadDim + d] = __float2bfloat16_rn(ov_r);
          if (d == r) {
            p.row_m2[row] = m_use;
            p.row_il[row] = l > 0.f ? 1.f / (l * float(p.num_q_heads)) : 0.f;
            if (p.row_lse) p.row_lse[row] = (m_use + __log2f(l)) * 0.69314718055994531f;
          }
        } else {
          float* dst = p.part + (size_t(w) * kFwdRows + r) * kPartStride;
          reinterpret_cast<__half*>(dst)[d] = __float2half_rn(ov_r);
          if (d == r) reinterpret_cast<float4*>(dst + kHeadDim / 2)[0] = make_float4(m_ref[r], l, 0.f, 0.f);
        }
      }
      return true;
    };
    for (int w = blockIdx.x; w < total_items && !bad; w += gridDim.x) {
      const Item it = decode_item(p, prefix, w);
      const int n = it.t_end - it.t_begin;
      if (n == 0) continue;
      const int rows = it.req.n_q * G;   // <= 16 on this path
      const bool ok = rows <= 4   ? run_item(std::integral_constant<int, 4>{}, it, w, n)
                      : rows <= 8 ? run_item(std::integral_constant<int, 8>{}, it, w, n)
                                  : run_item(std::integral_constant<int, 16>{}, it, w, n);
      if (!ok) bad = 1;
    }
    if (bad) raise_abort(ctl, p.err);
  } else if (warp == 4 || warp == 5) {
    // ------------------------------------------------------------ producers
    const bool is_k = (warp == 4);
    const CUtensorMap* tm_pool = is_k ? &tm_k : &tm_v;
    const CUtensorMap* tm_qkv = is_k ? &tm_kq : &tm_vq;
    uint8_t* sbase = is_k ? sK : sV;
    const int nstages = is_k ? kKSt : kVSt;
    uint64_t* full = is_k ? ctl->kfull : ctl->vfull;
    uint64_t* empty = is_k ? ctl->kempty : ctl->vempty;
    uint32_t t_glob = 0, q_iter = 0;
    int bad = 0;
    for (int w = blockIdx.x; w < total_items && !bad; w += gridDim.x) {
      const Item it = decode_item(p, prefix, w);
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
          // the unit's 16 rows: G query heads of the KV head for 16 / G tokens
          mbar_arrive_expect_tx(&ctl->q_full, kQBytes);
          tma_load_3d(sQ, &tm_q, &ctl->q_full, 0, it.g * G, it.req.q0);
          tma_load_3d(sQ + kQHalf, &tm_q, &ctl->q_full, 64, it.g * G, it.req.q0);
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
          TileDesc* dsc = &ctl->desc[slot];
          const unsigned full_pages = __ballot_sync(0xffffffffu, lane < kPagesPerTile && pg.nvalid == kPage);
          if (doc) {
            if (lane < kPagesPerTile) dsc->nvalid[lane] = uint8_t(pg.nvalid);
            if (lane == 0) { dsc->kind = 0; dsc->kbase = 0; dsc->full = (full_pages == 0xffu) ? 1 : 0; }
          } else if (lane == 0) {
            dsc->kind = 1;
            dsc->kbase = (tile - it.n_doc_tiles) * kBN;
            dsc->full = 0;
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(&ctl->desc_full[slot]);
        }
        const int s = t % nstages;
        if (t >= uint32_t(nstages) && !mbar_wait(&empty[s], ((t / nstages) - 1) & 1, abort_flag)) {
          bad = 1;
          break;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive_expect_tx(&full[s], kTile);
        __syncwarp();
        uint8_t* dst = sbase + s * kTile;
        if (doc) {
          if (lane < kPagesPerTile) {
            const int row = pg.page >= 0 ? ((p.layer * p.num_pages + pg.page) * p.num_kv_heads + it.g) * kPage
                                         : -kPage;   // fully out of range: the box is zero-filled
            tma_load_2d(dst + lane * kPage * 128, tm_pool, &full[s], 0, row);
            tma_load_2d(dst + kHalf + lane * kPage * 128, tm_pool, &full[s], 64, row);
          }
        } else if (lane == 0) {
          const int kq0 = it.req.q0 + (tile - it.n_doc_tiles) * kBN;
          tma_load_3d(dst, tm_qkv, &full[s], 0, it.g, kq0);
          tma_load_3d(dst + kHalf, tm_qkv, &full[s], 64, it.g, kq0);
        }
      }
      t_glob += n;
    }
    if (bad) raise_abort(ctl, p.err);
    if (lane == 0 && ctl->abort) {
      const uint32_t first = t_glob > uint32_t(nstages) ? t_glob - nstages : 0;
      for (uint32_t t = first; t < t_glob; ++t) wait_quiet(&full[t % nstages], (t / nstages) & 1);
      if (is_k && q_iter > 0) wait_quiet(&ctl->q_full, (q_iter - 1) & 1);
    }
    __syncwarp();
  } else if (warp == 7) {
    // ------------------------------------------------------------ convert warp
    // The query block's own V_q tile (a bf16 input) rounded to fp16 in place,
    // rows past the query block zeroed; doc V tiles are fp16 in the pool.
    uint32_t t_glob = 0;
    int bad = 0;
    uint32_t range = 0;
    for (int w = blockIdx.x; w < total_items && !bad; w += gridDim.x) {
      const Item it = decode_item(p, prefix, w);
      const int n = it.t_end - it.t_begin;
      for (int i = 0; i < n; ++i) {
        const uint32_t t = t_glob + i;
        const int tile = it.t_begin + i;
        const int s = t % kVSt;
        if (!mbar_wait(&ctl->vfull[s], (t / kVSt) & 1, abort_flag)) { bad = 1; break; }
        if (tile >= it.n_doc_tiles) {
          const int rows = min(kBN, it.req.n_q - (tile - it.n_doc_tiles) * kBN);
          uint8_t* base = sV + s * kTile;
#pragma unroll 4
          for (int u = lane; u < kBN * (kHeadDim / 8); u += 32) {
            const int r = u >> 4, c = u & 15;   // row, 16-byte chunk of the row
            uint4* at = reinterpret_cast<uint4*>(base + (c >> 3) * kHalf + r * 128 + ((c & 7) << 4));
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
    // ------------------------------------------------------------ MMA issuer (warp 6)
    if (lane == 0) {
      const uint32_t q_base = smem_u32(sQ);
      uint32_t t_glob = 0, q_iter = 0, n_items = 0;
      int bad = 0;
      for (int w = blockIdx.x; w < total_items && !bad; w += gridDim.x) {
        const Item it = decode_item(p, prefix, w);
        const int n = it.t_end - it.t_begin;
        if (n == 0) continue;
        if (!mbar_wait(&ctl->q_full, q_iter & 1, abort_flag)) { bad = 1; break; }
        tc_fence_after();
        // S^T of tile j of the item into buffer (tile parity)
        auto qk = [&](int j) {
          const uint32_t t = t_glob + j;
          const int s = t % kKSt;
          if (!mbar_wait(&ctl->kfull[s], (t / kKSt) & 1, abort_flag)) return false;
          tc_fence_after();
          const uint32_t k_base = smem_u32(sK + s * kTile);
#pragma unroll
          for (int kk = 0; kk < kHeadDim / 16; ++kk)
            mma_ss(tmem + kColS + 16u * (t & 1u), kmajor(k_base, kk, kHalf), kmajor(q_base, kk, kQHalf), kIdescQK,
                   kk > 0);
          tc_commit(&ctl->s_full[t & 1]);
          tc_commit(&ctl->kempty[s]);
          if (j == n - 1) tc_commit(&ctl->q_empty);   // the rest of the item reads no Q
          return true;
        };
        for (int j = 0; j < n && j < 2 && !bad; ++j)
          if (!qk(j)) bad = 1;
        for (int i = 0; i < n && !bad; ++i) {
          const uint32_t t = t_glob + i;
          const int sv = t % kVSt;
          const int bsel = int(t & 1u);
          const bool v_doc = it.t_begin + i < it.n_doc_tiles;
          if (!mbar_wait(v_doc ? &ctl->vfull[sv] : &ctl->vconv[sv], (t / kVSt) & 1, abort_flag)) { bad = 1; break; }
          if (i == 0 && n_items > 0 && !mbar_wait(&ctl->o_free, (n_items - 1) & 1, abort_flag)) { bad = 1; break; }
          if (!mbar_wait(&ctl->p_full[bsel], (t >> 1) & 1, abort_flag)) { bad = 1; break; }
          tc_fence_after();
          const uint32_t v_base = smem_u32(sV + sv * kTile);
          const uint32_t p_base = smem_u32(sP + bsel * kPBytes);
#pragma unroll
          for (int kk = 0; kk < kBN / 16; ++kk)
            mma_ss(tmem + kColO, vt_desc(v_base, kk), kmajor(p_base, kk, kPHalf), kIdescPV, (i > 0) || (kk > 0));
          tc_commit(&ctl->pv_done[bsel]);
          tc_commit(&ctl->vempty[sv]);
          if (i == n - 1) tc_commit(&ctl->o_full);
          if (i + 2 < n && !qk(i + 2)) { bad = 1; break; }
        }
        if (bad) break;
        t_glob += n;
        ++q_iter;
        ++n_items;
      }
      if (bad) raise_abort(ctl, p.err);
      tc_commit(&ctl->teardown);
      wait_quiet(&ctl->teardown, 0);
    }
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 6) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

__host__ size_t decode_smem_bytes(int num_requests) {
  return 1024 + dec::kSmemData + sizeof(dec::Ctrl) + sizeof(int32_t) * (num_requests + 1) + 64;
}

cudaError_t launch_decode_attn(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                               const CUtensorMap& tkq, const CUtensorMap& tvq, const FwdParams& p, int grid,
                               cudaStream_t stream) {
  const size_t smem = decode_smem_bytes(p.batch.num_requests);
  static SmemAttr attr;
  cudaError_t e = ensure_smem_attr(decode_attn_kernel, attr, smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(decode_attn_kernel, dim3(grid), dim3(dec::kThreads), smem, stream, 1, tq, tk, tv, tkq, tvq, p);
}

}  // namespace rag
