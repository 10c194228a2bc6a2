// Shared device-side definitions: batch geometry, work decomposition and the
// workspace layout used by the attention, combine, impact and top-k kernels.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "ptx.cuh"

namespace rag {

constexpr int kPage = 16;             // tokens per pool page
constexpr int kHeadDim = 128;         // head_dim of the tensor-core path
constexpr int kBM = 128;              // attention rows (query token x head-in-group) per Q tile
constexpr int kQTiles = 2;            // Q tiles per attention work item
constexpr int kFwdRows = kBM * kQTiles;
constexpr int kBN = 128;              // keys per tile
constexpr int kPagesPerTile = kBN / kPage;
constexpr int kImpactRows = 256;      // rows per impact-pass block (MMA N)
constexpr int kMaxRequests = 4096;
constexpr int kPartStride = 68;       // 32-bit words per partial row: O/l as 64 fp16 pairs, m, l, pad

// device error word bits (rag_last_device_error reports them)
enum : int32_t {
  kDevErrPage = 1,       // a page id outside [0, num_pages)
  kDevErrGeometry = 2,   // a chunk whose page count is not ceil(len / 16)
  kDevErrTimeout = 4,    // a pipeline wait gave up
  kDevErrRange = 8,      // a V value beyond the fp16 range was saturated when stored as fp16
};

struct BatchDev {
  const int32_t* req_chunk_off;    // [B+1]
  const int32_t* chunk_doc_off;    // [C+1]
  const int32_t* chunk_page_off;   // [C+1]
  const int32_t* page_ids;         // [num_page_refs]
  const int32_t* q_off;            // [B+1]
  int32_t num_requests;
  // host-side totals and maxima; a request that breaks them is skipped and
  // reported (kDevErrGeometry) so that no kernel reads or writes out of range
  int32_t num_chunks, num_page_refs, total_q, total_doc, max_q, max_pages, max_doc;
};

struct ReqInfo {
  int32_t c0, c1;       // chunk-list entries of the request
  int32_t doc0, n_doc;  // first doc token (over the batch) and doc tokens
  int32_t p0, n_pages;  // first page reference and pages
  int32_t q0, n_q;      // first query token and query tokens
};

__device__ __forceinline__ ReqInfo load_req(const BatchDev& B, int b) {
  ReqInfo r;
  r.c0 = __ldg(B.req_chunk_off + b);
  r.c1 = __ldg(B.req_chunk_off + b + 1);
  r.doc0 = __ldg(B.chunk_doc_off + r.c0);
  r.n_doc = __ldg(B.chunk_doc_off + r.c1) - r.doc0;
  r.p0 = __ldg(B.chunk_page_off + r.c0);
  r.n_pages = __ldg(B.chunk_page_off + r.c1) - r.p0;
  r.q0 = __ldg(B.q_off + b);
  r.n_q = __ldg(B.q_off + b + 1) - r.q0;
  return r;
}

// A request whose descriptor entries stay inside the host-declared sizes.
__device__ __forceinline__ bool req_ok(const BatchDev& B, const ReqInfo& r) {
  return r.c0 >= 0 && r.c0 <= r.c1 && r.c1 <= B.num_chunks && r.p0 >= 0 && r.n_pages >= 0 &&
         r.p0 + r.n_pages <= B.num_page_refs && r.n_pages <= B.max_pages && r.q0 >= 0 && r.n_q >= 0 &&
         r.q0 + r.n_q <= B.total_q && r.n_q <= B.max_q && r.doc0 >= 0 && r.n_doc >= 0 &&
         r.doc0 + r.n_doc <= B.total_doc && r.n_doc <= B.max_doc && r.n_doc <= r.n_pages * kPage;
}

__host__ __device__ __forceinline__ int ceil_div(int a, int b) { return (a + b - 1) / b; }

// Tiles of one request: ceil(pages / 8) doc tiles in page-list order, then
// the query block's keys in tiles of 128.
__device__ __forceinline__ int doc_tiles(const ReqInfo& r) { return ceil_div(r.n_pages, kPagesPerTile); }

// Attention work units: (request, kv head, 256-row block, split of the key tiles).
struct FwdShape {
  int n_rt, n_split;
};
__device__ __forceinline__ FwdShape fwd_shape(const BatchDev& B, const ReqInfo& r, int G, int tiles_per_split) {
  FwdShape s;
  if (r.n_q <= 0 || !req_ok(B, r)) { s.n_rt = 0; s.n_split = 0; return s; }
  s.n_rt = ceil_div(r.n_q * G, kFwdRows);
  s.n_split = ceil_div(doc_tiles(r) + ceil_div(r.n_q, kBN), tiles_per_split);
  return s;
}

// Query-key tiles that a block of rows ending at token `last_tok` can see.
__device__ __forceinline__ int query_tiles_upto(int last_tok) { return last_tok / kBN + 1; }

// Impact work units: (request, kv head, 256-row block, split of key tiles).
__device__ __forceinline__ FwdShape impact_shape(const BatchDev& B, const ReqInfo& r, int G,
                                                int tiles_per_split) {
  FwdShape s;
  if (r.n_q <= 0 || !req_ok(B, r)) { s.n_rt = 0; s.n_split = 0; return s; }
  s.n_rt = ceil_div(r.n_q * G, kImpactRows);
  s.n_split = ceil_div(doc_tiles(r) + ceil_div(r.n_q, kBN), tiles_per_split);
  return s;
}

// Locate the chunk of global page reference `gref` inside chunk-list range
// [c0, c1): the last c with chunk_page_off[c] <= gref.
__device__ __forceinline__ int chunk_of_page(const BatchDev& B, int c0, int c1, int gref) {
  int lo = c0, hi = c1 - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (__ldg(B.chunk_page_off + mid) <= gref) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// One page of a doc tile: where it lives and which of its slots are real.
struct PageRef {
  int32_t page;     // physical page, or -1 when absent/invalid
  int32_t nvalid;   // valid slots (0..16)
  int32_t lstart;   // logical doc position of slot 0 within the request
  int32_t chunk;    // chunk-list entry the page belongs to (-1 when absent)
};

__device__ __forceinline__ PageRef page_ref(const BatchDev& B, const ReqInfo& r, int ref, int num_pages,
                                            int32_t* err) {
  PageRef p;
  p.page = -1; p.nvalid = 0; p.lstart = 0; p.chunk = -1;
  if (ref >= r.n_pages) return p;
  const int gref = r.p0 + ref;
  const int c = chunk_of_page(B, r.c0, r.c1, gref);
  const int cp0 = __ldg(B.chunk_page_off + c), cp1 = __ldg(B.chunk_page_off + c + 1);
  const int k = gref - cp0;
  const int cstart = __ldg(B.chunk_doc_off + c);
  const int len = __ldg(B.chunk_doc_off + c + 1) - cstart;
  if (k < 0 || gref >= cp1 || len < 0 || cstart < r.doc0 || cstart + len > r.doc0 + r.n_doc) {
    if (err) atomicOr(err, kDevErrGeometry);
    return p;
  }
  int nv = len - k * kPage;
  if (nv <= 0 || (gref == cp1 - 1 && nv > kPage)) {
    if (err) atomicOr(err, kDevErrGeometry);
  }
  nv = nv < 0 ? 0 : (nv > kPage ? kPage : nv);
  const int page = __ldg(B.page_ids + gref);
  if (page < 0 || page >= num_pages) {
    if (err) atomicOr(err, kDevErrPage);
    return p;
  }
  p.page = page;
  p.nvalid = nv;
  p.lstart = cstart - r.doc0 + k * kPage;
  p.chunk = c;
  return p;
}

// A request's chunk table staged in shared memory by a producer warp, so that
// resolving the 8 pages of a tile costs one global load (the page ids, one
// tile ahead) instead of a chain of dependent loads.
constexpr int kChunkCache = 64;
struct ChunkCache {
  int32_t n;                            // chunks cached; -1: too many, use global memory
  int32_t page_off[kChunkCache + 1];    // chunk_page_off[c0 ..= c1]
  int32_t doc_off[kChunkCache + 1];     // chunk_doc_off[c0 ..= c1]
};

__device__ __forceinline__ void load_chunk_cache(ChunkCache* cc, const BatchDev& B, const ReqInfo& r, int lane) {
  const int nc = r.c1 - r.c0;
  if (nc <= kChunkCache) {
    for (int i = lane; i <= nc; i += 32) {
      cc->page_off[i] = __ldg(B.chunk_page_off + r.c0 + i);
      cc->doc_off[i] = __ldg(B.chunk_doc_off + r.c0 + i);
    }
  }
  if (lane == 0) cc->n = nc <= kChunkCache ? nc : -1;
  __syncwarp();
}

// Physical page id of page `ref` of the request (or -1 past its pages).
__device__ __forceinline__ int32_t load_page_id(const BatchDev& B, const ReqInfo& r, int ref) {
  return ref < r.n_pages ? __ldg(B.page_ids + r.p0 + ref) : -1;
}

// page_ref with the chunk table from the cache and a page id loaded earlier.
__device__ __forceinline__ PageRef page_ref_cached(const ChunkCache* cc, const BatchDev& B, const ReqInfo& r,
                                                   int ref, int32_t page, int num_pages, int32_t* err) {
  if (cc->n < 0) return page_ref(B, r, ref, num_pages, err);
  PageRef p;
  p.page = -1; p.nvalid = 0; p.lstart = 0; p.chunk = -1;
  if (ref >= r.n_pages) return p;
  const int gref = r.p0 + ref;
  int lo = 0, hi = cc->n - 1;   // last local chunk with page_off <= gref
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (cc->page_off[mid] <= gref) lo = mid; else hi = mid - 1;
  }
  const int cp0 = cc->page_off[lo], cp1 = cc->page_off[lo + 1];
  const int k = gref - cp0;
  const int cstart = cc->doc_off[lo];
  const int len = cc->doc_off[lo + 1] - cstart;
  if (k < 0 || gref >= cp1 || len < 0 || cstart < r.doc0 || cstart + len > r.doc0 + r.n_doc) {
    if (err) atomicOr(err, kDevErrGeometry);
    return p;
  }
  int nv = len - k * kPage;
  if (nv <= 0 || (gref == cp1 - 1 && nv > kPage)) {
    if (err) atomicOr(err, kDevErrGeometry);
  }
  nv = nv < 0 ? 0 : (nv > kPage ? kPage : nv);
  if (page < 0 || page >= num_pages) {
    if (err) atomicOr(err, kDevErrPage);
    return p;
  }
  p.page = page;
  p.nvalid = nv;
  p.lstart = cstart - r.doc0 + k * kPage;
  p.chunk = r.c0 + lo;
  return p;
}

// RoPE re-basing of one K tile in shared memory (TurboRAG page,
// "Implementation": position ids of precompute and inference must agree).
// The tile is 128 keys x 128 channels of bf16, stored as two 64-channel
// halves (16 KB apart), each 128B-swizzled: the 16-byte column c of row r
// sits at r * 128 + ((c ^ (r & 7)) * 16) in both halves, so one 16-byte load
// from each half holds the 8 rotary pairs (i, i + 64), i = 8c .. 8c + 7.
// Key r belongs to page r / 16 of the tile, whose chunk-list entry is
// kchunk[r / 16] (-1: not a cached key, left alone); pair i of entry e turns
// by the angle in table[e * 64 + i] = (cos, sin). Each pair is rotated in
// fp32 and rounded once to bf16. One warp, every lane on one column c.
__device__ __forceinline__ void rope_rotate_tile(uint8_t* tile, const int32_t* kchunk, const float2* table,
                                                 int lane) {
  const int c = lane & 7;
  int cur = -1;
  float2 cs[8];
#pragma unroll 1
  for (int r = lane >> 3; r < 128; r += 4) {
    const int e = kchunk[r >> 4];
    if (e < 0) continue;
    if (e != cur) {
      const float4* t4 = reinterpret_cast<const float4*>(table + int64_t(e) * 64 + c * 8);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float4 v = __ldg(t4 + j);
        cs[2 * j] = make_float2(v.x, v.y);
        cs[2 * j + 1] = make_float2(v.z, v.w);
      }
      cur = e;
    }
    uint4* p0 = reinterpret_cast<uint4*>(tile + r * 128 + ((c ^ (r & 7)) << 4));
    uint4* p1 = reinterpret_cast<uint4*>(reinterpret_cast<uint8_t*>(p0) + 16384);
    uint4 a = *p0, b = *p1;
    uint32_t* aw = reinterpret_cast<uint32_t*>(&a);
    uint32_t* bw = reinterpret_cast<uint32_t*>(&b);
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const float x0 = __uint_as_float(aw[w] << 16), x1 = __uint_as_float(aw[w] & 0xffff0000u);
      const float y0 = __uint_as_float(bw[w] << 16), y1 = __uint_as_float(bw[w] & 0xffff0000u);
      const float2 c0 = cs[2 * w], c1 = cs[2 * w + 1];
      const float nx0 = fmaf(x0, c0.x, -(y0 * c0.y)), ny0 = fmaf(y0, c0.x, x0 * c0.y);
      const float nx1 = fmaf(x1, c1.x, -(y1 * c1.y)), ny1 = fmaf(y1, c1.x, x1 * c1.y);
      aw[w] = pack_bf16x2(nx0, nx1);
      bw[w] = pack_bf16x2(ny0, ny1);
    }
    *p0 = a;
    *p1 = b;
  }
}

// Workspace layout (bytes, each region 256-aligned):
//   [0, 256)                   error word and flags
//   item prefix                (kMaxRequests + 1) int32
//   row_m2                     total_q * H_q fp32   (reference max, log2 units)
//   row_il                     total_q * H_q fp32   (1 / (l * H_q))
//   partials                   items * 256 * kPartStride 32-bit words
//   RoPE table                 num_chunks * 64 (cos, sin) fp32 pairs
struct WsLayout {
  size_t off_prefix, off_m2, off_il, off_part, off_rope, total;
};

__host__ __device__ inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

__host__ __device__ inline WsLayout ws_layout(int64_t total_q, int num_q_heads, int64_t max_items,
                                              int64_t num_chunks) {
  WsLayout w;
  size_t at = 256;
  w.off_prefix = at; at = align256(at + sizeof(int32_t) * (kMaxRequests + 1));
  w.off_m2 = at; at = align256(at + sizeof(float) * size_t(total_q) * num_q_heads);
  w.off_il = at; at = align256(at + sizeof(float) * size_t(total_q) * num_q_heads);
  w.off_part = at; at = align256(at + sizeof(float) * size_t(max_items) * kFwdRows * kPartStride);
  w.off_rope = at; at = align256(at + sizeof(float) * 2 * 64 * size_t(num_chunks));
  w.total = at;
  return w;
}

}  // namespace rag
