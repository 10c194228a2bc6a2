// Host side of the C ABI: argument validation, TMA tensor maps, work
// planning (split-KV sizing against the SM count), launches, device-error
// readback and optional per-kernel event timing.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstring>
#include <mutex>
#include <unordered_map>
#include <vector>

#include "rag_prefill.h"
#include "params.cuh"

namespace rag {

constexpr int kSimtMaxKeysHost = 8192;
constexpr int kTopkMaxKHost = 16384;
constexpr int kRcMinDModel = 64;

// ------------------------------------------------------------ profiling

enum Kind { kKindPoolWrite = 0, kKindAttn, kKindCombine, kKindImpact, kKindTopk, kKindSimtAttn, kKindSimtImpact,
            kKindRcPlan, kKindRcCopy, kKindRcGemm, kKindRope, kKindKvDecode, kKindDecAttn, kNumKinds };

struct ProfRecord {
  int kind;
  cudaEvent_t start, stop;
};

static std::atomic<int64_t> g_launches{0};
static std::atomic<int> g_last_cuda_error{0};

void note_cuda_error(cudaError_t e) {
  if (e != cudaSuccess) g_last_cuda_error.store(int(e));
}
static std::atomic<int> g_prof_on{0};
static std::mutex g_prof_mu;
static std::vector<ProfRecord> g_prof;
static std::vector<cudaEvent_t> g_event_pool;

static cudaEvent_t take_event() {
  if (!g_event_pool.empty()) {
    cudaEvent_t e = g_event_pool.back();
    g_event_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}

// Inside a stream capture the events become external event-record nodes of
// the graph, which stay readable with cudaEventElapsedTime after each replay.
static void record_event(cudaEvent_t ev, cudaStream_t stream) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(stream, &cs) == cudaSuccess && cs == cudaStreamCaptureStatusActive)
    cudaEventRecordWithFlags(ev, stream, cudaEventRecordExternal);
  else
    cudaEventRecord(ev, stream);
}

struct LaunchScope {
  int kind;
  cudaStream_t stream;
  cudaEvent_t start = nullptr, stop = nullptr;
  LaunchScope(int k, cudaStream_t s) : kind(k), stream(s) {
    if (g_prof_on.load()) {
      std::lock_guard<std::mutex> lk(g_prof_mu);
      start = take_event();
      stop = take_event();
      record_event(start, stream);
    }
  }
  void done(cudaError_t e) {
    if (e == cudaSuccess) g_launches.fetch_add(1);
    else note_cuda_error(e);
    if (start) {
      record_event(stop, stream);
      std::lock_guard<std::mutex> lk(g_prof_mu);
      g_prof.push_back({kind, start, stop});
    }
  }
};

// ------------------------------------------------------------ tensor maps

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// Encoded maps are kept per host thread (no lock), keyed by everything the
// encoding reads, so that a call whose tensors were seen before (the layers
// of a step, the steps of a serving loop) skips the driver call. A map holds
// only the address and the geometry, so a key match is an exact reuse.
struct MapKey {
  const void* base;
  int rank;
  uint64_t dims[3];
  uint64_t strides[2];
  uint32_t box[3];
  bool operator==(const MapKey& o) const { return std::memcmp(this, &o, sizeof(MapKey)) == 0; }
};
struct MapKeyHash {
  size_t operator()(const MapKey& k) const {
    const unsigned char* b = reinterpret_cast<const unsigned char*>(&k);
    uint64_t h = 1469598103934665603ull;   // FNV-1a over the key's bytes
    for (size_t i = 0; i < sizeof(MapKey); ++i) h = (h ^ b[i]) * 1099511628211ull;
    return size_t(h);
  }
};
constexpr size_t kMapCacheMax = 4096;   // entries kept per host thread before the cache starts over

// bf16 tensor with rank (<= 3) dims (innermost first), 128B swizzle, zero fill
static bool make_map(CUtensorMap* m, const void* base, int rank, const uint64_t* dims, const uint64_t* strides_bytes,
                     const uint32_t* box) {
  MapKey k;
  std::memset(&k, 0, sizeof(k));   // padding too: keys compare as bytes
  k.base = base;
  k.rank = rank;
  for (int i = 0; i < rank; ++i) {
    k.dims[i] = dims[i];
    k.box[i] = box[i];
    if (i + 1 < rank) k.strides[i] = strides_bytes[i];
  }
  thread_local std::unordered_map<MapKey, CUtensorMap, MapKeyHash> cache;
  const auto hit = cache.find(k);
  if (hit != cache.end()) {
    *m = hit->second;
    return true;
  }
  auto fn = encode_fn();
  if (!fn) return false;
  uint32_t elem_strides[5] = {1, 1, 1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), dims, strides_bytes, box,
                  elem_strides, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return false;
  if (cache.size() >= kMapCacheMax) cache.clear();
  cache.emplace(k, *m);
  return true;
}

// ------------------------------------------------------------ helpers

static int num_sms() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) dev = 0;
  thread_local int known[kMaxDevices] = {};   // per device, read once per host thread
  if (known[dev] <= 0) {
    int n = 148;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    known[dev] = n;
  }
  return known[dev];
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static int cdiv(int64_t a, int64_t b) { return int((a + b - 1) / b); }

struct Plan {
  int tiles_per_split = 1;
  int direct = 0;
  int grid = 1;
  int64_t max_items = 0;
  int max_units_rt = 0;   // row tiles (or blocks) of the largest request
};

// Split the key tiles of every (request, kv head, row block) unit so that
// the work fills the SMs in whole waves. rows_per_unit: 128 (attention) or
// 256 (impact).
enum class PlanFor { kAttention, kImpact };
static Plan plan_split_uncached(const rag_batch& b, int num_kv_heads, int group, int rows_per_unit, int sms,
                                PlanFor what);

// plan_split reads only these batch totals and the shape, so its result is
// kept per host thread for the last few distinct inputs (every layer of a
// step, every step of a batch reuses one).
static Plan plan_split(const rag_batch& b, int num_kv_heads, int group, int rows_per_unit, int sms, PlanFor what) {
  struct Key {
    int32_t v[10];
  };
  constexpr int kPlanCache = 8;
  thread_local Key keys[kPlanCache];
  thread_local Plan plans[kPlanCache];
  thread_local int n = 0, next = 0;
  Key k = {{b.num_requests, b.max_pages, b.max_q, b.total_q, b.num_page_refs, num_kv_heads, group, rows_per_unit,
            sms, int32_t(what)}};
  for (int i = 0; i < n; ++i)
    if (std::memcmp(&keys[i], &k, sizeof(Key)) == 0) return plans[i];
  const Plan pl = plan_split_uncached(b, num_kv_heads, group, rows_per_unit, sms, what);
  const int slot = n < kPlanCache ? n++ : (next++ % kPlanCache);
  keys[slot] = k;
  plans[slot] = pl;
  return pl;
}

static Plan plan_split_uncached(const rag_batch& b, int num_kv_heads, int group, int rows_per_unit, int sms,
                                PlanFor what) {
  Plan pl;
  const int B = std::max(1, b.num_requests);
  const int tiles_max = cdiv(b.max_pages, kPagesPerTile) + cdiv(b.max_q, kBN);
  const double avg_q = double(b.total_q) / B;
  const double avg_pages = double(b.num_page_refs) / B;
  const int rt_avg = std::max(1, cdiv(int64_t(std::ceil(avg_q * group)), rows_per_unit));
  const int tiles_avg = std::max(1, cdiv(int64_t(std::ceil(avg_pages)), kPagesPerTile) +
                                        cdiv(int64_t(std::ceil(avg_q)), kBN));
  const double units = double(num_kv_heads) * B * rt_avg;
  // Every split length from 2 tiles to the whole row, with a fixed cost per
  // item (Q load, pipeline fill and the partial-row epilogue, about two
  // tiles' worth by measurement). One request: its items are alike, and the busiest SM runs
  // ceil(items / sms) of them. Several requests: items differ in length and
  // are dealt out round-robin, so the estimate is the list-scheduling bound,
  // the average load per SM plus one longest item.
  // Measured: 2 beats 3 by 5.5 % on 16 batched requests, equal elsewhere; an
  // attention unit of one Q tile (at most 128 rows: decode steps, one query
  // head per KV head) runs its tiles faster (two S buffers, one softmax
  // warpgroup), so its fixed cost is more tiles' worth: 4 beats 2 by 15 % on
  // the 16-request decode step, and 3 (7 % slower) and 8 (30 % slower) there.
  const bool one_q_tile = what == PlanFor::kAttention && avg_q * group <= kBM;
  const double kItemOverheadTiles = one_q_tile ? 4.0 : 2.0;
  const double total_tiles = units * tiles_avg;
  double best = 1e300;
  int best_ts = std::max(tiles_max, 1);
  for (int ts = std::min(2, std::max(tiles_max, 1)); ts <= std::max(tiles_max, 1); ++ts) {
    const double items = units * std::ceil(double(tiles_avg) / ts);
    const double cost = B == 1 ? std::ceil(items / sms) * (ts + kItemOverheadTiles)
                               : (total_tiles + items * kItemOverheadTiles) / sms + ts + kItemOverheadTiles;
    if (cost < best + 1e-9) {   // ties go to the longer split (fewer partial rows)
      best = cost;
      best_ts = ts;
    }
  }
  pl.tiles_per_split = std::max(1, best_ts);
  pl.direct = pl.tiles_per_split >= tiles_max ? 1 : 0;
  const int64_t rt_sum_bound = cdiv(int64_t(b.total_q) * group, rows_per_unit) + b.num_requests;
  pl.max_items = int64_t(num_kv_heads) * rt_sum_bound * std::max(1, cdiv(tiles_max, pl.tiles_per_split));
  pl.grid = int(std::max<int64_t>(1, std::min<int64_t>(sms, pl.max_items)));
  pl.max_units_rt = std::max(1, cdiv(int64_t(b.max_q) * group, rows_per_unit));
  return pl;
}

static rag_status check_pool(const rag_kv_pool* pool) {
  if (!pool || !pool->k || !pool->v) return RAG_ERR_INVALID_ARG;
  if (!aligned16(pool->k) || !aligned16(pool->v)) return RAG_ERR_INVALID_ARG;
  if (pool->page_size != kPage) return RAG_ERR_UNSUPPORTED;
  if (pool->num_layers <= 0 || pool->num_pages <= 0 || pool->num_kv_heads <= 0) return RAG_ERR_SHAPE;
  if (pool->dtype == RAG_BF16) {
    if (pool->head_dim != kHeadDim) return RAG_ERR_UNSUPPORTED;
  } else if (pool->dtype == RAG_F32) {
    if (pool->head_dim != 64 && pool->head_dim != 128) return RAG_ERR_UNSUPPORTED;
  } else {
    return RAG_ERR_UNSUPPORTED;
  }
  const int64_t rows = int64_t(pool->num_layers) * pool->num_pages * pool->num_kv_heads * kPage;
  if (rows >= (int64_t(1) << 31)) return RAG_ERR_UNSUPPORTED;
  return RAG_OK;
}

static rag_status check_batch(const rag_batch* b) {
  if (!b) return RAG_ERR_INVALID_ARG;
  if (b->num_requests < 0 || b->num_requests > kMaxRequests) return RAG_ERR_UNSUPPORTED;
  if (b->num_chunks < 0 || b->num_page_refs < 0 || b->total_q < 0 || b->total_doc < 0 || b->max_q < 0 ||
      b->max_doc < 0 || b->max_pages < 0)
    return RAG_ERR_SHAPE;
  if (b->num_requests > 0 &&
      (!b->req_chunk_off || !b->chunk_doc_off || !b->chunk_page_off || !b->q_off ||
       (b->num_page_refs > 0 && !b->page_ids)))
    return RAG_ERR_INVALID_ARG;
  if (b->max_q > b->total_q || b->max_doc > b->total_doc || b->max_pages > b->num_page_refs) return RAG_ERR_SHAPE;
  if (int64_t(b->max_pages) * kPage < b->max_doc) return RAG_ERR_SHAPE;
  return RAG_OK;
}

static BatchDev to_dev(const rag_batch& b) {
  BatchDev d;
  d.req_chunk_off = b.req_chunk_off;
  d.chunk_doc_off = b.chunk_doc_off;
  d.chunk_page_off = b.chunk_page_off;
  d.page_ids = b.page_ids;
  d.q_off = b.q_off;
  d.num_requests = b.num_requests;
  d.num_chunks = b.num_chunks;
  d.num_page_refs = b.num_page_refs;
  d.total_q = b.total_q;
  d.total_doc = b.total_doc;
  d.max_q = b.max_q;
  d.max_pages = b.max_pages;
  d.max_doc = b.max_doc;
  return d;
}

static size_t workspace_bytes_for(const rag_kv_pool& pool, const rag_batch& b, int num_q_heads) {
  const int G = num_q_heads / pool.num_kv_heads;
  const Plan pf = plan_split(b, pool.num_kv_heads, G, kFwdRows, num_sms(), PlanFor::kAttention);
  const bool bf16 = pool.dtype == RAG_BF16;
  return ws_layout(b.total_q, num_q_heads, bf16 ? pf.max_items : 0, bf16 ? b.num_chunks : 0).total;
}

}  // namespace rag

using namespace rag;

extern "C" {

int32_t rag_abi_version(void) { return RAG_ABI_VERSION; }

const char* rag_status_string(int32_t s) {
  switch (s) {
    case RAG_OK: return "ok";
    case RAG_ERR_INVALID_ARG: return "invalid argument";
    case RAG_ERR_SHAPE: return "inconsistent shape";
    case RAG_ERR_PAGE_OOB: return "page id outside the pool";
    case RAG_ERR_UNSUPPORTED: return "unsupported configuration";
    case RAG_ERR_CUDA: return "CUDA runtime error";
    case RAG_ERR_TIMEOUT: return "device pipeline wait timed out";
    case RAG_ERR_WORKSPACE: return "workspace missing or too small";
    case RAG_ERR_GEOMETRY: return "chunk page count does not match its length";
    case RAG_ERR_RANGE: return "a V value beyond the fp16 range was saturated";
    case RAG_ERR_NO_FREE_PAGES: return "too few free pages for the copy-on-write recompute";
    default: return "unknown status";
  }
}

int32_t rag_num_sms(void) { return num_sms(); }

int32_t rag_recompute_count(int32_t n_doc, double r) {
  if (n_doc <= 0) return 0;
  const int k = int(double(n_doc) * r);
  return k < 1 ? 1 : k;
}

rag_status rag_kv_pool_write(const rag_kv_pool* pool, int32_t layer, const int32_t* page_ids, int32_t n_pages,
                             int32_t n_tokens, const void* k, const void* v, int32_t* device_err, void* stream) {
  rag_status st = check_pool(pool);
  if (st != RAG_OK) return st;
  if (layer < 0 || layer >= pool->num_layers) return RAG_ERR_INVALID_ARG;
  if (n_tokens < 0 || n_pages != (n_tokens + kPage - 1) / kPage) return RAG_ERR_SHAPE;
  if (n_tokens == 0) return RAG_OK;
  if (!page_ids || !k || !v || !aligned16(k) || !aligned16(v)) return RAG_ERR_INVALID_ARG;
  PoolWriteParams p;
  p.pool_k = static_cast<uint8_t*>(pool->k);
  p.pool_v = static_cast<uint8_t*>(pool->v);
  p.k = static_cast<const uint8_t*>(k);
  p.v = static_cast<const uint8_t*>(v);
  p.page_ids = page_ids;
  p.err = device_err;
  p.layer = layer;
  p.num_pages = pool->num_pages;
  p.num_kv_heads = pool->num_kv_heads;
  p.n_tokens = n_tokens;
  p.row_bytes = pool->head_dim * (pool->dtype == RAG_BF16 ? 2 : 4);
  p.v_to_f16 = pool->dtype == RAG_BF16 ? 1 : 0;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  LaunchScope ls(kKindPoolWrite, s);
  cudaError_t e = launch_pool_write(p, n_pages, s);
  ls.done(e);
  return e == cudaSuccess ? RAG_OK : RAG_ERR_CUDA;
}

size_t rag_workspace_size(const rag_kv_pool* pool, const rag_batch* batch, int32_t num_q_heads) {
  if (check_pool(pool) != RAG_OK || check_batch(batch) != RAG_OK) return 0;
  if (num_q_heads <= 0 || num_q_heads % pool->num_kv_heads != 0) return 0;
  return workspace_bytes_for(*pool, *batch, num_q_heads);
}

rag_status rag_workspace_init(void* workspace, size_t workspace_bytes, void* stream) {
  if (!workspace || workspace_bytes < 256) return RAG_ERR_WORKSPACE;
  return cudaMemsetAsync(workspace, 0, 256, static_cast<cudaStream_t>(stream)) == cudaSuccess ? RAG_OK
                                                                                            : RAG_ERR_CUDA;
}

}  // extern "C"

namespace rag {

// The fused prefill of one layer; rope_base > 0 re-bases the cached keys to
// their concatenated positions (bf16 pools only).
static rag_status fused_prefill(const rag_kv_pool* pool, int32_t layer, const rag_batch* batch, const void* q,
                                int32_t num_q_heads, const void* kq, const void* vq, float sm_scale,
                                double rope_base, void* o, float* row_lse, float* impact, void* workspace,
                                size_t workspace_bytes, void* stream) {
  rag_status st = check_pool(pool);
  if (st != RAG_OK) return st;
  st = check_batch(batch);
  if (st != RAG_OK) return st;
  if (layer < 0 || layer >= pool->num_layers) return RAG_ERR_INVALID_ARG;
  if (num_q_heads <= 0 || num_q_heads % pool->num_kv_heads != 0) return RAG_ERR_SHAPE;
  const int G = num_q_heads / pool->num_kv_heads;
  const rag_batch& b = *batch;
  if (b.total_q > 0 && (!q || !kq || !vq || !o)) return RAG_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(kq) || !aligned16(vq) || !aligned16(o)) return RAG_ERR_INVALID_ARG;
  if ((row_lse && (reinterpret_cast<uintptr_t>(row_lse) & 3u)) || (impact && (reinterpret_cast<uintptr_t>(impact) & 3u)))
    return RAG_ERR_INVALID_ARG;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return RAG_ERR_WORKSPACE;
  const size_t need = workspace_bytes_for(*pool, b, num_q_heads);
  if (workspace_bytes < need) return RAG_ERR_WORKSPACE;
  const float scale = sm_scale > 0.f ? sm_scale : 1.0f / std::sqrt(float(pool->head_dim));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int32_t* err = reinterpret_cast<int32_t*>(ws);
  const int64_t impact_len = int64_t(b.total_doc) + b.total_q;

  if (b.num_requests == 0) return RAG_OK;
  if (b.total_q == 0) {
    if (impact && impact_len > 0 && cudaMemsetAsync(impact, 0, sizeof(float) * impact_len, s) != cudaSuccess)
      return RAG_ERR_CUDA;
    return RAG_OK;
  }

  if (pool->dtype == RAG_F32) {
    if (rope_base > 0.0) return RAG_ERR_UNSUPPORTED;
    if (b.max_doc + b.max_q > kSimtMaxKeysHost) return RAG_ERR_UNSUPPORTED;
    const WsLayout wl = ws_layout(b.total_q, num_q_heads, 0, 0);
    SimtParams p;
    p.batch = to_dev(b);
    p.num_pages = pool->num_pages;
    p.num_kv_heads = pool->num_kv_heads;
    p.num_q_heads = num_q_heads;
    p.group = G;
    p.layer = layer;
    p.head_dim = pool->head_dim;
    p.scale = scale;
    p.pool_k = static_cast<const float*>(pool->k);
    p.pool_v = static_cast<const float*>(pool->v);
    p.q = static_cast<const float*>(q);
    p.kq = static_cast<const float*>(kq);
    p.vq = static_cast<const float*>(vq);
    p.o = static_cast<float*>(o);
    p.row_lse = row_lse;
    p.row_m = reinterpret_cast<float*>(ws + wl.off_m2);
    p.row_l = reinterpret_cast<float*>(ws + wl.off_il);
    p.impact = impact;
    p.err = err;
    {
      LaunchScope ls(kKindSimtAttn, s);
      cudaError_t e = launch_simt_attn(p, b.total_q, s);
      ls.done(e);
      if (e != cudaSuccess) return RAG_ERR_CUDA;
    }
    if (impact) {
      LaunchScope ls(kKindSimtImpact, s);
      cudaError_t e = launch_simt_impact(p, b.max_doc + b.max_q, b.num_requests, s);
      ls.done(e);
      if (e != cudaSuccess) return RAG_ERR_CUDA;
    }
    return RAG_OK;
  }

  // ---- bf16 tensor-core path
  if (kBM % G != 0) return RAG_ERR_UNSUPPORTED;
  const int sms = num_sms();
  const Plan pf = plan_split(b, pool->num_kv_heads, G, kFwdRows, sms, PlanFor::kAttention);
  const WsLayout wl = ws_layout(b.total_q, num_q_heads, pf.max_items, b.num_chunks);
  const int H_kv = pool->num_kv_heads;
  const uint64_t pool_rows = uint64_t(pool->num_layers) * pool->num_pages * H_kv * kPage;

  // query blocks of at most 16 rows (decode steps) take the transposed kernel
  // of decode_fwd.cu: a key per thread instead of a row per thread
  const bool use_dec = rope_base <= 0.0 && int64_t(b.max_q) * G <= 16 && 16 % G == 0;
  CUtensorMap tm_q, tm_qd, tm_k, tm_v, tm_kq, tm_vq;
  {
    const uint64_t dq[3] = {uint64_t(kHeadDim), uint64_t(num_q_heads), uint64_t(b.total_q)};
    const uint64_t sq[2] = {uint64_t(kHeadDim) * 2, uint64_t(num_q_heads) * kHeadDim * 2};
    const uint32_t bq[3] = {64u, uint32_t(G), uint32_t(kBM / G)};
    const uint64_t dp[2] = {uint64_t(kHeadDim), pool_rows};
    const uint64_t sp[1] = {uint64_t(kHeadDim) * 2};
    const uint32_t bp[2] = {64u, uint32_t(kPage)};
    const uint64_t dk[3] = {uint64_t(kHeadDim), uint64_t(H_kv), uint64_t(b.total_q)};
    const uint64_t sk[2] = {uint64_t(kHeadDim) * 2, uint64_t(H_kv) * kHeadDim * 2};
    const uint32_t bk[3] = {64u, 1u, uint32_t(kBN)};
    if (!make_map(&tm_q, q, 3, dq, sq, bq) || !make_map(&tm_k, pool->k, 2, dp, sp, bp) ||
        !make_map(&tm_v, pool->v, 2, dp, sp, bp) || !make_map(&tm_kq, kq, 3, dk, sk, bk) ||
        !make_map(&tm_vq, vq, 3, dk, sk, bk))
      return RAG_ERR_CUDA;
    // the decode kernel's Q box is its 16 rows: G query heads of 16 / G tokens
    const uint32_t bqd[3] = {64u, uint32_t(G), uint32_t(use_dec ? 16 / G : 1)};
    if (use_dec && !make_map(&tm_qd, q, 3, dq, sq, bqd)) return RAG_ERR_CUDA;
  }
  float* row_m2 = reinterpret_cast<float*>(ws + wl.off_m2);
  float* row_il = reinterpret_cast<float*>(ws + wl.off_il);
  int32_t* item_prefix = reinterpret_cast<int32_t*>(ws + wl.off_prefix);
  float* part = reinterpret_cast<float*>(ws + wl.off_part);
  const float scale_log2 = scale * 1.4426950408889634f;
  float2* rope = nullptr;
  if (rope_base > 0.0) {
    rope = reinterpret_cast<float2*>(ws + wl.off_rope);
    LaunchScope ls(kKindRope, s);
    cudaError_t e = launch_rope_table(to_dev(b), rope_base, rope, s);
    ls.done(e);
    if (e != cudaSuccess) return RAG_ERR_CUDA;
  }

  FwdParams fp;
  fp.batch = to_dev(b);
  fp.num_pages = pool->num_pages;
  fp.num_kv_heads = H_kv;
  fp.num_q_heads = num_q_heads;
  fp.group = G;
  fp.layer = layer;
  fp.tiles_per_split = pf.tiles_per_split;
  fp.direct = pf.direct;
  fp.scale_log2 = scale_log2;
  fp.o = static_cast<__nv_bfloat16*>(o);
  fp.row_lse = row_lse;
  fp.row_m2 = row_m2;
  fp.row_il = row_il;
  fp.part = part;
  fp.item_prefix = item_prefix;
  fp.err = err;
  fp.impact_zero = impact;
  fp.impact_len = impact ? impact_len : 0;
  fp.max_items = pf.max_items;
  fp.rope = rope;
  {
    LaunchScope ls(use_dec ? kKindDecAttn : kKindAttn, s);
    cudaError_t e = use_dec ? launch_decode_attn(tm_qd, tm_k, tm_v, tm_kq, tm_vq, fp, pf.grid, s)
                            : launch_attn_fwd(tm_q, tm_k, tm_v, tm_kq, tm_vq, fp, pf.grid, s);
    ls.done(e);
    if (e != cudaSuccess) return RAG_ERR_CUDA;
  }
  if (!pf.direct) {
    CombineParams cp;
    cp.batch = fp.batch;
    cp.num_kv_heads = H_kv;
    cp.num_q_heads = num_q_heads;
    cp.group = G;
    cp.tiles_per_split = pf.tiles_per_split;
    cp.part = part;
    cp.item_prefix = item_prefix;
    cp.max_items = pf.max_items;
    cp.o = fp.o;
    cp.row_lse = row_lse;
    cp.row_m2 = row_m2;
    cp.row_il = row_il;
    LaunchScope ls(kKindCombine, s);
    const int64_t block_rows = std::min<int64_t>(kFwdRows, int64_t(b.max_q) * G);
    cudaError_t e = launch_attn_combine(cp, pf.max_units_rt, int(block_rows), b.num_requests, s);
    ls.done(e);
    if (e != cudaSuccess) return RAG_ERR_CUDA;
  }
  if (impact) {
    const Plan pi = plan_split(b, H_kv, G, kImpactRows, sms, PlanFor::kImpact);
    ImpactParams ip;
    ip.batch = fp.batch;
    ip.num_pages = pool->num_pages;
    ip.num_kv_heads = H_kv;
    ip.num_q_heads = num_q_heads;
    ip.group = G;
    ip.layer = layer;
    ip.tiles_per_split = pi.tiles_per_split;
    ip.scale_log2 = scale_log2;
    ip.row_m2 = row_m2;
    ip.row_il = row_il;
    ip.impact = impact;
    ip.err = err;
    ip.rope = rope;
    LaunchScope ls(kKindImpact, s);
    cudaError_t e = launch_impact(tm_q, tm_k, tm_kq, ip, pi.grid, s);
    ls.done(e);
    if (e != cudaSuccess) return RAG_ERR_CUDA;
  }
  return RAG_OK;
}

}  // namespace rag

extern "C" {

rag_status rag_fused_prefill_attn(const rag_kv_pool* pool, int32_t layer, const rag_batch* batch, const void* q,
                                  int32_t num_q_heads, const void* kq, const void* vq, float sm_scale, void* o,
                                  float* row_lse, float* impact, void* workspace, size_t workspace_bytes,
                                  void* stream) {
  return fused_prefill(pool, layer, batch, q, num_q_heads, kq, vq, sm_scale, 0.0, o, row_lse, impact, workspace,
                       workspace_bytes, stream);
}

rag_status rag_fused_prefill_attn_rope(const rag_kv_pool* pool, int32_t layer, const rag_batch* batch,
                                       const void* q, int32_t num_q_heads, const void* kq, const void* vq,
                                       float sm_scale, double rope_base, void* o, float* row_lse, float* impact,
                                       void* workspace, size_t workspace_bytes, void* stream) {
  if (!(rope_base > 1.0) || !std::isfinite(rope_base)) return RAG_ERR_INVALID_ARG;
  return fused_prefill(pool, layer, batch, q, num_q_heads, kq, vq, sm_scale, rope_base, o, row_lse, impact,
                       workspace, workspace_bytes, stream);
}

rag_status rag_impact_topk(const float* impact, const rag_batch* batch, double r, int32_t k_cap, int32_t* topk_idx,
                           float* topk_val, int32_t* k_out, void* stream) {
  rag_status st = check_batch(batch);
  if (st != RAG_OK) return st;
  if (!(r > 0.0 && r < 1.0)) return RAG_ERR_INVALID_ARG;
  const rag_batch& b = *batch;
  if (b.num_requests == 0) return RAG_OK;
  if (!impact || !topk_idx) return RAG_ERR_INVALID_ARG;
  const int kmax = rag_recompute_count(b.max_doc, r);
  if (k_cap < std::max(kmax, 1)) return RAG_ERR_SHAPE;
  if (kmax > kTopkMaxKHost) return RAG_ERR_UNSUPPORTED;
  TopkParams p;
  p.batch = to_dev(b);
  p.impact = impact;
  p.r = r;
  p.k_cap = k_cap;
  p.k_max = std::max(kmax, 1);
  p.topk_idx = topk_idx;
  p.topk_val = topk_val;
  p.k_out = k_out;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  LaunchScope ls(kKindTopk, s);
  cudaError_t e = launch_topk(p, b.num_requests, p.k_max, s);
  ls.done(e);
  return e == cudaSuccess ? RAG_OK : RAG_ERR_CUDA;
}

// ------------------------------------------------------------ KV decode into the pool

rag_status rag_kv_decode(const rag_kv_pool* pool, int32_t layer, int32_t n_chunks, const int32_t* chunk_tok_off,
                         const int32_t* chunk_page_off, const int32_t* page_ids, int32_t total_pages, int32_t bits,
                         const void* codes_k, const void* codes_v, const float* scale_k, const float* offset_k,
                         const float* scale_v, const float* offset_v, int32_t* device_err, void* stream) {
  rag_status st = check_pool(pool);
  if (st != RAG_OK) return st;
  if (pool->dtype != RAG_BF16) return RAG_ERR_UNSUPPORTED;
  if (layer < 0 || layer >= pool->num_layers) return RAG_ERR_INVALID_ARG;
  if (bits != 4 && bits != 8) return RAG_ERR_UNSUPPORTED;
  if (n_chunks < 0 || total_pages < 0) return RAG_ERR_SHAPE;
  if (n_chunks == 0 || total_pages == 0) return RAG_OK;
  if (!chunk_tok_off || !chunk_page_off || !page_ids || !codes_k || !codes_v || !scale_k || !offset_k ||
      !scale_v || !offset_v)
    return RAG_ERR_INVALID_ARG;
  // codes: 8-byte (8-bit) or 4-byte (4-bit) loads per 8 channels; scales: 16-byte loads
  if ((reinterpret_cast<uintptr_t>(codes_k) | reinterpret_cast<uintptr_t>(codes_v)) & 7u) return RAG_ERR_INVALID_ARG;
  if (!aligned16(scale_k) || !aligned16(offset_k) || !aligned16(scale_v) || !aligned16(offset_v))
    return RAG_ERR_INVALID_ARG;
  KvDecodeParams p;
  p.pool_k = static_cast<__nv_bfloat16*>(pool->k);
  p.pool_v = static_cast<__nv_bfloat16*>(pool->v);
  p.chunk_tok_off = chunk_tok_off;
  p.chunk_page_off = chunk_page_off;
  p.page_ids = page_ids;
  p.codes_k = static_cast<const uint8_t*>(codes_k);
  p.codes_v = static_cast<const uint8_t*>(codes_v);
  p.scale_k = scale_k;
  p.offset_k = offset_k;
  p.scale_v = scale_v;
  p.offset_v = offset_v;
  p.err = device_err;
  p.layer = layer;
  p.num_pages = pool->num_pages;
  p.num_kv_heads = pool->num_kv_heads;
  p.n_chunks = n_chunks;
  p.bits = bits;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  LaunchScope ls(kKindKvDecode, s);
  cudaError_t e = launch_kv_decode(p, total_pages, s);
  ls.done(e);
  return e == cudaSuccess ? RAG_OK : RAG_ERR_CUDA;
}

// ------------------------------------------------------------ selective recompute

size_t rag_recompute_plan_size(const rag_batch* batch, int32_t k_cap) {
  if (check_batch(batch) != RAG_OK || k_cap < 1) return 0;
  const RcPlanLayout l = rc_plan_layout(int64_t(batch->num_requests) * k_cap, batch->num_page_refs);
  return size_t(l.words) * sizeof(int32_t);
}

rag_status rag_recompute_plan(const rag_batch* batch, const int32_t* topk_idx, int32_t k_cap, const int32_t* k,
                              const int32_t* free_pages, int32_t n_free, int32_t x_by_selection,
                              int32_t* page_ids_out, void* plan, size_t plan_bytes, void* stream) {
  rag_status st = check_batch(batch);
  if (st != RAG_OK) return st;
  if (k_cap < 1 || n_free < 0) return RAG_ERR_SHAPE;
  const rag_batch& b = *batch;
  if (!plan || (reinterpret_cast<uintptr_t>(plan) & 255u)) return RAG_ERR_WORKSPACE;
  if (plan_bytes < rag_recompute_plan_size(batch, k_cap)) return RAG_ERR_WORKSPACE;
  if (b.num_requests > 0 && (!topk_idx || !k)) return RAG_ERR_INVALID_ARG;
  if (b.num_page_refs > 0 && !page_ids_out) return RAG_ERR_INVALID_ARG;
  if (n_free > 0 && !free_pages) return RAG_ERR_INVALID_ARG;
  RcPlanParams p;
  p.batch = to_dev(b);
  p.topk_idx = topk_idx;
  p.k = k;
  p.free_pages = free_pages;
  p.page_ids_out = page_ids_out;
  p.plan = static_cast<int32_t*>(plan);
  p.lay = rc_plan_layout(int64_t(b.num_requests) * k_cap, b.num_page_refs);
  p.k_cap = k_cap;
  p.n_free = n_free;
  p.by_selection = x_by_selection ? 1 : 0;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  LaunchScope ls(kKindRcPlan, s);
  cudaError_t e = launch_rc_plan(p, s);
  ls.done(e);
  return e == cudaSuccess ? RAG_OK : RAG_ERR_CUDA;
}

rag_status rag_recompute_kv(const rag_kv_pool* pool, int32_t layer, const rag_batch* batch, int32_t k_cap,
                            const void* plan, size_t plan_bytes, const void* x, int64_t x_rows, int32_t d_model,
                            const void* w_k, const void* w_v, void* stream) {
  rag_status st = check_pool(pool);
  if (st != RAG_OK) return st;
  st = check_batch(batch);
  if (st != RAG_OK) return st;
  if (pool->dtype != RAG_BF16) return RAG_ERR_UNSUPPORTED;
  if (layer < 0 || layer >= pool->num_layers) return RAG_ERR_INVALID_ARG;
  if (k_cap < 1) return RAG_ERR_SHAPE;
  if (d_model < kRcMinDModel || d_model % 64 != 0 || d_model > (1 << 20)) return RAG_ERR_UNSUPPORTED;
  if (x_rows < 1 || x_rows >= (int64_t(1) << 31)) return RAG_ERR_SHAPE;
  if (!plan || (reinterpret_cast<uintptr_t>(plan) & 255u)) return RAG_ERR_WORKSPACE;
  if (plan_bytes < rag_recompute_plan_size(batch, k_cap)) return RAG_ERR_WORKSPACE;
  if (!x || !w_k || !w_v || !aligned16(x) || !aligned16(w_k) || !aligned16(w_v)) return RAG_ERR_INVALID_ARG;
  const rag_batch& b = *batch;
  const int H_kv = pool->num_kv_heads;
  const RcPlanLayout lay = rc_plan_layout(int64_t(b.num_requests) * k_cap, b.num_page_refs);
  const int64_t max_tok = int64_t(b.num_requests) * k_cap;
  if (max_tok == 0) return RAG_OK;
  const int hpt = (H_kv % 2 == 0) ? 2 : 1;   // output heads per projection tile
  CUtensorMap tm_x, tm_xt, tm_wk, tm_wv;
  {
    const uint64_t dx[2] = {uint64_t(d_model), uint64_t(x_rows)};
    const uint64_t sx[1] = {uint64_t(d_model) * 2};
    const uint32_t bx[2] = {64u, 1u};       // gather4: one row per box
    const uint32_t bxt[2] = {64u, 128u};    // consecutive rows: one 128-row box
    const uint64_t dw[2] = {uint64_t(d_model), uint64_t(H_kv) * kHeadDim};
    const uint32_t bw[2] = {64u, uint32_t(128 * hpt)};   // the rows of hpt heads
    if (!make_map(&tm_x, x, 2, dx, sx, bx) || !make_map(&tm_xt, x, 2, dx, sx, bxt) ||
        !make_map(&tm_wk, w_k, 2, dw, sx, bw) || !make_map(&tm_wv, w_v, 2, dw, sx, bw))
      return RAG_ERR_CUDA;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int sms = num_sms();
  {
    RcCopyParams cp;
    cp.pool_k = static_cast<uint8_t*>(pool->k);
    cp.pool_v = static_cast<uint8_t*>(pool->v);
    cp.plan = static_cast<int32_t*>(const_cast<void*>(plan));
    cp.lay = lay;
    cp.layer = layer;
    cp.num_pages = pool->num_pages;
    cp.num_kv_heads = H_kv;
    const int grid = int(std::max<int64_t>(1, std::min<int64_t>(int64_t(4) * sms, b.num_page_refs)));
    LaunchScope ls(kKindRcCopy, s);
    cudaError_t e = launch_rc_copy(cp, grid, s);
    ls.done(e);
    if (e != cudaSuccess) return RAG_ERR_CUDA;
  }
  RcGemmParams gp;
  gp.pool_k = static_cast<__nv_bfloat16*>(pool->k);
  gp.pool_v = static_cast<__nv_bfloat16*>(pool->v);
  gp.plan = static_cast<int32_t*>(const_cast<void*>(plan));
  gp.lay = lay;
  gp.layer = layer;
  gp.num_pages = pool->num_pages;
  gp.num_kv_heads = H_kv;
  gp.d_model = d_model;
  gp.x_rows = int32_t(x_rows);
  gp.heads_per_tile = hpt;
  gp.max_tok = max_tok;
  const int64_t tiles_bound = ((max_tok + 127) / 128) * (2 * H_kv / hpt);
  const int grid = int(std::max<int64_t>(1, std::min<int64_t>(sms, tiles_bound)));
  LaunchScope ls(kKindRcGemm, s);
  cudaError_t e = launch_rc_gemm(tm_x, tm_xt, tm_wk, tm_wv, gp, grid, s);
  ls.done(e);
  return e == cudaSuccess ? RAG_OK : RAG_ERR_CUDA;
}

rag_status rag_recompute_status(const void* plan, int32_t* counts, void* stream) {
  if (!plan) return RAG_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int32_t hdr[4] = {0, 0, 0, 0};
  if (cudaMemcpyAsync(hdr, plan, sizeof(hdr), cudaMemcpyDeviceToHost, s) != cudaSuccess) return RAG_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return RAG_ERR_CUDA;
  if (counts) {
    counts[0] = hdr[kRcHdrTok];
    counts[1] = hdr[kRcHdrCow];
    counts[2] = hdr[kRcHdrNeeded];
  }
  const int32_t bits = hdr[kRcHdrErr];
  if (bits & kDevErrTimeout) return RAG_ERR_TIMEOUT;
  if (bits & kRcErrNoFree) return RAG_ERR_NO_FREE_PAGES;
  if (bits & kDevErrPage) return RAG_ERR_PAGE_OOB;
  if (bits & kDevErrGeometry) return RAG_ERR_GEOMETRY;
  if (bits & kDevErrRange) return RAG_ERR_RANGE;
  return RAG_OK;
}

rag_status rag_last_device_error(void* workspace, int32_t* bits, void* stream) {
  if (!workspace) return RAG_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int32_t host = 0;
  if (cudaMemcpyAsync(&host, workspace, sizeof(int32_t), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return RAG_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return RAG_ERR_CUDA;
  if (host != 0 && cudaMemsetAsync(workspace, 0, sizeof(int32_t), s) != cudaSuccess) return RAG_ERR_CUDA;
  if (bits) *bits = host;
  if (host & kDevErrTimeout) return RAG_ERR_TIMEOUT;
  if (host & kDevErrPage) return RAG_ERR_PAGE_OOB;
  if (host & kDevErrGeometry) return RAG_ERR_GEOMETRY;
  if (host & kDevErrRange) return RAG_ERR_RANGE;
  return RAG_OK;
}

int64_t rag_launch_count(void) { return g_launches.load(); }

const char* rag_last_cuda_error(void) {
  return cudaGetErrorName(static_cast<cudaError_t>(g_last_cuda_error.load()));
}

void rag_profile_enable(int32_t on) { g_prof_on.store(on ? 1 : 0); }

rag_status rag_profile_peek(double* ms, int64_t* launches, int32_t n_kinds) {
  std::vector<ProfRecord> recs;
  {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    recs = g_prof;
  }
  std::vector<double> acc(kNumKinds, 0.0);
  std::vector<int64_t> cnt(kNumKinds, 0);
  rag_status st = RAG_OK;
  for (auto& r : recs) {
    float t = 0.f;
    if (cudaEventSynchronize(r.stop) != cudaSuccess || cudaEventElapsedTime(&t, r.start, r.stop) != cudaSuccess)
      st = RAG_ERR_CUDA;
    acc[r.kind] += t;
    cnt[r.kind] += 1;
  }
  for (int i = 0; i < n_kinds && i < kNumKinds; ++i) {
    if (ms) ms[i] = acc[i];
    if (launches) launches[i] = cnt[i];
  }
  return st;
}

rag_status rag_profile_collect(double* ms, int64_t* launches, int32_t n_kinds) {
  std::vector<ProfRecord> recs;
  {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    recs.swap(g_prof);
  }
  std::vector<double> acc(kNumKinds, 0.0);
  std::vector<int64_t> cnt(kNumKinds, 0);
  rag_status st = RAG_OK;
  for (auto& r : recs) {
    float t = 0.f;
    if (cudaEventSynchronize(r.stop) != cudaSuccess || cudaEventElapsedTime(&t, r.start, r.stop) != cudaSuccess)
      st = RAG_ERR_CUDA;
    acc[r.kind] += t;
    cnt[r.kind] += 1;
  }
  {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    for (auto& r : recs) {
      g_event_pool.push_back(r.start);
      g_event_pool.push_back(r.stop);
    }
  }
  for (int i = 0; i < n_kinds && i < kNumKinds; ++i) {
    if (ms) ms[i] = acc[i];
    if (launches) launches[i] = cnt[i];
  }
  return st;
}

}  // extern "C"
