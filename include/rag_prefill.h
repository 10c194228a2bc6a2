/*
 * rag_prefill.h - C ABI of the precomputed-KV RAG prefill hot path on B200
 * (sm_100a): paged-pool gather, causal attention of the query block over the
 * concatenated chunk caches, CacheBlend Impact, and top-k recompute selection.
 *
 * Method (cited by page title and section):
 *   - TurboRAG page, "Technical Details / KV cache precompute": every chunk's
 *     per-layer K, V are computed once offline (listing `precompute_kv_cache`)
 *     and reused; at query time K_combined = Concat(K^(1), ..., K^(m), K^(Q))
 *     and likewise V, in retrieval order, along the sequence axis (listing
 *     `turborag_inference`).
 *   - TurboRAG page, "Causal vs non-causal attention":
 *     Attention(Q, K, V) = softmax(Q K^T / sqrt(d_k) + M_causal) V. Query token
 *     j of a request sits at position N_doc + j, so every doc key is visible
 *     to it and the mask is causal only inside the query block.
 *   - CacheBlend page, "Mathematical formulation": Impact(i) = sum over tokens
 *     j outside doc(i) of alpha_{j,i}; here j ranges over the query tokens and
 *     the per-head sums are averaged over the H_q query heads.
 *   - CacheBlend page, "Recompute ratio trade-off" and the listing
 *     `select_tokens_for_recompute`: k = max(1, int(N_doc * r)) doc tokens of
 *     largest Impact.
 *
 * Conventions for every entry point:
 *   - Ownership: the library never allocates or frees device memory. All
 *     tensors and the workspace belong to the caller; `stream` is a
 *     cudaStream_t passed as void* (NULL = legacy default stream) and every
 *     call is asynchronous on it unless stated otherwise.
 *   - Device pointers must be 16-byte aligned (TMA); strides are implied by
 *     the shapes (dense, row-major, innermost dimension last).
 *   - Argument, shape and dtype errors are reported synchronously by the
 *     return value and nothing is launched. Problems the device finds (a page
 *     id outside the pool, a chunk whose page count is not ceil(len / 16), a
 *     pipeline wait that gave up) are recorded in the workspace error word,
 *     never trapped, and reported by rag_last_device_error.
 *   - Indices of doc tokens are logical positions within their request,
 *     0 .. N_doc,b - 1, in concatenation order.
 *   - Stream order holds as usual. The kernels are launched with programmatic
 *     stream serialization. When the previous kernel in the stream is one of
 *     this library's attention, combine, Impact or top-k kernels, the next
 *     one may start while it finishes: it sets up and reads its own inputs
 *     (the pool, the batch descriptors, q, kq, vq), none of which those
 *     kernels write, and writes global memory only after the previous kernel
 *     has completed. Kernels that write pool pages, page tables or the RoPE
 *     table (pool write, KV decode, recompute, RoPE table) and every kernel
 *     not of this library let the next kernel start only when they complete.
 */
#ifndef RAG_PREFILL_H_
#define RAG_PREFILL_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define RAG_API __attribute__((visibility("default")))
#else
#define RAG_API
#endif

#define RAG_ABI_VERSION 1
#define RAG_PAGE_SIZE 16

typedef enum {
  RAG_OK = 0,
  RAG_ERR_INVALID_ARG = 1, /* null/misaligned pointer, bad scalar            */
  RAG_ERR_SHAPE = 2,       /* inconsistent sizes                              */
  RAG_ERR_PAGE_OOB = 3,    /* device: a page id outside [0, num_pages)        */
  RAG_ERR_UNSUPPORTED = 4, /* valid request the library does not implement    */
  RAG_ERR_CUDA = 5,        /* a CUDA runtime call failed                      */
  RAG_ERR_TIMEOUT = 6,     /* device: a pipeline wait gave up                 */
  RAG_ERR_WORKSPACE = 7,   /* workspace missing or smaller than required      */
  RAG_ERR_GEOMETRY = 8,    /* device: chunk pages do not match its length     */
  RAG_ERR_RANGE = 9,       /* device: a V value of magnitude >= 65536 (or
                              inf/nan) was stored or used as fp16 and was
                              saturated to +-65504 (nan kept)                */
  RAG_ERR_NO_FREE_PAGES = 10 /* device: the copy-on-write recompute needs more
                              private pages than the free list holds          */
} rag_status;

typedef enum { RAG_BF16 = 0, RAG_F32 = 1 } rag_dtype;

/* The paged pool of precomputed chunk caches (caller-owned device memory).
 * k, v: [num_layers][num_pages][num_kv_heads][16][head_dim].
 * Page p of layer l, kv head g holds 16 consecutive tokens of one chunk.
 * Element types: RAG_F32 keeps K and V in fp32. RAG_BF16 (a bf16 cache)
 * keeps K in bf16 and V in fp16, the type in which V enters the product
 * with the attention weights. rag_kv_pool_write stores the fp16 value of each
 * bf16 V value (exact for magnitudes in [2^-14, 65280], within 2^-25 below);
 * rag_kv_decode and rag_recompute_kv round their fp32 V values once to fp16.
 * All round to nearest even; magnitudes beyond the fp16 range, inf and nan
 * saturate to +-65504 (nan kept) and the writing call reports RAG_ERR_RANGE.
 * Supported: RAG_BF16 with head_dim 128 (tensor-core path), RAG_F32 with
 * head_dim 64 or 128 (CUDA-core path). */
typedef struct {
  void* k;
  void* v;
  int32_t num_layers;
  int32_t num_pages;
  int32_t num_kv_heads;
  int32_t page_size; /* must be RAG_PAGE_SIZE */
  int32_t head_dim;
  int32_t dtype;     /* rag_dtype */
} rag_kv_pool;

/* One batch of B requests. The int32 arrays are DEVICE pointers; the scalars
 * are host-side totals and maxima used to size launches and the workspace.
 * Request b retrieved the chunk-list entries [req_chunk_off[b],
 * req_chunk_off[b+1]) in retrieval order; an entry may repeat a chunk.
 *   req_chunk_off  [B+1]  prefix over requests of chunk-list entries
 *   chunk_doc_off  [C+1]  prefix over the chunk list of chunk lengths (tokens)
 *   chunk_page_off [C+1]  prefix over the chunk list of page counts; entry c
 *                         must have ceil(len_c / 16) pages
 *   page_ids       [P]    physical page of each referenced page, in order
 *   q_off          [B+1]  prefix over requests of query tokens
 * Request b's doc tokens are chunk_doc_off[req_chunk_off[b]] ..
 * chunk_doc_off[req_chunk_off[b+1]] - 1; its query tokens are q_off[b] ..
 * q_off[b+1] - 1. */
typedef struct {
  int32_t num_requests;  /* B, 0 .. 4096 */
  int32_t num_chunks;    /* C */
  int32_t num_page_refs; /* P */
  int32_t total_q;       /* q_off[B] */
  int32_t total_doc;     /* chunk_doc_off[C] */
  int32_t max_q;         /* max_b query tokens */
  int32_t max_doc;       /* max_b doc tokens */
  int32_t max_pages;     /* max_b pages referenced by one request */
  const int32_t* req_chunk_off;
  const int32_t* chunk_doc_off;
  const int32_t* chunk_page_off;
  const int32_t* page_ids;
  const int32_t* q_off;
} rag_batch;

/* ABI version of the loaded library (RAG_ABI_VERSION). */
RAG_API int32_t rag_abi_version(void);

/* Static text for a rag_status value. */
RAG_API const char* rag_status_string(int32_t status);

/* Number of SMs of the current device (launch sizing). */
RAG_API int32_t rag_num_sms(void);

/* Pool write (TurboRAG page, "Technical Details / KV cache precompute"; the
 * listing `precompute_kv_cache`): store one chunk's dense K, V
 * [n_tokens][num_kv_heads][head_dim] (pool dtype: bf16 or fp32, device) into
 * the pages page_ids[0 .. n_pages-1] (device int32) of `layer`. Token t goes
 * to page page_ids[t / 16], slot t % 16; the slots of the last page beyond
 * n_tokens are zeroed. n_pages must equal ceil(n_tokens / 16). In a bf16 pool
 * V is stored as fp16 (see rag_kv_pool). *device_err (optional device int32,
 * may be NULL) collects bits: 1 a page id outside the pool (skipped), 8 a V
 * value saturated. */
RAG_API rag_status rag_kv_pool_write(const rag_kv_pool* pool, int32_t layer, const int32_t* page_ids, int32_t n_pages,
                             int32_t n_tokens, const void* k, const void* v, int32_t* device_err, void* stream);

/* Bytes of workspace rag_fused_prefill_attn needs for this pool, batch and
 * head count (0 on invalid arguments). The workspace holds the device error
 * word, per-row softmax statistics and split-KV partials; it must be zeroed
 * once before first use (rag_workspace_init) and may be reused across calls
 * on one stream. */
RAG_API size_t rag_workspace_size(const rag_kv_pool* pool, const rag_batch* batch, int32_t num_q_heads);

/* Clear the workspace's error word (async on `stream`). */
RAG_API rag_status rag_workspace_init(void* workspace, size_t workspace_bytes, void* stream);

/* Fused prefill of one layer for the whole batch:
 *   gather [K_1; ...; K_m; K_q] through the page table (TurboRAG page,
 *   Concat equation), then for every query head h (KV head h / G) and query
 *   token j of request b:  O[j,h] = sum_i softmax_i(scale * Q[j,h] . K_i) V_i
 *   over keys i <= N_doc,b + j (TurboRAG page, causal attention equation).
 * q      [total_q][num_q_heads][head_dim]   pool dtype, device
 * kq, vq [total_q][num_kv_heads][head_dim]  the query block's own K, V
 * sm_scale <= 0 selects 1 / sqrt(head_dim).
 * o      [total_q][num_q_heads][head_dim]   output, pool dtype
 * row_lse optional [total_q][num_q_heads] fp32: log sum_i exp(scale Q.K_i)
 * impact  optional [total_doc + total_q] fp32 output. When given, the call
 *   also computes CacheBlend's Impact (CacheBlend page, "Mathematical
 *   formulation"): for request b the segment at offset
 *   chunk_doc_off[req_chunk_off[b]] + q_off[b] holds, for each of its
 *   N_doc,b + q_b key positions i, (1/H_q) sum_h sum_j alpha^h_{j,i}; the doc
 *   part comes first. The impacts of a request's segment add up to q_b.
 *   Pass it on the layer whose attention selects tokens (the last layer).
 * workspace: device, >= rag_workspace_size() bytes, 256-byte aligned.
 * Precision (bf16 pool): scores and the softmax run in fp32; the PV product
 * takes the weights P and V in fp16 (P keeps 3 more mantissa bits than bf16)
 * with an fp32 accumulator. The pool holds V as fp16 already; the query
 * block's vq (bf16) is rounded to fp16 the same way, and a vq value of
 * magnitude 65536 or more (or inf/nan) is saturated and the call reports
 * RAG_ERR_RANGE through rag_last_device_error. */
RAG_API rag_status rag_fused_prefill_attn(const rag_kv_pool* pool, int32_t layer, const rag_batch* batch, const void* q,
                                  int32_t num_q_heads, const void* kq, const void* vq, float sm_scale, void* o,
                                  float* row_lse, float* impact, void* workspace, size_t workspace_bytes,
                                  void* stream);

/* rag_fused_prefill_attn with the cached keys re-based to their positions in
 * the concatenated sequence (TurboRAG page, "Implementation": with rotary
 * position embeddings, the position ids of the offline precompute and of
 * inference must agree). Each chunk's cached K is taken to carry RoPE at its
 * chunk-local positions 0 .. n_c - 1; chunk-list entry e of a request starts at
 * offset o_e (the doc tokens of the request's entries before it), and every
 * key of it is turned by o_e positions: rotary pair i (channels i and i + 64)
 * by the angle o_e * rope_base^(-2i/128). The rotated key is rounded once to
 * bf16 (the cache dtype) before the products. The query block's q, kq are
 * expected with RoPE at their positions N_doc,b + j already applied. The pool
 * itself is not modified (the rotation happens on the way from HBM to the
 * tensor core, in attention and in the Impact pass alike). rope_base > 1
 * (10000 for Llama-2, 500000 for Llama-3); bf16 pools only. The workspace
 * holds a (cos, sin) table per chunk-list entry, rebuilt by every call. */
RAG_API rag_status rag_fused_prefill_attn_rope(const rag_kv_pool* pool, int32_t layer, const rag_batch* batch,
                                               const void* q, int32_t num_q_heads, const void* kq, const void* vq,
                                               float sm_scale, double rope_base, void* o, float* row_lse,
                                               float* impact, void* workspace, size_t workspace_bytes,
                                               void* stream);

/* Same computation as rag_fused_prefill_attn, for callers that cannot
 * allocate device memory (a runtime that gives a plugin only its input and
 * output buffers, a deployment whose device memory is planned once at start-up,
 * a loop that must never wait on an allocator). The pages have no counterpart
 * of this entry point; it exists only for such callers.
 * Instead of a caller workspace it uses one fixed device array of 64 MiB that
 * lives in this library's device image: every GPU on which the library has been
 * loaded keeps it until the process exits, and nothing is allocated per call.
 * A batch whose workspace (rag_workspace_size) exceeds 64 MiB is rejected with
 * RAG_ERR_WORKSPACE before anything is launched.
 * All calls share that one array and it keeps the last call's contents: the
 * call clears the error word it needs zeroed, but calls that overlap on the GPU
 * (different streams, or different host threads, on one device) race on it;
 * serialise them on one stream.
 * The first call on each device looks up the array's device address (with that
 * device current); make that first call before any stream capture. The address
 * is kept for the life of the process: after cudaDeviceReset (or any other
 * reset of the device's primary context) the library's device image is loaded
 * again and the kept address is stale, so a process that resets a device must
 * not call this entry point on it afterwards.
 * device_err: optional device int32 that receives the call's device error bits
 * (as rag_last_device_error reports them: 1 page, 2 geometry, 4 timeout,
 * 8 range).
 * Other arguments and outputs as for rag_fused_prefill_attn. */
RAG_API rag_status rag_fused_prefill_attn_static(const rag_kv_pool* pool, int32_t layer, const rag_batch* batch,
                                                 const void* q, int32_t num_q_heads, const void* kq,
                                                 const void* vq, float sm_scale, void* o, float* row_lse,
                                                 float* impact, int32_t* device_err, void* stream);

/* Recompute count for a request with n_doc doc tokens (CacheBlend page,
 * "Recompute ratio trade-off" and listing): max(1, int(n_doc * r)) with the
 * product in double precision, and 0 when n_doc is 0. Host function. */
RAG_API int32_t rag_recompute_count(int32_t n_doc, double r);

/* Top-k recompute selection for every request (CacheBlend listing
 * `select_tokens_for_recompute`, torch.topk over the doc slice):
 * impact   as written by rag_fused_prefill_attn (device fp32)
 * r        recompute ratio, 0 < r < 1
 * k_cap    row length of the outputs, >= rag_recompute_count(max_doc, r).
 *          The selection itself is limited to k = rag_recompute_count(max_doc,
 *          r) <= 16384 per request (RAG_ERR_UNSUPPORTED above that); k_cap
 *          may be larger, the rest of each row is padding
 * topk_idx [B][k_cap] int32 device output: the k_b doc positions of largest
 *          impact ordered by (impact descending, position ascending); the
 *          rest of the row is -1
 * topk_val optional [B][k_cap] fp32: their impacts (0 past k_b)
 * k_out    optional [B] int32: k_b */
RAG_API rag_status rag_impact_topk(const float* impact, const rag_batch* batch, double r, int32_t k_cap,
                           int32_t* topk_idx, float* topk_val, int32_t* k_out, void* stream);

/* ---- Decode of quantized chunk caches into the pool ---------------------------
 * CacheGen page, "How the technology works": a prefilled chunk's KV cache is
 * kept (or sent) as a compact stream and decoded on the GPU into a KV cache
 * from which generation starts; its glossary names quantization with
 * different compression levels for different parts of the cache. The pages
 * give no stream format; this entry point decodes the plainest one they
 * support: per chunk, layer, KV head and channel, b-bit codes (b = 8 or 4,
 * chosen per call, i.e. per layer) of a uniform quantization with an fp32
 * scale and offset. value = fp32 fma(code, scale, offset), rounded once to
 * the type the pool stores it in (bf16 for K, fp16 for V, see rag_kv_pool).
 *
 * One call decodes n_chunks chunks of one layer (bf16 pool, head_dim 128):
 *   chunk_tok_off  [n_chunks+1] device int32: token prefix over the chunks
 *   chunk_page_off [n_chunks+1] device int32: page prefix; chunk c owns
 *                  ceil(n_c / 16) pages
 *   page_ids       [total_pages] device int32: destination pages, in order
 *   codes_k/v      [total_tokens][num_kv_heads][128 * bits / 8] device bytes,
 *                  8-byte aligned (4 bits: even channel in the low nibble)
 *   scale_k/v, offset_k/v [n_chunks][num_kv_heads][128] device fp32, 16-byte
 *                  aligned
 * Token t of chunk c lands in slot t % 16 of page page_ids[chunk_page_off[c] +
 * t / 16]; the last page's slots past the chunk are zeroed. A page id outside
 * the pool or a chunk whose page count is not ceil(n_c / 16) is skipped and
 * recorded in *device_err (optional device int32: 1 page, 2 geometry, 8 a V
 * value saturated). */
RAG_API rag_status rag_kv_decode(const rag_kv_pool* pool, int32_t layer, int32_t n_chunks,
                                 const int32_t* chunk_tok_off, const int32_t* chunk_page_off,
                                 const int32_t* page_ids, int32_t total_pages, int32_t bits, const void* codes_k,
                                 const void* codes_v, const float* scale_k, const float* offset_k,
                                 const float* scale_v, const float* offset_v, int32_t* device_err, void* stream);

/* ---- Selective recompute of the chosen tokens' K and V ---------------------
 * CacheBlend page, "Contributions" (only the tokens of high attention impact
 * are recomputed when the cached KV are fused) and "How it works" (after the
 * high-Impact tokens are found, their KV values are recomputed and generation
 * runs on the fused cache). A chunk's pages are shared by every request that
 * retrieved it, so the recompute never writes them: each page reference that
 * holds a selected token gets a private page (copy on write) and the
 * request's page table is rewritten to point at it.
 *
 * Use: rag_impact_topk -> rag_recompute_plan (once) -> rag_recompute_kv for
 * every layer, with the layer's hidden states of the selected tokens and its
 * K/V projection weights -> attention with page_ids_out as the page table. */

/* Bytes of the plan buffer for this batch and top-k row length (0 on invalid
 * arguments). */
RAG_API size_t rag_recompute_plan_size(const rag_batch* batch, int32_t k_cap);

/* Plan the copy-on-write pages and the destination of every selected token.
 * topk_idx [B][k_cap], k [B]: as written by rag_impact_topk (device int32);
 *   request b's selected doc positions are topk_idx[b][0 .. k[b]-1].
 * free_pages [n_free] device int32: page ids of the pool the caller reserved
 *   for private copies (distinct, unused by any page table). They are handed
 *   out in ascending order of page reference over the whole batch.
 * x_by_selection: 0 -> the hidden state of request b's position i is row
 *   chunk_doc_off[req_chunk_off[b]] + i of the x array given to
 *   rag_recompute_kv ([total_doc][d_model], every doc token of the batch);
 *   1 -> row t, the token's rank in the batch's selection (requests in order,
 *   then topk order: [sum_b k[b]][d_model]).
 * page_ids_out [num_page_refs] device int32: the batch's page table after copy
 *   on write (may be batch->page_ids itself, updated in place).
 * plan: device buffer of rag_recompute_plan_size bytes, 256-byte aligned,
 *   written here and read by rag_recompute_kv; one plan serves every layer.
 * If the selection needs more private pages than n_free, nothing is remapped
 * (page_ids_out = page_ids), rag_recompute_kv then writes nothing, and
 * rag_recompute_status reports RAG_ERR_NO_FREE_PAGES with the count needed.
 * A selected position outside its request is skipped (RAG_ERR_GEOMETRY). */
RAG_API rag_status rag_recompute_plan(const rag_batch* batch, const int32_t* topk_idx, int32_t k_cap,
                                      const int32_t* k, const int32_t* free_pages, int32_t n_free,
                                      int32_t x_by_selection, int32_t* page_ids_out, void* plan,
                                      size_t plan_bytes, void* stream);

/* One layer of the recompute (bf16 pool, head_dim 128):
 *   every private page first receives, for this layer, the K and V of every
 *   slot that is not selected from the page it replaces (all KV heads);
 *   every selected token's rows are recomputed from its hidden state:
 *   K = x W_K^T, V = x W_V^T (fp32 accumulation, one rounding to the stored
 *   type: bf16 for K, fp16 for V, see rag_kv_pool), split into num_kv_heads
 *   heads of 128, and stored into its slot of its private page. The copy
 *   and the recompute never write the same bytes.
 * x   [x_rows][d_model] bf16 device, rows as x_by_selection of the plan says;
 * w_k, w_v [num_kv_heads * 128][d_model] bf16 device (a linear layer's weight);
 * d_model a multiple of 64. batch and k_cap as given to rag_recompute_plan.
 * Device problems (a free page id outside the pool, a row past x_rows, a wait
 * that gave up, a V value saturated) are recorded in the plan and reported by
 * rag_recompute_status. */
RAG_API rag_status rag_recompute_kv(const rag_kv_pool* pool, int32_t layer, const rag_batch* batch, int32_t k_cap,
                                    const void* plan, size_t plan_bytes, const void* x, int64_t x_rows,
                                    int32_t d_model, const void* w_k, const void* w_v, void* stream);

/* Synchronise `stream` and read the plan's counts: counts[0] selected tokens
 * recomputed, counts[1] private pages used, counts[2] private pages the
 * selection needs (optional, 3 int32, host). Returns RAG_OK or the most
 * severe of RAG_ERR_TIMEOUT, RAG_ERR_NO_FREE_PAGES, RAG_ERR_PAGE_OOB,
 * RAG_ERR_GEOMETRY. */
RAG_API rag_status rag_recompute_status(const void* plan, int32_t* counts, void* stream);

/* Synchronise `stream`, read and clear the workspace error word. Returns
 * RAG_OK when the device reported nothing, else the most severe of
 * RAG_ERR_TIMEOUT, RAG_ERR_PAGE_OOB, RAG_ERR_GEOMETRY, RAG_ERR_RANGE; *bits
 * (optional) receives the raw bits (1 page, 2 geometry, 4 timeout, 8 range). */
RAG_API rag_status rag_last_device_error(void* workspace, int32_t* bits, void* stream);

/* Self-test of the device-side failure detection (not a step of the method;
 * the pages have no counterpart). Launches one CTA on `stream` in which one
 * role waits on an mbarrier that nothing completes, with a limit of limit_ns
 * (1 .. 2e9 ns), while a second role waits on another such barrier with the
 * pipelines' full 2 s limit. The first wait runs out, records the timeout bit
 * (4) in *device_err (device int32, OR-ed in) and raises the CTA's abort flag;
 * the second role must then leave at once. The kernel therefore ends after
 * about limit_ns, never hangs, and leaves the context usable: this is the
 * mechanism every pipeline wait of the library uses to turn a stall into
 * RAG_ERR_TIMEOUT. */
RAG_API rag_status rag_selftest_wait_timeout(int32_t* device_err, int64_t limit_ns, void* stream);

/* Name of the last CUDA runtime error a call of this library met (the detail
 * behind a RAG_ERR_CUDA return), or "cudaSuccess". Host function. */
RAG_API const char* rag_last_cuda_error(void);

/* Kernel launches this library has made in this process (all entry points). */
RAG_API int64_t rag_launch_count(void);

/* Per-kernel timing: when enabled, every launch is bracketed by CUDA events
 * on its stream. rag_profile_collect synchronises, writes the summed device
 * milliseconds and launch counts per kernel kind (0 pool write, 1 attention,
 * 2 split combine, 3 impact, 4 top-k, 5 fp32 attention, 6 fp32 impact,
 * 7 recompute plan, 8 recompute page copy, 9 recompute projection,
 * 10 RoPE table, 11 KV decode, 12 attention of query blocks of at most 16
 * rows, e.g. decode steps) into
 * the first n_kinds entries of ms and launches (either may be NULL), and
 * resets the record. */
RAG_API void rag_profile_enable(int32_t on);
RAG_API rag_status rag_profile_collect(double* ms, int64_t* launches, int32_t n_kinds);

/* Like rag_profile_collect, but keeps the record. Launches recorded while a
 * stream was being captured into a CUDA graph become event nodes of the graph;
 * after each replay this reads that replay's per-kernel device times. */
RAG_API rag_status rag_profile_peek(double* ms, int64_t* launches, int32_t n_kinds);

#ifdef __cplusplus
}
#endif

#endif /* RAG_PREFILL_H_ */
