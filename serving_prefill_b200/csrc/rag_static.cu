// Fixed-scratch variant of the fused prefill entry point.
//
// Some callers cannot allocate device memory at all: a serving runtime that
// hands a plugin only its input and output buffers, an embedded deployment
// whose memory budget is planned once at start-up, or a latency-critical
// loop that must never block on an allocator. rag_fused_prefill_attn needs a
// caller-provided workspace; this variant instead uses one file-scope device
// array of kStaticScratchBytes. The array belongs to this library's device
// image, so every GPU on which it has been loaded keeps it until the process
// exits.
#include <cuda_runtime.h>

#include <mutex>

#include "rag_prefill.h"

namespace {

constexpr size_t kStaticScratchBytes = size_t(64) << 20;   // 64 MiB
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};   // device address of the array, per device

// The host-side name g_static_scratch is not a device address; look the real
// address up once per device, with that device current, and reuse it.
rag_status scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return RAG_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || p == nullptr) return RAG_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return RAG_OK;
}

}  // namespace

extern "C" RAG_API rag_status rag_fused_prefill_attn_static(const rag_kv_pool* pool, int32_t layer,
                                                            const rag_batch* batch, const void* q,
                                                            int32_t num_q_heads, const void* kq, const void* vq,
                                                            float sm_scale, void* o, float* row_lse, float* impact,
                                                            int32_t* device_err, void* stream) {
  const size_t need = rag_workspace_size(pool, batch, num_q_heads);
  if (need > kStaticScratchBytes) return RAG_ERR_WORKSPACE;
  void* scratch = nullptr;
  rag_status st = scratch_address(&scratch);
  if (st != RAG_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // The array keeps the previous call's contents; only the error word has to
  // start at zero (everything else is written before it is read).
  if (cudaMemsetAsync(scratch, 0, sizeof(int32_t), s) != cudaSuccess) return RAG_ERR_CUDA;
  st = rag_fused_prefill_attn(pool, layer, batch, q, num_q_heads, kq, vq, sm_scale, o, row_lse, impact, scratch,
                              kStaticScratchBytes, stream);
  if (st != RAG_OK) return st;
  if (device_err &&
      cudaMemcpyAsync(device_err, scratch, sizeof(int32_t), cudaMemcpyDeviceToDevice, s) != cudaSuccess)
    return RAG_ERR_CUDA;
  return RAG_OK;
}
