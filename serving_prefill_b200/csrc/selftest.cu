// Self-test of the device-side failure detection that every pipeline of the
// library relies on: a bounded mbarrier wait that gives up, raises the CTA's
// abort flag and records a timeout in the error word, and a second role of
// the CTA that leaves its own wait as soon as it sees the flag. Nothing here
// faults or hangs: both waits end, by the limit or by the flag.
#include <cuda_runtime.h>

#include "rag_prefill.h"
#include "params.cuh"

namespace rag {

__global__ void __launch_bounds__(64, 1) wait_selftest_kernel(int32_t* err, uint64_t limit_ns) {
  __shared__ uint64_t never[2];   // barriers no thread ever arrives on
  __shared__ int abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(&never[0], 1);
    mbar_init(&never[1], 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  volatile int* abort = &abort_flag;
  if (lane == 0) {
    if (warp == 0) {
      // the short wait runs out: report it and tell the other role
      if (!mbar_wait_for(&never[0], 0, abort, limit_ns)) {
        atomicOr(err, kDevErrTimeout);
        *abort = 1;
      }
    } else {
      // the full-length wait ends on the abort flag, long before its limit
      mbar_wait(&never[1], 0, abort);
    }
  }
  __syncthreads();
}

}  // namespace rag

extern "C" RAG_API rag_status rag_selftest_wait_timeout(int32_t* device_err, int64_t limit_ns, void* stream) {
  if (!device_err || limit_ns <= 0 || limit_ns > int64_t(rag::kWaitLimitNs)) return RAG_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const cudaError_t e = rag::launch_plain(rag::wait_selftest_kernel, dim3(1), dim3(64), 0, s, device_err,
                                          uint64_t(limit_ns));
  rag::note_cuda_error(e);
  return e == cudaSuccess ? RAG_OK : RAG_ERR_CUDA;
}
