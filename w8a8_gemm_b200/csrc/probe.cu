// probe.cu -- test-only kernels for the library's failure reporting.  The
// timeout probe waits on an mbarrier that nothing ever arrives on, with the
// same bounded wait the GEMM and quantize kernels use, and records the timeout
// in the device error word: the path a real stall would take (give up, report,
// return), without faulting or hanging the GPU.  The bounds probe (debug build
// only) stores through the checked path to an index one past the extent it
// names, inside a buffer that has that extra element, and the check records
// the store it skipped.
#include <cuda_runtime.h>
#include <stdint.h>

#include "sm100.cuh"
#include "sq_internal.h"

namespace sq {
namespace {

__global__ void timeout_probe_kernel(uint64_t limit_ns, int *status) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  // Phase 0 never completes: no thread arrives on `bar`.
  const bool done = mbar_wait(&bar, 0, limit_ns);
  if (!done && threadIdx.x == 0) atomicExch(status, static_cast<int>(SQ_ERR_DEVICE_TIMEOUT));
}

__global__ void bounds_probe_kernel(int32_t *buf, int64_t n, int *status) {
  const int64_t i = n;  // one past the extent the check is given
  if (store_ok(status, i >= 0 && i < n)) buf[i] = -1;
}

}  // namespace

cudaError_t launch_bounds_probe(int32_t *buf, int64_t n, int *status, cudaStream_t stream) {
  bounds_probe_kernel<<<1, 1, 0, stream>>>(buf, n, status);
  return cudaGetLastError();
}

cudaError_t launch_timeout_probe(uint32_t limit_us, int *status, cudaStream_t stream) {
  timeout_probe_kernel<<<1, 32, 0, stream>>>(static_cast<uint64_t>(limit_us) * 1000u, status);
  return cudaGetLastError();
}

}  // namespace sq
