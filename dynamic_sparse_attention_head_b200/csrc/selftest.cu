// Failure-detection self-test: a bounded wait that runs out.  Every pipeline wait of the
// library's kernels is an mbarrier wait bounded by the global timer (mbar_wait): on expiry the
// waiting thread raises the CTA's abort flag, the CTA unwinds without trapping, and the
// timeout is recorded in the workspace's status word for msa_device_status.  This kernel makes
// one such wait expire on purpose (a barrier no thread arrives at) and records it the same way,
// so that the reporting path can be checked on a GPU without a hang or a fault.
#include <cuda_runtime.h>
#include <stdint.h>

#include "kernels.h"
#include "msa_internal.h"
#include "ptx.cuh"

namespace msa {

namespace {

__global__ void wait_probe_kernel(uint32_t* status, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);  // expects one arrival, which never comes
    abort = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0 && !mbar_wait(&bar, 0, &abort, limit_ns)) atomicOr(status, DEV_ERR_TIMEOUT);
  __syncthreads();
}

}  // namespace

cudaError_t launch_wait_probe(uint32_t* status, uint64_t limit_ns, cudaStream_t st) {
  count_launches(1);
  wait_probe_kernel<<<1, 32, 0, st>>>(status, limit_ns);
  return cudaGetLastError();
}

}  // namespace msa
