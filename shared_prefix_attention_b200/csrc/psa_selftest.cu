// Failure-detection self-test: exercises the bounded mbarrier wait that every
// kernel of the library uses, so a caller (or a test) can see the timeout
// path report PSA_ERR_TIMEOUT through the status word without any real
// kernel being starved.  Nothing here faults, traps or spins without limit.
#include <cuda_runtime.h>

#include "psa.h"
#include "psa_device.cuh"

namespace psa {
namespace {

// One warp.  Thread 0 initialises a barrier that expects one arrival and,
// when `arrive` is set, performs it.  Every thread then runs the bounded
// wait on that phase; the first thread to give up raises the CTA's abort
// flag and writes PSA_ERR_TIMEOUT, and the others return on seeing the flag.
__global__ void __launch_bounds__(32, 1) wait_selftest_kernel(int arrive, int32_t* dev_status) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncwarp();
  if (threadIdx.x == 0 && arrive) mbar_arrive(&bar);
  __syncwarp();
  const bool ok = mbar_wait(&bar, 0, &abort_flag, dev_status);
  // A wait that gave up must have left the CTA flagged and the status set.
  if (!ok && !abort_flag) report_status(dev_status, PSA_ERR_INVALID_ARG);
}

}  // namespace
}  // namespace psa

extern "C" int psa_wait_selftest(int32_t arrive, int32_t* dev_status, void* stream) {
  if (!dev_status) return PSA_ERR_INVALID_ARG;
  psa::wait_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(arrive != 0,
                                                                             dev_status);
  return cudaGetLastError() == cudaSuccess ? PSA_OK : PSA_ERR_CUDA;
}
