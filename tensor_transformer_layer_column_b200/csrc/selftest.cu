// Failure-detection self-test: exercises the bounded-wait path that every
// kernel of the library uses, without faulting, trapping or hanging anything.
// One thread waits on an mbarrier that nothing will ever complete; the wait
// gives up after `limit_ns`, the thread records a code in the device error
// word and the kernel returns.  The host then reads the code back through
// tp_check_error (TP_ERR_TIMEOUT), exactly as after a real stalled wait.
#include <cuda_runtime.h>

#include "internal.h"
#include "sm100_ptx.cuh"
#include "tp_layer.h"

namespace tp {
namespace {

constexpr unsigned int ERR_SELFTEST_WAIT = 0x0F1;

__global__ void wait_timeout_kernel(uint64_t limit_ns, unsigned int* err) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0 && !mbar_wait(&bar, 0, limit_ns) && err != nullptr)
    atomicCAS(err, 0u, ERR_SELFTEST_WAIT);
}

}  // namespace
}  // namespace tp

extern "C" tp_status tp_selftest_wait_timeout(unsigned long long limit_ns, tp_stream stream) {
  if (limit_ns < 1000000ull || limit_ns > 10000000000ull) return TP_ERR_INVALID_ARG;
  unsigned int* err = tp::error_word();
  if (err == nullptr) return TP_ERR_CUDA;
  tp::wait_timeout_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(limit_ns, err);
  return tp::cuda_status(cudaGetLastError());
}
