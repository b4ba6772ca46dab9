// selftest.cu -- a diagnostic kernel for the library's bounded waits.
//
// Every wait of the tensor-core kernels on an mbarrier phase is bounded: after a limit it sets
// DSA_DEVERR_TIMEOUT in the device error word and the kernel returns instead of hanging.  This
// kernel exercises that path on purpose, with a short limit: one thread initialises an mbarrier
// that nothing ever arrives on and waits for its first phase through the same bounded wait the
// kernels use.  The wait runs out after `limit_cycles` SM cycles, the error bit is set, and the
// kernel exits normally, leaving the context usable.
#include "common.cuh"
#include "internal.h"

namespace dsa {
namespace {

__global__ void bounded_wait_kernel(long long limit_cycles, int* err) {
  __shared__ uint64_t bar;
  if (threadIdx.x != 0) return;
  mbar_init(&bar, 1);
  fence_mbar_init();
  mbar_wait(&bar, 0, err, nullptr, limit_cycles);  // no thread arrives: this wait gives up
}

}  // namespace

cudaError_t launch_bounded_wait_selftest(long long limit_cycles, int* err, cudaStream_t s) {
  bounded_wait_kernel<<<1, 32, 0, s>>>(limit_cycles, err);
  return cudaGetLastError();
}

}  // namespace dsa
