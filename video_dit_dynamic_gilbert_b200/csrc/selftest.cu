// Test hook for failure detection: the bounded mbarrier wait every kernel uses, on a
// barrier that nothing ever arrives at, so that the wait must give up, record its
// expiry in the device error word and return (no trap, no hang, the context stays
// usable).  Not part of the attention path; nothing in it is called by the other
// entry points.
#include "common.cuh"
#include "internal.h"
#include "tc.cuh"

namespace asa {
namespace {

constexpr unsigned int kErrSelftest = 16u;

__global__ void wait_timeout_kernel(unsigned int* __restrict__ err_word, long long limit) {
  __shared__ __align__(8) unsigned long long bar;
  const uint32_t b = smem_u32(&bar);
  if (threadIdx.x == 0) {
    tc::mbar_init(b, 1);
    tc::fence_barrier_init();
  }
  __syncthreads();
  const bool ok = tc::mbar_wait(b, 0, limit);  // no arrive is ever made on `bar`
  if (!ok && threadIdx.x == 0) atomicOr(err_word, kErrSelftest);
}

}  // namespace

cudaError_t launch_wait_timeout(unsigned int* err_word, long long limit, cudaStream_t stream) {
  wait_timeout_kernel<<<1, 32, 0, stream>>>(err_word, limit);
  return cudaGetLastError();
}

}  // namespace asa
