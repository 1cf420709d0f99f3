// Self-test of the bounded waits every kernel of the library relies on: a
// kernel waits on an mbarrier that nothing ever arrives on, through the same
// bounded-wait helper, and must give up after its limit (about a second),
// report PYR_ETIMEOUT in the status word and return, leaving the context
// usable. No fault, trap or unbounded loop is involved.
#include "pyr_common.cuh"
#include "tc_util.cuh"

namespace pyr {
namespace {

__global__ void wait_selftest_kernel(int* status) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    tc::mbar_init(&bar, 1);
    tc::fence_mbar_init();
    abort_flag = 0;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const bool ok = tc::mbar_wait(&bar, 0, (volatile int*)&abort_flag);  // no arrival ever comes
    if (!ok) report(status, PYR_ETIMEOUT);
  }
  __syncthreads();
}

}  // namespace
}  // namespace pyr

extern "C" int pyr_selftest_wait(int* dev_status, void* stream) {
  if (!dev_status) return PYR_EINVAL;
  pyr::wait_selftest_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(dev_status);
  return cudaGetLastError() == cudaSuccess ? PYR_OK : PYR_ECUDA;
}
