// pkm_selftest.cu -- the failure path of the bounded waits, exercised
// without any GPU fault: one CTA waits on an mbarrier phase that nothing
// completes, using the same wait as the pipelined kernels
// (mbar_wait_or_abort) with a short poll limit.  The wait runs out, records
// PKM_ERR_TIMEOUT in the device status word and the kernel returns, so the
// context stays usable; *done tells the host that every thread got past
// the wait.
#include "common.cuh"
#include "kernels.h"

namespace pkm {

namespace {

__global__ void __launch_bounds__(32) wait_timeout_kernel(unsigned long long limit,
                                                          int32_t* status, int32_t* done) {
  __shared__ uint64_t bar;
  __shared__ volatile int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);  // one arrival expected; none comes
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  const bool got = mbar_wait_or_abort(&bar, 0, &abort_flag, status, limit);
  __syncthreads();
  if (threadIdx.x == 0) *done = got ? 2 : 1;
}

}  // namespace

}  // namespace pkm

using namespace pkm;

extern "C" {

PKM_API pkm_status pkm_check_wait_timeout(int64_t polls, int32_t* done, pkm_stream_t stream) {
  if (polls < 1 || polls > (int64_t(1) << 20) || !done ||
      (reinterpret_cast<uintptr_t>(done) & 3u))
    return PKM_ERR_INVALID_ARG;
  int32_t* status = status_ptr();
  if (!status) return PKM_ERR_CUDA;
  wait_timeout_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      (unsigned long long)polls, status, done);
  note_launch();
  return cudaGetLastError() == cudaSuccess ? PKM_OK : PKM_ERR_CUDA;
}

}  // extern "C"
