// Self-test of the bounded waits that every pipeline kernel of the library
// uses (no counterpart in the pages).  A wait on an mbarrier phase that never
// completes must give up after its poll limit, set the caller's abort flag
// and record its code in the error word -- instead of hanging the GPU -- and a
// wait on a phase that does complete must return without an error.
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/sa.h"
#include "sa_internal.h"
#include "tc_common.cuh"

namespace sa {
namespace {

constexpr int kTimedOutCode = 77;

__global__ void bounded_wait_probe_kernel(int* err, uint32_t limit) {
  __shared__ uint64_t never, once;
  __shared__ int abort_flag;
  if (threadIdx.x != 0) return;
  tc::mbar_init(&never, 1);
  tc::mbar_init(&once, 1);
  abort_flag = 0;
  tc::fence_barrier_init();
  // nothing ever arrives on `never`: the wait must run out
  const bool got = tc::mbar_wait(&never, 0, &abort_flag, err, kTimedOutCode, limit);
  err[2] = got ? 1 : 0;
  err[3] = abort_flag;
  // `once` completes its first phase: the wait must succeed without an error
  volatile int no_abort = 0;
  tc::mbar_arrive(&once);
  const bool ok = tc::mbar_wait(&once, 0, &no_abort, err + 1, kTimedOutCode + 1, limit);
  err[4] = ok ? 1 : 0;
}

}  // namespace
}  // namespace sa

extern "C" sa_status sa_self_test_bounded_wait(int32_t* err, uint32_t poll_limit, sa_stream_t stream) {
  if (err == nullptr || poll_limit == 0) {
    sa::set_last_error("err must be a device pointer to 5 int32 and poll_limit > 0");
    return SA_ERR_INVALID_ARG;
  }
  sa::bounded_wait_probe_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(err, poll_limit);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    sa::set_last_error("bounded-wait probe launch failed: %s", cudaGetErrorString(e));
    return SA_ERR_CUDA;
  }
  return SA_OK;
}
