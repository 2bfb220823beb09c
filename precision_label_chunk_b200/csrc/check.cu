// check.cu -- a check of the library's failure detection that faults nothing.
//
// Every pipelined kernel waits on mbarriers through tc::mbar_wait, which gives
// up after a cycle limit; the kernel then records ELMO_ETIMEOUT in its status
// word and winds down.  wait_check_kernel runs that same wait on a barrier
// nothing ever arrives on, so the give-up path runs for real.
#include "elmo_common.cuh"
#include "elmo_internal.h"
#include "tc_ptx.cuh"

namespace elmo {
namespace {

__global__ void wait_check_kernel(long long limit_cycles, int32_t* __restrict__ status) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    tc::mbar_init(&bar, 1);
    abort_flag = 0;
    tc::fence_barrier_init();
  }
  __syncthreads();
  volatile int* abort = &abort_flag;
  if (threadIdx.x == 0 && !tc::mbar_wait(&bar, 0, abort, limit_cycles)) {
    *abort = 1;
    if (atomicCAS(status, 0, (int)ELMO_ETIMEOUT) == 0) status[1] = ELMO_WAIT_CHECK_SITE;
  }
}

}  // namespace

cudaError_t launch_wait_check(long long limit_cycles, int32_t* status, cudaStream_t s) {
  cudaError_t e = cudaMemsetAsync(status, 0, 2 * sizeof(int32_t), s);
  if (e != cudaSuccess) return e;
  wait_check_kernel<<<1, 32, 0, s>>>(limit_cycles, status);
  return cudaGetLastError();
}

}  // namespace elmo
