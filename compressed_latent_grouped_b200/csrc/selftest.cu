// Self-test of the failure reporting every kernel of this library relies on:
// a bounded mbarrier wait that runs out sets CCGQA_DEVERR_TIMEOUT and returns,
// instead of hanging the GPU.  The kernel waits on a barrier nothing arrives
// on, with a caller-chosen short limit, through the same mbar_wait the
// attention, projection and pre-attention kernels use.
#include "kernels.h"
#include "sm100.cuh"

namespace ccgqa {
namespace {

using namespace sm100;

__global__ void wait_timeout_kernel(int32_t* dev_err, long long limit) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  // nobody arrives: every thread's wait gives up (after `limit` cycles, or at
  // once when another thread of the block already has)
  mbar_wait(&bar, 0, &abort_flag, dev_err, limit);
}

}  // namespace
}  // namespace ccgqa

extern "C" __attribute__((visibility("default"))) ccgqa_status ccgqa_selftest_wait_timeout(
    int64_t limit_cycles, int32_t* dev_err, void* stream) {
  if (limit_cycles < 1 || limit_cycles > ccgqa::kWaitLimitCycles) return CCGQA_ERR_INVALID_ARG;
  if (!ccgqa::stream_allowed(static_cast<cudaStream_t>(stream))) return CCGQA_ERR_INVALID_ARG;
  ccgqa::wait_timeout_kernel<<<1, 64, 0, static_cast<cudaStream_t>(stream)>>>(
      dev_err, static_cast<long long>(limit_cycles));
  ccgqa::count_launches(1);
  return cudaGetLastError() == cudaSuccess ? CCGQA_OK : CCGQA_ERR_CUDA;
}
