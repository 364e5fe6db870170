// Shared device/host helpers for the CCGQA kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/ccgqa.h"

namespace ccgqa {

// Element conversions used by every templated kernel.
__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }
template <typename T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}

// OR an error bit into the caller's device status word (nullable).
__device__ __forceinline__ void raise_dev_err(int32_t* dev_err, int32_t bit) {
  if (dev_err) atomicOr(dev_err, bit);
}

// Cycles a bounded in-kernel wait may spin before it gives up (about one
// second at the B200's clock).  A healthy wait ends in microseconds.
constexpr long long kWaitLimitCycles = 2000000000LL;

// Host-side launch accounting (ccgqa_launch_count); while the calling thread
// records a graph the kernels count towards the graph instead.
void count_launches(int n);
// False while the calling thread records a graph on a stream other than st.
bool stream_allowed(cudaStream_t st);

// cudaFuncSetAttribute(func, MaxDynamicSharedMemorySize, bytes) on the current
// device, skipped when an earlier call already allowed at least `bytes`
// (the attribute is per device, the check costs a lock and a map lookup).
cudaError_t allow_smem(const void* func, int bytes);

// Streaming multiprocessors of the current device (looked up once per device;
// 148, a B200's count, when no device answers, e.g. for a workspace-size query
// on a machine without one).
int sm_count();

// Programmatic dependent launch.  A kernel launched by launch_pdl may be
// scheduled while the kernel before it on the stream is still finishing (once
// every CTA of that kernel has run pdl_trigger() or exited).  Every such kernel
// runs pdl_wait() in all its threads as its first statement: the wait returns
// when the previous kernel has completed and its memory writes are visible, so
// nothing (global memory, TMEM) is touched before it.  The overlap gained is
// the launch and CTA scheduling of this kernel during the previous one's tail.
// Kernels launched without the attribute see pdl_wait() return at once.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
// Both in one call: the first statement of every kernel launched by launch_pdl.
__device__ __forceinline__ void pdl_enter() {
  pdl_wait();
  pdl_trigger();
}

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<Args&&>(args)...);
}

}  // namespace ccgqa
