// common.cuh - small device helpers shared by the VDA kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace vda {

// Device error word of this library (per device).  Kernels that give up a
// bounded wait OR in an error code; vda_device_status() reads and clears it.
__device__ unsigned int g_device_error = 0u;

enum DeviceError : unsigned int {
  kErrWaitTimeout = 1u,   // an mbarrier / flag wait exceeded its iteration limit
};

__device__ __forceinline__ void raise_device_error(unsigned int code) {
  atomicOr(&g_device_error, code);
}

// Failure-detection self test: a flag that nothing ever sets, and a kernel
// whose single thread waits for it with the same kind of bounded poll the
// pipelines use.  The wait runs out after max_polls polls, records a wait
// time-out in the error word and the kernel returns normally, so the
// context stays usable.
__device__ int g_selftest_flag = 0;

__global__ void k_wait_selftest(long long max_polls) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  volatile int* flag = &g_selftest_flag;
  for (long long i = 0; i < max_polls; ++i) {
    if (*flag != 0) return;
    __nanosleep(128);
  }
  raise_device_error(kErrWaitTimeout);
}

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

__device__ __forceinline__ float sigmoidf_accurate(float x) { return 1.0f / (1.0f + expf(-x)); }

}  // namespace vda
