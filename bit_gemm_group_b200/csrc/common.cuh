// common.cuh -- device helpers shared by the libwq kernels (sm_100a only).
//
// * error recording into the library-owned device status word
// * numeric helpers (IEEE division, round-half-even, fp16/bf16 conversion)
// * launch-side helpers (grid sizing against the SM count)
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "wq.h"

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "libwq is written for sm_100a (B200) only"
#endif

namespace wq {

// Record the first device-side error: later errors do not overwrite it.
__device__ __forceinline__ void record_error(int* status, int code) {
  if (status != nullptr) atomicCAS(status, 0, code);
}

// One IEEE-754 binary32 division, round to nearest even.  The quantizers'
// codes are defined by this quotient bit for bit; their reciprocal-multiply
// fast paths reproduce it exactly and fall back to it near rounding
// boundaries.
__device__ __forceinline__ float div_rn(float a, float b) { return __fdiv_rn(a, b); }

// Round half to even on a float (numpy/torch `round` semantics).
__device__ __forceinline__ float round_even(float v) { return rintf(v); }

__device__ __forceinline__ float f16_round_trip(float v, unsigned short* bits) {
  __half h = __float2half_rn(v);
  *bits = __half_as_ushort(h);
  return __half2float(h);
}

template <typename T>
__device__ __forceinline__ float to_f32(T v);
template <>
__device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }
template <>
__device__ __forceinline__ float to_f32<__half>(__half v) { return __half2float(v); }

__device__ __forceinline__ uint32_t lane_id() {
  uint32_t l;
  asm volatile("mov.u32 %0, %%laneid;" : "=r"(l));
  return l;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_min(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fminf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

}  // namespace wq

// ---------------------------------------------------------------------------
// Host-side helpers (defined in wq_api.cu)
// ---------------------------------------------------------------------------
namespace wq_host {
// check (once per device) that the current device is sm_100 and set up the
// status word; WQ_OK or an error status
int ensure_device();
// device pointer of the status word on the current device
int* status_ptr();
// number of SMs of the current device
int sm_count();
// remember a CUDA error for wq_last_cuda_error(); returns WQ_ERR_CUDA
int cuda_fail(cudaError_t e, const char* where);
}  // namespace wq_host

#define WQ_CUDA_CHECK(expr)                                              \
  do {                                                                   \
    cudaError_t _e = (expr);                                             \
    if (_e != cudaSuccess) return wq_host::cuda_fail(_e, #expr);         \
  } while (0)

#define WQ_LAUNCH_CHECK(where)                                           \
  do {                                                                   \
    cudaError_t _e = cudaGetLastError();                                 \
    if (_e != cudaSuccess) return wq_host::cuda_fail(_e, where);         \
  } while (0)
