// la_common.cuh -- small device helpers shared by the kernel files.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace la {

// Feature map of "1.6 长上下文与高效注意力", section 线性注意力: phi(x) = elu(x) + 1
// with elu's alpha = 1, i.e. x + 1 for x > 0 and exp(x) otherwise; or the identity.
__device__ __forceinline__ float feature_map(float x, int phi) {
  if (phi) return x > 0.f ? x + 1.f : expf(x);
  return x;
}

template <typename T>
__device__ __forceinline__ float to_f32(T x);
template <>
__device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T>
__device__ __forceinline__ T from_f32(float x);
template <>
__device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

// Decay powers gamma^n.  powf(g, 0) is 1 for every g (including 0), which is
// the diagonal of the decay mask.
__device__ __forceinline__ float decay_pow(float g, int n) { return powf(g, (float)n); }

}  // namespace la
