// Scalar helpers of the SIMT (CUDA-core, float32) kernels: typed loads and stores of the
// storage dtype, and the activation with its first and second derivatives.
#pragma once
#include <cuda_bf16.h>
#include <math.h>

namespace tttk {

__device__ __forceinline__ float ldf(const float* p) { return *p; }
__device__ __forceinline__ float ldf(const __nv_bfloat16* p) { return __bfloat162float(*p); }
__device__ __forceinline__ void stf(float* p, float v) { *p = v; }
__device__ __forceinline__ void stf(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }

__device__ __forceinline__ float sigm(float x) { return 1.f / (1.f + expf(-x)); }
// act = 0: identity; act = 1: SiLU(z) = z sigmoid(z)
__device__ __forceinline__ float actf(int act, float z) { return act ? z * sigm(z) : z; }
__device__ __forceinline__ float act1(int act, float z) {
  if (!act) return 1.f;
  const float s = sigm(z);
  return s * (1.f + z * (1.f - s));
}
__device__ __forceinline__ float act2(int act, float z) {
  if (!act) return 0.f;
  const float s = sigm(z);
  return s * (1.f - s) * (2.f + z * (1.f - 2.f * s));
}

}  // namespace tttk
