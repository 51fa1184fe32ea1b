// Helpers of the SIMT (CUDA-core, float32) kernels: typed loads and stores of the storage
// dtype, the activation with its first and second derivatives, and the warp-per-row causal
// score product.
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

// One causal row of a score-like product, with a warp over the contraction, in segments of 32
// entries: kM of them, fully unrolled (for a row operand held in registers), or, with kM = 0,
// nm of them. a(m) gives this lane's entry lane + 32 m of the row operand and b(r, m) the
// matching entry of column r's operand (already weighted); both must return 0 past the end of
// the contraction. For each column r < ncol the warp sums the products with a butterfly; four
// columns go at once so that their reductions overlap. Lane u of each group of four hands
// column r + u to put(r + u, sum). Every lane of the warp must call it with the same ncol.
// Lanes read consecutive entries of one row at a time, so global loads are coalesced and
// shared-memory loads are free of bank conflicts.
template <int kM, typename Afn, typename Bfn, typename Put>
__device__ __forceinline__ void warp_row_dots(int nm, int ncol, Afn a, Bfn b, Put put) {
  const int lane = threadIdx.x & 31;
  for (int r = 0; r < ncol; r += 4) {
    int ru[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) ru[u] = min(r + u, ncol - 1);  // past the end: result unused
    float p[4] = {0.f, 0.f, 0.f, 0.f};
    auto segment = [&](int m) {
      const float av = a(m);
#pragma unroll
      for (int u = 0; u < 4; ++u) p[u] += av * b(ru[u], m);
    };
    if (kM > 0) {
#pragma unroll
      for (int m = 0; m < kM; ++m) segment(m);
    } else {
#pragma unroll 4
      for (int m = 0; m < nm; ++m) segment(m);
    }
#pragma unroll
    for (int o = 16; o; o >>= 1)
#pragma unroll
      for (int u = 0; u < 4; ++u) p[u] += __shfl_xor_sync(0xffffffffu, p[u], o);
    const float v = lane == 0 ? p[0] : lane == 1 ? p[1] : lane == 2 ? p[2] : p[3];
    if (lane < 4 && r + lane < ncol) put(r + lane, v);
  }
}

}  // namespace tttk
