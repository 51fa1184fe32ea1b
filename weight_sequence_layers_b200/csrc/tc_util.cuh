// Epilogue helpers shared by the tcgen05 TTT kernels: activations, 32-element row moves
// between registers and 128B-swizzled shared-memory panels, and the per-chunk scans of the
// learning rate and the log decay.
#pragma once
#include <cuda_bf16.h>

#include "common.cuh"

namespace tttk {
namespace {

__device__ __forceinline__ float sigm(float x) { return 1.f / (1.f + __expf(-x)); }
__device__ __forceinline__ float act_f(int act, float z) { return act ? z * sigm(z) : z; }
__device__ __forceinline__ float act_d1(int act, float z) {
  if (!act) return 1.f;
  const float s = sigm(z);
  return s * (1.f + z * (1.f - s));
}

// Reads 32 bf16 (16-byte chunks c0..c0+3 of `row`) of a swizzled panel as floats.
__device__ __forceinline__ void ld_row32(uint32_t panel, int row, int c0, float (&x)[32]) {
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    uint32_t a, b, c, d;
    ld_shared_v4(panel + sw128_off(row, c0 + k), a, b, c, d);
    x[8 * k + 0] = bf16lo(a); x[8 * k + 1] = bf16hi(a);
    x[8 * k + 2] = bf16lo(b); x[8 * k + 3] = bf16hi(b);
    x[8 * k + 4] = bf16lo(c); x[8 * k + 5] = bf16hi(c);
    x[8 * k + 6] = bf16lo(d); x[8 * k + 7] = bf16hi(d);
  }
}
__device__ __forceinline__ void st_row32(uint32_t panel, int row, int c0, const float (&x)[32]) {
#pragma unroll
  for (int k = 0; k < 4; ++k)
    st_shared_v4(panel + sw128_off(row, c0 + k), pack_bf16x2(x[8 * k], x[8 * k + 1]),
                 pack_bf16x2(x[8 * k + 2], x[8 * k + 3]), pack_bf16x2(x[8 * k + 4], x[8 * k + 5]),
                 pack_bf16x2(x[8 * k + 6], x[8 * k + 7]));
}
__device__ __forceinline__ void st_global_bf16x32(__nv_bfloat16* dst, const float (&x)[32]) {
  uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int k = 0; k < 4; ++k)
    d[k] = make_uint4(pack_bf16x2(x[8 * k], x[8 * k + 1]), pack_bf16x2(x[8 * k + 2], x[8 * k + 3]),
                      pack_bf16x2(x[8 * k + 4], x[8 * k + 5]),
                      pack_bf16x2(x[8 * k + 6], x[8 * k + 7]));
}


// Per-chunk scans by one warp (C = 32 * PER tokens starting at tok0):
//   eta_r = 2 sigmoid(beta_r + b), L_r = sum_{t<=r} log gamma_t (chunk-local),
//   gam_r = exp(L_r), eLC_r = exp(L_C - L_r),
//   cfac_r  = eta_r exp(L_{last of r's 64-group} - L_r)   (<= eta_r),
//   cfacT_r = exp(L_r - L_{first of r's 64-group})         (<= 1).
// Every exponent is <= 0: no 1/Gamma is formed, strong decay underflows to 0 instead.
template <int C>
__device__ __forceinline__ void chunk_scan_warp(const float* beta, const float* gamma, size_t tok0,
                                                float lr_bias, float* eta, float* L, float* gam,
                                                float* eLC, float* cfac, float* cfacT) {
  constexpr int PER = C / 32;
  const int lane = threadIdx.x & 31;
  float lg[PER];
  float run = 0.f;
#pragma unroll
  for (int k = 0; k < PER; ++k) {
    const int r = lane * PER + k;
    run += gamma ? __logf(gamma[tok0 + r]) : 0.f;
    lg[k] = run;
    eta[r] = 2.f * sigm(beta[tok0 + r] + lr_bias);
  }
  float incl = run;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const float o = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += o;
  }
  const float excl = incl - run;
  const float LC = __shfl_sync(0xffffffffu, incl, 31);
#pragma unroll
  for (int k = 0; k < PER; ++k) L[lane * PER + k] = lg[k] + excl;
  __syncwarp();
#pragma unroll
  for (int k = 0; k < PER; ++k) {
    const int r = lane * PER + k;
    const float Lr = L[r];
    gam[r] = __expf(Lr);
    eLC[r] = __expf(LC - Lr);
    cfac[r] = eta[r] * __expf(L[r | 63] - Lr);
    cfacT[r] = __expf(Lr - L[r & ~63]);
  }
  __syncwarp();
}

// 32 consecutive floats -> 16 packed bf16 pairs (even index in the low half).
__device__ __forceinline__ void pack32(const float (&x)[32], uint32_t (&w)[16]) {
#pragma unroll
  for (int j = 0; j < 16; ++j) w[j] = pack_bf16x2(x[2 * j], x[2 * j + 1]);
}

}  // namespace
}  // namespace tttk
