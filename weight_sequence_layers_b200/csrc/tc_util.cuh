// Epilogue helpers shared by the tcgen05 TTT kernels: activations, 32-element row moves
// between registers and 128B-swizzled shared-memory panels, and the per-chunk scans of the
// learning rate and the log decay.
#pragma once
#include <cuda_bf16.h>

#include "common.cuh"

namespace tttk {
namespace {

// Sigmoid with the hardware exponential and the fast approximate division (bf16-level
// accuracy is enough here; 1 + exp(-x) above 2^126 gives 0, the right limit).
__device__ __forceinline__ float sigm(float x) { return __fdividef(1.f, 1.f + __expf(-x)); }

// Activation of the fast-weight network (ACT = 0 identity, 1 SiLU) and its derivative; a
// compile-time choice so the identity path carries no transcendental at all.
template <int ACT>
__device__ __forceinline__ float act_f(float z) {
  if constexpr (ACT == 1) return z * sigm(z);
  return z;
}
// act(z) and act'(z) from one sigmoid.
template <int ACT>
__device__ __forceinline__ void act_both(float z, float& f, float& d1) {
  if constexpr (ACT == 1) {
    const float s = sigm(z);
    f = z * s;
    d1 = s * (1.f + z * (1.f - s));
  } else {
    f = z;
    d1 = 1.f;
  }
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
//   cF16_r = eta_r exp(L_{r16} - L_r) and cT16_r = exp(L_r - L_{r16}) with r16 = r & ~15.
// beta and gamma may point to global or shared memory (gamma NULL: no decay).
template <int C>
__device__ __forceinline__ void chunk_scan_warp(const float* beta, const float* gamma, float lr_bias,
                                                float* eta, float* L, float* gam, float* eLC,
                                                float* cF16, float* cT16) {
  constexpr int PER = C / 32;
  const int lane = threadIdx.x & 31;
  float lg[PER];
  float run = 0.f;
#pragma unroll
  for (int k = 0; k < PER; ++k) {
    const int r = lane * PER + k;
    run += gamma ? __logf(gamma[r]) : 0.f;
    lg[k] = run;
    eta[r] = 2.f * sigm(beta[r] + lr_bias);
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
    const float Lr = L[r], L16 = L[r & ~15];
    gam[r] = __expf(Lr);
    eLC[r] = __expf(LC - Lr);
    cF16[r] = eta[r] * __expf(L16 - Lr);
    cT16[r] = __expf(Lr - L16);
  }
  __syncwarp();
}

// -S for one query s (chunk-local) against 32 keys r0.. (r0 % 32 == 0), packed to bf16 pairs:
//   S_sr = P_sr eta_r exp(L_s - L_r) = P_sr exp(L_s - L_{r16}) cF16_r,  r16 = r & ~15,
// with one exponential per 16 keys. MASK: some keys lie after s and are zeroed.
template <bool MASK>
__device__ __forceinline__ void score_weights32(const float (&pv)[32], const float* Lv,
                                                const float* cF16, int s, float Ls, int r0,
                                                uint32_t (&pk)[16]) {
#pragma unroll
  for (int g16 = 0; g16 < 2; ++g16) {
    const int r16 = r0 + 16 * g16;
    float a = -__expf(Ls - Lv[r16]);
    if (MASK && s < r16) a = 0.f;
    const float4* c4 = reinterpret_cast<const float4*>(cF16 + r16);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float4 cf = c4[k];
      const int j = 16 * g16 + 4 * k;
      float x0 = pv[j] * cf.x * a, x1 = pv[j + 1] * cf.y * a;
      float x2 = pv[j + 2] * cf.z * a, x3 = pv[j + 3] * cf.w * a;
      if (MASK) {
        const int r = r16 + 4 * k;
        if (r > s) x0 = 0.f;
        if (r + 1 > s) x1 = 0.f;
        if (r + 2 > s) x2 = 0.f;
        if (r + 3 > s) x3 = 0.f;
      }
      pk[8 * g16 + 2 * k] = pack_bf16x2(x0, x1);
      pk[8 * g16 + 2 * k + 1] = pack_bf16x2(x2, x3);
    }
  }
}

// -dP^T for one key r (chunk-local) against 32 queries s0.. (s0 % 32 == 0), packed to bf16:
//   M^T_rs = eta_r exp(L_s - L_r) = eta_r exp(L_{s16} - L_r) cT16_s,  s16 = s & ~15,
// for s >= r, with one exponential per 16 queries. MASK: some queries precede r.
template <bool MASK>
__device__ __forceinline__ void score_weights32_k(const float (&pv)[32], const float* Lv,
                                                  const float* cT16, int r, float Lr, float er,
                                                  int s0, uint32_t (&pk)[16]) {
#pragma unroll
  for (int g16 = 0; g16 < 2; ++g16) {
    const int s16 = s0 + 16 * g16;
    float a = -er * __expf(Lv[s16] - Lr);
    if (MASK && s16 + 15 < r) a = 0.f;
    const float4* c4 = reinterpret_cast<const float4*>(cT16 + s16);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float4 cf = c4[k];
      const int j = 16 * g16 + 4 * k;
      float x0 = pv[j] * cf.x * a, x1 = pv[j + 1] * cf.y * a;
      float x2 = pv[j + 2] * cf.z * a, x3 = pv[j + 3] * cf.w * a;
      if (MASK) {
        const int s = s16 + 4 * k;
        if (s < r) x0 = 0.f;
        if (s + 1 < r) x1 = 0.f;
        if (s + 2 < r) x2 = 0.f;
        if (s + 3 < r) x3 = 0.f;
      }
      pk[8 * g16 + 2 * k] = pack_bf16x2(x0, x1);
      pk[8 * g16 + 2 * k + 1] = pack_bf16x2(x2, x3);
    }
  }
}

// Causal weights of a query row s against 32 keys of key half idx (r = rbase + 32 idx + j):
// -S or -dP packed to bf16. A half is entirely unmasked when its keys precede the warp's rows.
struct QWeights {
  const float *L, *cF16;
  int s, rbase;
  float Ls;
  __device__ bool full(int idx, int q) const { return idx < q; }
  __device__ void operator()(const float (&pv)[32], int idx, bool mask, uint32_t (&pk)[16]) const {
    if (mask) score_weights32<true>(pv, L, cF16, s, Ls, rbase + 32 * idx, pk);
    else score_weights32<false>(pv, L, cF16, s, Ls, rbase + 32 * idx, pk);
  }
};
// The same for a key row r against 32 queries of query half idx (s = sbase + 32 idx + j):
// -S^T or -dP^T. A half is entirely unmasked when its queries follow the warp's rows.
struct KWeights {
  const float *L, *cT16;
  int r, sbase;
  float Lr, er;
  __device__ bool full(int idx, int q) const { return idx > q; }
  __device__ void operator()(const float (&pv)[32], int idx, bool mask, uint32_t (&pk)[16]) const {
    if (mask) score_weights32_k<true>(pv, L, cT16, r, Lr, er, sbase + 32 * idx, pk);
    else score_weights32_k<false>(pv, L, cT16, r, Lr, er, sbase + 32 * idx, pk);
  }
};

// In-place packing of a 128-column fp32 score block held in TMEM by the thread's row (tb =
// TMEM address of the row's column 0). Column pair p (64 columns [64p, 64p+64), halves
// idx = 2p, 2p+1) becomes 32 bf16-pair columns at [OUT p, OUT p + 32); every column is read
// before the same thread overwrites it. With OUT = 32 the packed block is contiguous (the MMA
// reading it as A takes K-step j at 8 j); with OUT = 64 each warpgroup packs inside its own
// 64 columns (K-step j at 64 (j / 4) + 8 (j % 4)). Halves are classified per warp (q = TMEM
// lane quadrant = rows [32q, 32q+32) of the block): on a diagonal block a half is the warp's
// own diagonal, entirely unmasked or entirely masked (written as zeros without a load).
template <int OUT, typename F>
__device__ __forceinline__ void pack_in_place(uint32_t tb, int p0, int p1, int q, bool diag,
                                              const F& weights) {
  for (int pair = p0; pair < p1; ++pair) {
    int kind[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int idx = 2 * pair + h;
      kind[h] = diag ? (idx == q ? 2 : weights.full(idx, q) ? 1 : 0) : 1;
    }
    float pv[2][32];
#pragma unroll
    for (int h = 0; h < 2; ++h)
      if (kind[h] != 0) tmem_ld32(tb + 64 * pair + 32 * h, pv[h]);
    tmem_wait_ld();
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint32_t pk[16];
      if (kind[h] == 0) {
#pragma unroll
        for (int j = 0; j < 16; ++j) pk[j] = 0u;
      } else {
        weights(pv[h], 2 * pair + h, kind[h] == 2, pk);
      }
      tmem_st16u(tb + OUT * pair + 16 * h, pk);
    }
  }
}
// TMEM column of K-step j (16 keys) of a block packed by pack_in_place<OUT>.
template <int OUT>
__host__ __device__ constexpr uint32_t packed_col(int j) {
  return OUT == 32 ? 8 * j : 64 * (j / 4) + 8 * (j % 4);
}

// Bulk copy of `bytes` (multiple of 16, 16-byte aligned) from global to shared memory,
// completing on `bar`.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
      : "memory");
}

}  // namespace
}  // namespace tttk
