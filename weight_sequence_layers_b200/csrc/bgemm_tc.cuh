// Batched tcgen05 GEMM with a fused epilogue: for every batch b (grid y) and 128-row tile m0
// (grid x),
//   D[b][m0 .. m0+127][0 .. N) = sum over terms t of A_t[b] B_t[b]       (bf16 in, fp32 in TMEM)
// and the epilogue functor sees each row of D, 32 columns at a time. A_t is always K-major
// (rows = M, contiguous along K); B_t is K-major (N rows, contiguous along K) or, with N = 64,
// MN-major (rows = K, contiguous along N). Operands arrive by 3-D TMA (inner, rows, batch), 64
// K-elements per stage, and the MMA is issued by one thread (M = 128, N = 64..256).
//
// Warp roles: 0 TMA producer, 1 MMA issue, 2-5 epilogue (one accumulator row per thread).
// Every wait is bounded; a wait that runs out records the timeout and the CTA skips its work.
#pragma once
#include <cuda_bf16.h>

#include "common.cuh"

namespace tttk {
namespace bg {

constexpr int kThreads = 192;

struct Term {
  int K;              // contraction length, a multiple of 64
  int a_k0, a_row;    // A: inner coordinate of K = 0 and row of the tile's first row (+ m0)
  int b_k0, b_row;    // B K-major: inner of K = 0, first of the N rows; MN-major: b_row = row
                      // of K = 0
};
struct Prob {
  int nterm;          // 0: the epilogue sees zeros
  Term t[3];
};

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* m, uint32_t bar,
                                            int c0, int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cta.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(bar), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

template <int N>
struct Layout {
  static constexpr uint32_t A_BYTES = 128 * 128;
  static constexpr uint32_t BK_BYTES = N * 128;   // K-major B: N rows x 64 K
  static constexpr uint32_t BM_BYTES = 64 * 128;  // MN-major B (N = 64): 64 K rows x 64 N
  static constexpr uint32_t B_BYTES = BK_BYTES > BM_BYTES ? BK_BYTES : BM_BYTES;
  static constexpr uint32_t STAGE = A_BYTES + B_BYTES;
  static constexpr int STAGES = N == 256 ? 2 : N == 128 ? 3 : 4;
  static constexpr uint32_t OFF_BAR = STAGES * STAGE;
};
struct __align__(8) Bars {
  uint64_t full[4], empty[4], acc;
  uint32_t tmem_base;
  int abort_flag;
};
template <int N>
constexpr size_t smem_bytes() { return Layout<N>::OFF_BAR + sizeof(Bars) + 1024; }

template <int N, int MN0, int MN1, int MN2, typename Epi>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap a0, const __grid_constant__ CUtensorMap b0,
                const __grid_constant__ CUtensorMap a1, const __grid_constant__ CUtensorMap b1,
                const __grid_constant__ CUtensorMap a2, const __grid_constant__ CUtensorMap b2,
                const Prob pr, const Epi epi, unsigned* err) {
  static_assert(N == 64 || N == 128 || N == 256, "N");
  static_assert((!MN0 && !MN1 && !MN2) || N == 64, "an MN-major B is 64 wide");
  using L = Layout<N>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  Bars* bars = reinterpret_cast<Bars*>(smem + L::OFF_BAR);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int m0 = blockIdx.x * 128, b = blockIdx.y;
  Abort ab{&bars->abort_flag, err};
  auto sA = [&](int s) { return sb + s * L::STAGE; };
  auto sB = [&](int s) { return sb + s * L::STAGE + L::A_BYTES; };
  if (threadIdx.x == 0) {
    for (int s = 0; s < L::STAGES; ++s) {
      mbar_init(smem_u32(&bars->full[s]), 1);
      mbar_init(smem_u32(&bars->empty[s]), 1);
    }
    mbar_init(smem_u32(&bars->acc), 1);
    bars->abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&bars->tmem_base), N);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 0) {
    if (lane == 0) {
      int it = 0;
#pragma unroll
      for (int t = 0; t < 3; ++t) {
        if (t >= pr.nterm) break;
        const CUtensorMap* A = t == 0 ? &a0 : t == 1 ? &a1 : &a2;
        const CUtensorMap* B = t == 0 ? &b0 : t == 1 ? &b1 : &b2;
        const bool mn = t == 0 ? MN0 : t == 1 ? MN1 : MN2;
        const Term tm = pr.t[t];
        bool ok = true;
        for (int k = 0; k < tm.K; k += 64, ++it) {
          const int s = it % L::STAGES;
          if (it >= L::STAGES &&
              !(ok = mbar_wait(smem_u32(&bars->empty[s]), ((it / L::STAGES) - 1) & 1, ab)))
            break;
          const uint32_t full = smem_u32(&bars->full[s]);
          mbar_arrive_expect_tx(full, L::A_BYTES + (mn ? L::BM_BYTES : L::BK_BYTES));
          tma_load_3d(sA(s), A, full, tm.a_k0 + k, tm.a_row + m0, b);
          if (mn)
            tma_load_3d(sB(s), B, full, 0, tm.b_row + k, b);
          else
            tma_load_3d(sB(s), B, full, tm.b_k0 + k, tm.b_row, b);
        }
        if (!ok) break;
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      int it = 0;
      bool ok = true;
#pragma unroll
      for (int t = 0; t < 3; ++t) {
        if (t >= pr.nterm || !ok) break;
        const bool mn = t == 0 ? MN0 : t == 1 ? MN1 : MN2;
        const uint32_t id = idesc_bf16(128, N, 0, mn ? 1 : 0);
        for (int k = 0; k < pr.t[t].K; k += 64, ++it) {
          const int s = it % L::STAGES;
          if (!(ok = mbar_wait(smem_u32(&bars->full[s]), (it / L::STAGES) & 1, ab))) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16_ss(tmem, sdesc_sw128(sA(s) + kk * 32, 16, 1024),
                        mn ? sdesc_sw128(sB(s) + kk * 2048, 0, 1024)
                           : sdesc_sw128(sB(s) + kk * 32, 16, 1024),
                        id, it > 0 || kk > 0);
          mma_commit(smem_u32(&bars->empty[s]));
        }
      }
      mma_commit(smem_u32(&bars->acc));
    }
  } else {
    const int q = warp & 3;
    const int lrow = q * 32 + lane;
    const uint32_t loff = (uint32_t)(q * 32) << 16;
    if (mbar_wait(smem_u32(&bars->acc), 0, ab)) {
      __syncwarp();
      tc_fence_after();
      auto st = epi.begin(b, m0 + lrow);
#pragma unroll 1
      for (int c32 = 0; c32 < N / 32; ++c32) {
        float v[32];
        if (pr.nterm) {
          tmem_ld32(tmem + loff + 32 * c32, v);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = 0.f;
        }
        epi.chunk(st, 32 * c32, v);
      }
      epi.end(st);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (bars->abort_flag) __nanosleep(100000);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, N);
  }
}

}  // namespace bg
}  // namespace tttk
