// In-Place TTT forward of the W_down fast weight on sm_100a tensor cores.
//
// Page "In-Place Test-Time Training", section "核心方法和技术细节": W_down of a gated MLP
// is the fast weight; the sequence is cut into chunks of C tokens and every chunk first
// applies the current weight, O_[i] = Z_[i] W^(i)T, then updates it with the chunk's
// inner-product gradient, W^(i+1) = W^(i) + eta Vhat_[i]^T Z_[i].
//
// One launch per chunk i runs both GEMMs of that chunk from a shared dynamic tile queue:
//   apply  tiles: O_i[128 tokens x 256 d_model] = Z_i (K-major) x Wb_i^T (K-major), K = d_ff
//   update tiles: W[128 d_model x 256 d_ff] += eta * Vhat_i^T (MN-major) x Z_i (MN-major),
//                 K = C; the epilogue keeps W in float32 and writes the bf16 copy Wb_{i+1}
//                 that the next chunk's apply tiles read.
// Apply tiles (long, K = d_ff) are handed out first, update tiles fill the remaining SMs.
// Warp roles: warp 0 issues TMA loads into a 4-stage ring, warp 1 issues tcgen05.mma into
// two TMEM accumulators of 128 x 256 fp32, warps 2-9 drain the accumulators (two warps per
// TMEM lane quadrant, each taking 128 of the 256 columns).
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"

namespace tttk {
namespace {

constexpr int BM = 128, BN = 256, BK = 64, STAGES = 4, RING = 4;
constexpr uint32_t A_BYTES = BM * BK * 2;      // 16 KB
constexpr uint32_t B_BYTES = BN * BK * 2;      // 32 KB
constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int kThreads = 320;
constexpr int kEpiWarps = 8;
constexpr uint32_t kTmemCols = 512;            // two 256-column accumulators

struct Params {
  int chunk, C, d_ff, d_model;
  int n_apply_n, n_upd_n, n_apply, n_total;
  int kb_apply, kb_upd;
  int wb_cur_row0, wb_next_row0;
  float lr;
  float* W;
  __nv_bfloat16* Wb;
  __nv_bfloat16* O;
  int* counter;
  unsigned* err;
};

struct Tile {
  int apply, m0, n0, nkb;
};

__device__ __forceinline__ Tile decode(const Params& p, int t) {
  Tile x;
  if (t < p.n_apply) {
    x.apply = 1;
    x.m0 = (t / p.n_apply_n) * BM;  // token offset inside the chunk
    x.n0 = (t % p.n_apply_n) * BN;  // d_model column
    x.nkb = p.kb_apply;
  } else {
    const int u = t - p.n_apply;
    x.apply = 0;
    x.m0 = (u / p.n_upd_n) * BM;    // d_model row
    x.n0 = (u % p.n_upd_n) * BN;    // d_ff column
    x.nkb = p.kb_upd;
  }
  return x;
}

struct __align__(8) Bars {
  uint64_t full[STAGES], empty[STAGES], acc_full[2], acc_empty[2], tile_full[RING],
      tile_empty[RING];
  int ring[RING];
  uint32_t tmem_base;
  int abort_flag;
};

__global__ void __launch_bounds__(kThreads, 1)
    inplace_chunk_kernel(const __grid_constant__ CUtensorMap tm_za,
                         const __grid_constant__ CUtensorMap tm_zb,
                         const __grid_constant__ CUtensorMap tm_wb,
                         const __grid_constant__ CUtensorMap tm_vh, const Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  Bars* bars = reinterpret_cast<Bars*>(smem + STAGES * STAGE_BYTES);
  const uint32_t stage0 = smem_u32(smem);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  Abort ab{&bars->abort_flag, p.err};

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(smem_u32(&bars->full[s]), 1);
      mbar_init(smem_u32(&bars->empty[s]), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(smem_u32(&bars->acc_full[a]), 1);
      mbar_init(smem_u32(&bars->acc_empty[a]), kEpiWarps);
    }
    for (int r = 0; r < RING; ++r) {
      mbar_init(smem_u32(&bars->tile_full[r]), 1);
      mbar_init(smem_u32(&bars->tile_empty[r]), 1 + kEpiWarps);
    }
    bars->abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tm_za);
    tma_prefetch_desc(&tm_zb);
    tma_prefetch_desc(&tm_wb);
    tma_prefetch_desc(&tm_vh);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&bars->tmem_base), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  const int row_base = p.chunk * p.C;  // first token of this chunk

  if (warp == 0) {
    if (lane == 0) {
      int r = 0, s = 0;
      uint32_t rph = 0, sph = 0;
      for (;;) {
        if (!mbar_wait(smem_u32(&bars->tile_empty[r]), rph ^ 1, ab)) break;
        const int t = atomicAdd(p.counter, 1);
        bars->ring[r] = t;
        mbar_arrive(smem_u32(&bars->tile_full[r]));
        if (++r == RING) { r = 0; rph ^= 1; }
        if (t >= p.n_total) break;
        const Tile x = decode(p, t);
        bool ok = true;
        for (int kb = 0; kb < x.nkb && ok; ++kb) {
          if (!mbar_wait(smem_u32(&bars->empty[s]), sph ^ 1, ab)) { ok = false; break; }
          const uint32_t fb = smem_u32(&bars->full[s]);
          const uint32_t sa = stage0 + s * STAGE_BYTES, sb = sa + A_BYTES;
          mbar_arrive_expect_tx(fb, STAGE_BYTES);
          if (x.apply) {
            tma_load_2d(sa, &tm_za, fb, kb * BK, row_base + x.m0);
            tma_load_2d(sb, &tm_wb, fb, kb * BK, p.wb_cur_row0 + x.n0);
          } else {
            const int tok = row_base + kb * BK;
            tma_load_2d(sa, &tm_vh, fb, x.m0, tok);
            tma_load_2d(sa + 8192, &tm_vh, fb, x.m0 + 64, tok);
            for (int j = 0; j < 4; ++j) tma_load_2d(sb + 8192 * j, &tm_zb, fb, x.n0 + 64 * j, tok);
          }
          if (++s == STAGES) { s = 0; sph ^= 1; }
        }
        if (!ok) break;
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      int r = 0, s = 0, acc = 0;
      uint32_t rph = 0, sph = 0, aph = 0;
      const uint32_t id_apply = idesc_bf16(BM, BN, 0, 0);
      const uint32_t id_upd = idesc_bf16(BM, BN, 1, 1);
      for (;;) {
        if (!mbar_wait(smem_u32(&bars->tile_full[r]), rph, ab)) break;
        const int t = bars->ring[r];
        mbar_arrive(smem_u32(&bars->tile_empty[r]));
        if (++r == RING) { r = 0; rph ^= 1; }
        if (t >= p.n_total) break;
        const Tile x = decode(p, t);
        if (!mbar_wait(smem_u32(&bars->acc_empty[acc]), aph ^ 1, ab)) break;
        tc_fence_after();
        const uint32_t d = tmem + acc * BN;
        bool ok = true;
        for (int kb = 0; kb < x.nkb; ++kb) {
          if (!mbar_wait(smem_u32(&bars->full[s]), sph, ab)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = stage0 + s * STAGE_BYTES, sb = sa + A_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            uint64_t ad, bd;
            if (x.apply) {
              ad = sdesc_sw128(sa + kk * 32, 16, 1024);
              bd = sdesc_sw128(sb + kk * 32, 16, 1024);
            } else {
              ad = sdesc_sw128(sa + kk * 2048, 8192, 1024);
              bd = sdesc_sw128(sb + kk * 2048, 8192, 1024);
            }
            mma_bf16_ss(d, ad, bd, x.apply ? id_apply : id_upd, (kb | kk) != 0);
          }
          mma_commit(smem_u32(&bars->empty[s]));
          if (++s == STAGES) { s = 0; sph ^= 1; }
        }
        if (!ok) break;
        mma_commit(smem_u32(&bars->acc_full[acc]));
        if (++acc == 2) { acc = 0; aph ^= 1; }
      }
    }
  } else {
    // Epilogue: warp w drains TMEM lanes 32*(w%4) .. +31 (thread = one accumulator row) and
    // columns [128 h, 128 h + 128) with h = (w - 2) / 4.
    const int q = warp & 3;
    const int row = q * 32 + lane;
    const int hcol = (warp - 2) / 4;
    int r = 0, acc = 0;
    uint32_t rph = 0, aph = 0;
    for (;;) {
      if (!mbar_wait(smem_u32(&bars->tile_full[r]), rph, ab)) break;
      const int t = bars->ring[r];
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bars->tile_empty[r]));
      if (++r == RING) { r = 0; rph ^= 1; }
      if (t >= p.n_total) break;
      const Tile x = decode(p, t);
      if (!mbar_wait(smem_u32(&bars->acc_full[acc]), aph, ab)) break;
      __syncwarp();
      tc_fence_after();
      for (int cb = hcol * (BN / 64); cb < (hcol + 1) * (BN / 64); ++cb) {
        float v[32];
        tmem_ld32(tmem_addr(tmem, q * 32, acc * BN + cb * 32), v);
        tmem_wait_ld();
        const int col0 = x.n0 + cb * 32;
        if (x.apply) {
          if (col0 < p.d_model) {
            uint4* dst = reinterpret_cast<uint4*>(
                p.O + (size_t)(row_base + x.m0 + row) * p.d_model + col0);
#pragma unroll
            for (int j = 0; j < 4; ++j)
              dst[j] = make_uint4(pack_bf16x2(v[8 * j], v[8 * j + 1]),
                                  pack_bf16x2(v[8 * j + 2], v[8 * j + 3]),
                                  pack_bf16x2(v[8 * j + 4], v[8 * j + 5]),
                                  pack_bf16x2(v[8 * j + 6], v[8 * j + 7]));
          }
        } else {
          const int m = x.m0 + row;
          if (col0 < p.d_ff && m < p.d_model) {
            float4* w = reinterpret_cast<float4*>(p.W + (size_t)m * p.d_ff + col0);
            uint4* wb =
                reinterpret_cast<uint4*>(p.Wb + (size_t)(p.wb_next_row0 + m) * p.d_ff + col0);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              float4 a0 = w[2 * j], a1 = w[2 * j + 1];
              a0.x += p.lr * v[8 * j + 0];
              a0.y += p.lr * v[8 * j + 1];
              a0.z += p.lr * v[8 * j + 2];
              a0.w += p.lr * v[8 * j + 3];
              a1.x += p.lr * v[8 * j + 4];
              a1.y += p.lr * v[8 * j + 5];
              a1.z += p.lr * v[8 * j + 6];
              a1.w += p.lr * v[8 * j + 7];
              w[2 * j] = a0;
              w[2 * j + 1] = a1;
              wb[j] = make_uint4(pack_bf16x2(a0.x, a0.y), pack_bf16x2(a0.z, a0.w),
                                 pack_bf16x2(a1.x, a1.y), pack_bf16x2(a1.z, a1.w));
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bars->acc_empty[acc]));
      if (++acc == 2) { acc = 0; aph ^= 1; }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (bars->abort_flag) __nanosleep(100000);  // let any load issued before the abort land
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

__global__ void to_bf16_kernel(const float* __restrict__ src, __nv_bfloat16* __restrict__ dst,
                               size_t n) {
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (size_t)gridDim.x * blockDim.x)
    dst[i] = __float2bfloat16_rn(src[i]);
}

constexpr size_t kSmemBytes = STAGES * STAGE_BYTES + sizeof(Bars) + 1024;

}  // namespace

size_t inplace_workspace(int T, int d_ff, int d_model, int C) {
  const size_t wb = 2 * (size_t)d_model * d_ff * 2;
  const size_t counters = ((size_t)(T / C) * sizeof(int) + 255) & ~size_t(255);
  return wb + counters;
}

cudaError_t inplace_run(int T, int d_ff, int d_model, int C, float lr, const void* Z,
                        const void* Vhat, float* W, void* O, void* ws, unsigned* err,
                        cudaStream_t s) {
  __nv_bfloat16* Wb = static_cast<__nv_bfloat16*>(ws);
  int* counters = reinterpret_cast<int*>(static_cast<uint8_t*>(ws) + 2 * (size_t)d_model * d_ff * 2);
  const int NC = T / C;
  CUtensorMap tza, tzb, twb, tvh;
  if (!make_tmap_bf16(&tza, Z, d_ff, T, d_ff, BK, BM) ||
      !make_tmap_bf16(&tzb, Z, d_ff, T, d_ff, 64, BK) ||
      !make_tmap_bf16(&twb, Wb, d_ff, 2 * (size_t)d_model, d_ff, BK, BN) ||
      !make_tmap_bf16(&tvh, Vhat, d_model, T, d_model, 64, BK))
    return cudaErrorInvalidValue;
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(inplace_chunk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  const size_t nW = (size_t)d_model * d_ff;
  to_bf16_kernel<<<sms * 4, 256, 0, s>>>(W, Wb, nW);
  e = cudaMemsetAsync(counters, 0, NC * sizeof(int), s);
  if (e != cudaSuccess) return e;
  Params p{};
  p.C = C;
  p.d_ff = d_ff;
  p.d_model = d_model;
  p.n_apply_n = (d_model + BN - 1) / BN;
  p.n_upd_n = (d_ff + BN - 1) / BN;
  p.n_apply = (C / BM) * p.n_apply_n;
  p.n_total = p.n_apply + (d_model / BM) * p.n_upd_n;
  p.kb_apply = d_ff / BK;
  p.kb_upd = C / BK;
  p.lr = lr;
  p.W = W;
  p.Wb = Wb;
  p.O = static_cast<__nv_bfloat16*>(O);
  p.err = err;
  const int grid = p.n_total < sms ? p.n_total : sms;
  for (int i = 0; i < NC; ++i) {
    p.chunk = i;
    p.wb_cur_row0 = (i & 1) * d_model;
    p.wb_next_row0 = ((i + 1) & 1) * d_model;
    p.counter = counters + i;
    inplace_chunk_kernel<<<grid, kThreads, kSmemBytes, s>>>(tza, tzb, twb, tvh, p);
  }
  count_launches(NC + 1);
  return cudaGetLastError();
}

}  // namespace tttk
