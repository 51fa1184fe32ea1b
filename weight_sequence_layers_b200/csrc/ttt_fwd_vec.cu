// tcgen05 forward of the chunkwise TTT layer with a per-feature (vector) decay, identity
// activation, d_k = d_v = 64 (bf16 operands, fp32 state and accumulators).
//
// Page "Modular TTT: Rethinking Test-Time Training as Composable Modules", section "权重衰减"
// (a forgetting factor per key feature, i.e. a decay matrix) with the chunk dual form of section
// "方法步骤详情". Per chunk, with W0 the chunk-start state and L_ti = sum_{t'<=t} log gamma_t'i
// (chunk-local, one per key feature i):
//   G     = K W0 - V (MSE) or -V (inner product)
//   W_end = diag(exp(L_C)) W0 - Khat^T diag(eta) G,    Khat_ri = k_ri exp(L_Ci - L_ri)
//   O     = R W0 + S V,   S_sr = eta_r sum_i q_si k_ri exp(L_si - L_ri)   (r <= s)
//           R = Q * exp(L) - S K (MSE) or Q * exp(L) (inner product)
// The per-feature weights inside the Q K^T contraction reach the tensor cores as scaled operands:
// for the 128-query block qb with reference token m (its 64th token),
//   qtilde_s = q_s * exp(L_s - L_m),   ktilde_r = k_r * exp(L_m - L_r),
// so that qtilde_s . ktilde_r = sum_i q_si k_ri exp(L_si - L_ri). On earlier key blocks every
// exponent is <= 0; on the diagonal block it spans at most 64 tokens of one feature's decay. A
// factor beyond exp(80) is clamped and recorded in the device error word (a range error).
//
// Three kernels:
//   prep   : one CTA per (batch, head, chunk): the per-feature log-decay scan and every decayed
//            operand (qtilde, ktilde per reference token, Khat) written once as bf16, with
//            exp(L_C) and exp(L_m); the backward reuses it (and keeps L itself).
//   vstate : one CTA per (batch, head) walks the chunks with the fp32 state in TMEM: Z = K W0,
//            -eta G, W = diag(exp(L_C)) W + Khat^T (-eta G); K and Khat arrive by TMA.
//   vout   : one CTA per (batch, head, chunk, 128-query block), two per SM:
//            P = qtilde ktilde^T, S = P * eta (causal), R, O = R W0 + S V.
#include <cuda_bf16.h>
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "tc_util.cuh"

namespace tttk {
namespace {

constexpr uint32_t PANEL = 128 * 128;  // 128 rows x 128 bytes: 128 tokens x 64 bf16
constexpr int VD = 64;                 // d_k = d_v
constexpr int kEpi = 8;
constexpr float kMaxExp = 80.f;        // largest exponent a scaled operand factor may take

struct VecParams {
  int BH, T, NC;
  float lr_bias;
  const float* beta;
  const float* W0;      // [BH, 64, 64]
  const float* GC;      // [BH, NC, 64] exp(L_C)
  const float* Em;      // [BH, NC, NB, 64] exp(L_m)
  float* W_final;       // nullable
  __nv_bfloat16* Wc;    // [BH, NC, 64, 64]
  __nv_bfloat16* O;
  int save_g;
};

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}
__device__ __forceinline__ float eta_of(const float* beta, size_t row, float lr_bias) {
  return 2.f * sigm(__ldg(beta + row) + lr_bias);
}

// ================================================================================== prep
// Thread (f = four adjacent key features, seg = one of 16 slices of the chunk). The slice
// boundaries fall on the reference tokens' successors (m + 1 = 64 and 192 for C = 256, 64 for
// C = 128), so L_m is a sum of whole slices. Every L_t is the same left-to-right sum in both
// passes, so the exponent at the reference token is exactly 0.
struct PrepParams {
  int NC;
  const float* gamma;
  const __nv_bfloat16* Q;
  const __nv_bfloat16* K;
  __nv_bfloat16 *Qt, *Kh, *Kt;
  float *GC, *Em, *Lf;
  unsigned* err;
};

__device__ __forceinline__ float clamped_exp(float e, bool& range) {
  if (e > kMaxExp) {
    e = kMaxExp;
    range = true;
  }
  return __expf(e);
}
__device__ __forceinline__ float4 log4(float4 g) {
  return make_float4(__logf(g.x), __logf(g.y), __logf(g.z), __logf(g.w));
}
__device__ __forceinline__ float4 add4(float4 a, float4 b) {
  return make_float4(a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w);
}
// four bf16 (8 bytes) times exp(e) each, rounded back to bf16
__device__ __forceinline__ uint2 scale4(uint2 x, float4 e, bool& range) {
  uint2 r;
  r.x = pack_bf16x2(bf16lo(x.x) * clamped_exp(e.x, range), bf16hi(x.x) * clamped_exp(e.y, range));
  r.y = pack_bf16x2(bf16lo(x.y) * clamped_exp(e.z, range), bf16hi(x.y) * clamped_exp(e.w, range));
  return r;
}

constexpr int kPrepSeg = 16;  // slices per chunk
constexpr int kPrepThreads = 128;  // 8 feature quads (32 features) x 16 slices

// One CTA per (batch, head, chunk, half of the features). Each thread loads its whole slice
// (gamma, q, k) into registers before any arithmetic, so every load is in flight at once.
template <int NB>
__global__ void __launch_bounds__(kPrepThreads) vec_prep_kernel(const PrepParams p) {
  constexpr int C = 128 * NB, SEG = C / kPrepSeg, NV = NB * (NB + 1) / 2;
  __shared__ float4 tot[kPrepSeg][8];
  const int f = threadIdx.x & 7, seg = threadIdx.x >> 3;
  const int fq = (blockIdx.x & 1) * 8 + f;  // feature quad 0..15
  const size_t bc = blockIdx.x >> 1;        // bh * NC + c
  const size_t r0 = bc * C + seg * SEG;     // first token row of this slice
  const float4* __restrict__ g = reinterpret_cast<const float4*>(p.gamma + r0 * VD) + fq;
  const uint2* __restrict__ q = reinterpret_cast<const uint2*>(p.Q + r0 * VD) + fq;
  const uint2* __restrict__ k = reinterpret_cast<const uint2*>(p.K + r0 * VD) + fq;
  float4 lg[SEG];
  uint2 qv[SEG], kv[SEG];
#pragma unroll
  for (int t = 0; t < SEG; ++t) {
    lg[t] = __ldg(g + t * (VD / 4));
    qv[t] = __ldg(q + t * (VD / 4));
    kv[t] = __ldg(k + t * (VD / 4));
  }
  {
    float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int t = 0; t < SEG; ++t) {
      lg[t] = log4(lg[t]);
      s = add4(s, lg[t]);
    }
    tot[seg][f] = s;
  }
  __syncthreads();
  float4 Lstart = make_float4(0.f, 0.f, 0.f, 0.f), LC = Lstart, Lm[NB];
#pragma unroll
  for (int kk = 0; kk < kPrepSeg; ++kk) {
    const float4 tk = tot[kk][f];
    if (kk < seg) Lstart = add4(Lstart, tk);
    LC = add4(LC, tk);
#pragma unroll
    for (int qb = 0; qb < NB; ++qb)
      if (kk == (128 * qb + 64) / SEG - 1) Lm[qb] = LC;
  }
  const int kb = seg * SEG / 128;
  bool range = false;
  float4 l = make_float4(0.f, 0.f, 0.f, 0.f);
  uint2* qt = reinterpret_cast<uint2*>(p.Qt + r0 * VD) + fq;
  uint2* kh = reinterpret_cast<uint2*>(p.Kh + r0 * VD) + fq;
  const float4 lmk = Lm[kb];
#pragma unroll
  for (int t = 0; t < SEG; ++t) {
    const int o = t * (VD / 4);
    l = add4(l, lg[t]);
    const float4 L = add4(Lstart, l);
    qt[o] = scale4(qv[t], make_float4(L.x - lmk.x, L.y - lmk.y, L.z - lmk.z, L.w - lmk.w), range);
    kh[o] = scale4(kv[t], make_float4(LC.x - L.x, LC.y - L.y, LC.z - L.z, LC.w - L.w), range);
    const int tr = (seg * SEG + t) & 127;  // row inside the key block
#pragma unroll
    for (int qb = 0; qb < NB; ++qb) {
      if (qb < kb) continue;
      const int v = qb * (qb + 1) / 2 + kb;
      const float4 m = Lm[qb];
      reinterpret_cast<uint2*>(p.Kt + ((bc * NV + v) * 128 + tr) * VD)[fq] =
          scale4(kv[t], make_float4(m.x - L.x, m.y - L.y, m.z - L.z, m.w - L.w), range);
    }
    if (p.Lf) reinterpret_cast<float4*>(p.Lf + r0 * VD)[o + fq] = L;
  }
  if (seg == 0) {
    reinterpret_cast<float4*>(p.GC + bc * VD)[fq] =
        make_float4(__expf(LC.x), __expf(LC.y), __expf(LC.z), __expf(LC.w));
#pragma unroll
    for (int qb = 0; qb < NB; ++qb)
      reinterpret_cast<float4*>(p.Em + (bc * NB + qb) * VD)[fq] = make_float4(
          __expf(Lm[qb].x), __expf(Lm[qb].y), __expf(Lm[qb].z), __expf(Lm[qb].w));
  }
  if (range) atomicOr(p.err, ERR_RANGE);
}

// ================================================================================= vstate
template <int NB>
struct VsL {
  static constexpr int C = 128 * NB;
  static constexpr uint32_t KBUF = C * 128;              // one chunk, 64 features
  static constexpr uint32_t OFF_K = 0;                   // two K chunks
  static constexpr uint32_t OFF_KH = 2 * KBUF;           // two Khat chunks
  static constexpr uint32_t OFF_V = 4 * KBUF;            // V (then G in place)
  static constexpr uint32_t OFF_UG = 5 * KBUF;           // -eta G
  static constexpr uint32_t OFF_W = 6 * KBUF;            // bf16 state copy, 64 x 64
  static constexpr uint32_t OFF_BAR = OFF_W + VD * 128;
  static constexpr uint32_t T_W = 0, T_Z = 64;
};
struct __align__(8) VsBars {
  uint64_t k_full[2], k_free[2], v_full, z_full, g_ready, w_full, w0_ready;
  uint32_t tmem_base;
  int abort_flag;
};
template <int NB>
constexpr uint32_t vs_bytes() { return VsL<NB>::OFF_BAR + sizeof(VsBars); }
constexpr int kVsThreads = 320;  // producer, MMA, 8 epilogue warps

template <int NB, int LOSS>
__global__ void __launch_bounds__(kVsThreads, 1)
    fwd_vstate_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmKh,
                      const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmG,
                      const VecParams p, unsigned* err) {
  using L = VsL<NB>;
  constexpr int C = L::C;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  const uint32_t sb = smem_u32(smem);
  const uint32_t sK = sb + L::OFF_K, sKH = sb + L::OFF_KH, sV = sb + L::OFF_V,
                 sUG = sb + L::OFF_UG, sW = sb + L::OFF_W;
  VsBars* bars = reinterpret_cast<VsBars*>(smem + L::OFF_BAR);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int bh = blockIdx.x;
  const int NC = p.NC;
  Abort ab{&bars->abort_flag, err};
#define BAR(x) smem_u32(&bars->x)
  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(BAR(k_full[i]), 1);
      mbar_init(BAR(k_free[i]), 1);
    }
    mbar_init(BAR(v_full), 1);
    mbar_init(BAR(z_full), 1);
    mbar_init(BAR(g_ready), kEpi);
    mbar_init(BAR(w_full), 1);
    mbar_init(BAR(w0_ready), kEpi);
    bars->abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmKh);
    tma_prefetch_desc(&tmV);
  }
  if (warp == 1) {
    tmem_alloc(BAR(tmem_base), 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      auto load_k = [&](int cc) {
        const uint32_t x = cc & 1, bar = BAR(k_full[x]);
        mbar_arrive_expect_tx(bar, 2 * L::KBUF);
        for (int h = 0; h < NB; ++h) {
          const int row = bh * p.T + cc * C + 128 * h;
          tma_load_2d(sK + x * L::KBUF + h * PANEL, &tmK, bar, 0, row);
          tma_load_2d(sKH + x * L::KBUF + h * PANEL, &tmKh, bar, 0, row);
        }
      };
      auto load_v = [&](int cc) {
        mbar_arrive_expect_tx(BAR(v_full), C * 128);
        tma_load_2d(sV, &tmV, BAR(v_full), 0, bh * p.T + cc * C);
      };
      load_k(0);
      load_v(0);
      if (NC > 1) load_k(1);
      for (int c = 0; c < NC; ++c) {
        // once every epilogue warp has formed this chunk's G from V: store G when it is kept,
        // then V of the next chunk into the same buffer
        if (!mbar_wait(BAR(g_ready), c & 1, ab)) break;
        if (p.save_g) {
          tma_store_2d(&tmG, sV, 0, bh * p.T + c * C);
          bulk_commit();
          if (c + 1 < NC) bulk_wait_read0();
        }
        if (c + 1 < NC) load_v(c + 1);
        if (c + 2 < NC) {
          if (!mbar_wait(BAR(k_free[c & 1]), (c >> 1) & 1, ab)) break;
          load_k(c + 2);
        }
      }
      if (p.save_g) bulk_wait0();
    }
  } else if (warp == 1) {
    // -------------------------------------------- MMA issue: Z = K W0, W += Khat^T (-eta G)
    if (lane == 0) {
      const uint32_t idZ = idesc_bf16(128, VD, 0, 1);  // K-major A, MN-major B
      const uint32_t idW = idesc_bf16(128, VD, 1, 1);  // MN-major A (Khat^T) and B
      for (int c = 0; c < NC; ++c) {
        const int x = c & 1;
        const uint32_t sKx = sK + x * L::KBUF, sKHx = sKH + x * L::KBUF;
        if (!mbar_wait(BAR(w0_ready), c & 1, ab) || !mbar_wait(BAR(k_full[x]), (c >> 1) & 1, ab))
          break;
        tc_fence_after();
        if constexpr (LOSS == 0) {
          for (int b = 0; b < NB; ++b) {
#pragma unroll
            for (int j = 0; j < VD / 16; ++j)
              mma_bf16_ss(tmem + L::T_Z + VD * b,
                          sdesc_sw128(sKx + b * PANEL + j * 32, 16, 1024),
                          sdesc_sw128(sW + j * 2048, 0, 1024), idZ, j > 0);
          }
          mma_commit(BAR(z_full));
        }
        if (!mbar_wait(BAR(g_ready), c & 1, ab)) break;
        tc_fence_after();
        // M = 128 over the 64 key features: the upper half of the result lanes repeats the lower
        // (LBO 0) and is never read
        for (int j = 0; j < C / 16; ++j)
          mma_bf16_ss(tmem + L::T_W, sdesc_sw128(sKHx + (j / 8) * PANEL + (j % 8) * 2048, 0, 1024),
                      sdesc_sw128(sUG + j * 2048, 0, 1024), idW, 1);
        mma_commit(BAR(w_full));
        mma_commit(BAR(k_free[x]));
      }
    }
  } else {
    // ------------------------------------------------------------------ epilogue
    const int ew = warp - 2, g = ew / 4, q = warp & 3;
    const int lrow = q * 32 + lane;
    const uint32_t loff = (uint32_t)(q * 32) << 16;
    const bool w_rows = q * 32 < VD;
    const int col = 32 * g;
    const float* GC = p.GC + (size_t)bh * NC * VD;
    auto wc_row = [&](int cc) { return p.Wc + ((size_t)(bh * NC + cc) * VD + lrow) * VD + col; };
    if (w_rows) {
      // chunk 0: the bf16 operand copy of W0, its checkpoint, diag(Gamma_C(0)) W0 into TMEM
      float w[32];
      const float4* src = reinterpret_cast<const float4*>(p.W0 + ((size_t)bh * VD + lrow) * VD + col);
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const float4 v = src[k];
        w[4 * k] = v.x; w[4 * k + 1] = v.y; w[4 * k + 2] = v.z; w[4 * k + 3] = v.w;
      }
      st_row32(sW, lrow, 4 * g, w);
      st_global_bf16x32(wc_row(0), w);
      const float g0 = __ldg(GC + lrow);
#pragma unroll
      for (int j = 0; j < 32; ++j) w[j] *= g0;
      tmem_st32(tmem + loff + L::T_W + 32 * g, w);
      tmem_wait_st();
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(BAR(w0_ready));
    for (int c = 0; c < NC; ++c) {
      const size_t r0 = (size_t)bh * p.T + (size_t)c * C;
      float eta[NB];
#pragma unroll
      for (int b = 0; b < NB; ++b) eta[b] = eta_of(p.beta, r0 + 128 * b + lrow, p.lr_bias);
      if (!mbar_wait(BAR(v_full), c & 1, ab) || (LOSS == 0 && !mbar_wait(BAR(z_full), c & 1, ab)))
        break;
      __syncwarp();
      tc_fence_after();
#pragma unroll
      for (int b = 0; b < NB; ++b) {
        const int row = 128 * b + lrow;
        float v[32], ug[32];
        ld_row32(sV, row, 4 * g, v);
        if constexpr (LOSS == 0) {
          float z[32];
          tmem_ld32(tmem + loff + L::T_Z + VD * b + 32 * g, z);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = z[j] - v[j];
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = -v[j];
        }
        const float ne = -eta[b];
#pragma unroll
        for (int j = 0; j < 32; ++j) ug[j] = ne * v[j];
        if (p.save_g) st_row32(sV, row, 4 * g, v);
        st_row32(sUG, row, 4 * g, ug);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(g_ready));
      // -------- the next chunk's state: bf16 copy, checkpoint, diag(Gamma_C) W in TMEM
      const bool more = c + 1 < NC;
      const float gn = (more && w_rows) ? __ldg(GC + (size_t)(c + 1) * VD + lrow) : 0.f;
      if (!mbar_wait(BAR(w_full), c & 1, ab)) break;
      __syncwarp();
      tc_fence_after();
      if (w_rows) {
        float w[32];
        tmem_ld32(tmem + loff + L::T_W + 32 * g, w);
        tmem_wait_ld();
        if (more) {
          st_row32(sW, lrow, 4 * g, w);
          st_global_bf16x32(wc_row(c + 1), w);
#pragma unroll
          for (int j = 0; j < 32; ++j) w[j] *= gn;
          tmem_st32(tmem + loff + L::T_W + 32 * g, w);
          tmem_wait_st();
        } else if (p.W_final) {
          float4* dst = reinterpret_cast<float4*>(p.W_final + ((size_t)bh * VD + lrow) * VD + col);
#pragma unroll
          for (int k = 0; k < 8; ++k)
            dst[k] = make_float4(w[4 * k], w[4 * k + 1], w[4 * k + 2], w[4 * k + 3]);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(w0_ready));
    }
  }
#undef BAR
  tc_fence_before();
  __syncthreads();
  if (bars->abort_flag) __nanosleep(100000);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

// =================================================================================== vout
// S_sr = P_sr eta_r for r <= s (the decay is inside P through the scaled operands), packed
// to bf16 pairs for one query s against 32 keys r0..
template <bool MASK>
__device__ __forceinline__ void eta_weights32(const float (&pv)[32], const float* eta, int s, int r0,
                                              uint32_t (&pk)[16]) {
  const float4* e4 = reinterpret_cast<const float4*>(eta + r0);
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const float4 e = e4[k];
    float x0 = pv[4 * k] * e.x, x1 = pv[4 * k + 1] * e.y, x2 = pv[4 * k + 2] * e.z,
          x3 = pv[4 * k + 3] * e.w;
    if (MASK) {
      const int r = r0 + 4 * k;
      if (r > s) x0 = 0.f;
      if (r + 1 > s) x1 = 0.f;
      if (r + 2 > s) x2 = 0.f;
      if (r + 3 > s) x3 = 0.f;
    }
    pk[2 * k] = pack_bf16x2(x0, x1);
    pk[2 * k + 1] = pack_bf16x2(x2, x3);
  }
}
struct EWeights {
  const float* eta;
  int s, rbase;
  __device__ bool full(int idx, int q) const { return idx < q; }
  __device__ void operator()(const float (&pv)[32], int idx, bool mask, uint32_t (&pk)[16]) const {
    if (mask) eta_weights32<true>(pv, eta, s, rbase + 32 * idx, pk);
    else eta_weights32<false>(pv, eta, s, rbase + 32 * idx, pk);
  }
};

// Out-of-place packing of one 128-column fp32 score block (src, the thread's TMEM row) into
// 64 bf16-pair columns at dst (K-step j of the MMA that reads it at dst + 8 j), one warpgroup.
template <typename F>
__device__ __forceinline__ void pack_block_to(uint32_t src, uint32_t dst, int q, bool diag,
                                              const F& weights) {
#pragma unroll 1
  for (int idx = 0; idx < 4; ++idx) {
    const int kind = diag ? (idx == q ? 2 : weights.full(idx, q) ? 1 : 0) : 1;
    uint32_t pk[16];
    if (kind == 0) {
#pragma unroll
      for (int j = 0; j < 16; ++j) pk[j] = 0u;
    } else {
      float pv[32];
      tmem_ld32(src + 32 * idx, pv);
      tmem_wait_ld();
      weights(pv, idx, kind == 2, pk);
    }
    tmem_st16u(dst + 16 * idx, pk);
  }
}


// Shared memory: five 128 x 64 bf16 slots used in turn
//   A: qtilde, then R (over it)
//   B: ktilde of key block 0, then V_0 (once P_0 is done)
//   C: ktilde of key block 1, then V_1 (once P_1 is done)            (second key block)
//   D: K_0 for S K, then W0 (once S K is done; inner product: W0 from the start)
//   E: K_1 for S K                                                     (MSE, second key block)
// TMEM (256 columns): packed S blocks [0, 64), [64, 128); one fp32 accumulator [128, 256) that
// takes each raw score block, then S K, then Zq.
struct VoL {
  static constexpr uint32_t OFF_A = 0, OFF_B = PANEL, OFF_C = 2 * PANEL, OFF_D = 3 * PANEL,
                            OFF_E = 4 * PANEL;
  static constexpr uint32_t OFF_F = 5 * PANEL;              // eta[256], exp(L_m)[64]
  static constexpr uint32_t OFF_BAR = OFF_F + (256 + 64) * 4;
  static constexpr uint32_t T_S = 0, T_ACC = 128;
};
enum { U_A, U_B, U_C, U_D, U_E, U_P, U_PK, U_PD0, U_PD1, U_SK, U_B2, U_C2, U_D2, U_R, U_ZQ,
       U_SCAN, U_NBARS };
struct __align__(8) VoBars {
  uint64_t b[U_NBARS];
  uint32_t tmem_base;
  int abort_flag;
};
constexpr uint32_t vo_bytes() { return VoL::OFF_BAR + sizeof(VoBars); }
constexpr int kVoThreads = 192;

template <int NB, int LOSS>
__global__ void __launch_bounds__(kVoThreads, 2)
    fwd_vout_kernel(const __grid_constant__ CUtensorMap tmQt, const __grid_constant__ CUtensorMap tmKt,
                    const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                    const __grid_constant__ CUtensorMap tmW, const VecParams p, unsigned* err) {
  constexpr int C = 128 * NB, NV = NB * (NB + 1) / 2;
  using L = VoL;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  const uint32_t sb = smem_u32(smem);
  const uint32_t sA = sb + L::OFF_A, sB = sb + L::OFF_B, sC = sb + L::OFF_C, sD = sb + L::OFF_D,
                 sE = sb + L::OFF_E;
  float* f_eta = reinterpret_cast<float*>(smem + L::OFF_F);
  float* f_eLm = f_eta + 256;
  VoBars* bars = reinterpret_cast<VoBars*>(smem + L::OFF_BAR);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  // the last chunk first, the heavier query block first
  const int per_c = p.BH * NB;
  const int c = p.NC - 1 - (int)blockIdx.x / per_c;
  const int rem = (int)blockIdx.x % per_c;
  const int bh = rem / NB, qb = NB - 1 - rem % NB;
  const int tokc = bh * p.T + c * C;
  const int bc = bh * p.NC + c;
  Abort ab{&bars->abort_flag, err};
#define UB(i) smem_u32(&bars->b[i])
  if (threadIdx.x == 0) {
    for (int i = 0; i < U_NBARS; ++i)
      mbar_init(UB(i), (i == U_PK || i == U_R || i == U_SCAN) ? 4 : 1);
    bars->abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&bars->tmem_base), 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  auto load = [&](uint32_t dst, const CUtensorMap* mp, int bar, int row) {
    mbar_arrive_expect_tx(UB(bar), PANEL);
    tma_load_2d(dst, mp, UB(bar), 0, row);
  };
  auto load_w = [&](int bar) {
    mbar_arrive_expect_tx(UB(bar), VD * 128);
    tma_load_2d(sD, &tmW, UB(bar), 0, bc * VD);
  };
  // first row of ktilde version (qb, kb) of this chunk
  auto kt_row = [&](int kb) { return ((bc * NV) + qb * (qb + 1) / 2 + kb) * 128; };

  if (warp == 0) {
    if (lane == 0) {
      load(sA, &tmQt, U_A, tokc + 128 * qb);
      load(sB, &tmKt, U_B, kt_row(0));
      if (qb == 1) load(sC, &tmKt, U_C, kt_row(1));
      if (LOSS == 0) {
        load(sD, &tmK, U_D, tokc);
        if (qb == 1) load(sE, &tmK, U_E, tokc + 128);
      } else {
        load_w(U_D);
      }
      // slots freed by the score MMAs take the values, the S K slot takes W0
      if (mbar_wait(UB(U_PD0), 0, ab)) load(sB, &tmV, U_B2, tokc);
      if (qb == 1 && mbar_wait(UB(U_PD1), 0, ab)) load(sC, &tmV, U_C2, tokc + 128);
      if (LOSS == 0 && mbar_wait(UB(U_SK), 0, ab)) load_w(U_D2);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idP = idesc_bf16(128, 128, 0, 0);  // qtilde ktilde^T: both K-major
      const uint32_t idN = idesc_bf16(128, VD, 0, 1);   // S K, S V, R W0: MN-major B
      const uint32_t tacc = tmem + L::T_ACC;
      do {
        if (!mbar_wait(UB(U_A), 0, ab)) break;
        bool ok = true;
        for (int b = 0; b <= qb && ok; ++b) {
          if (!(ok = mbar_wait(UB(b == 0 ? U_B : U_C), 0, ab))) break;
          // the accumulator is free once the previous block has been packed out of it
          if (b > 0 && !(ok = mbar_wait(UB(U_PK), 0, ab))) break;
          tc_fence_after();
          const uint32_t sKb = b == 0 ? sB : sC;
#pragma unroll
          for (int j = 0; j < VD / 16; ++j)
            mma_bf16_ss(tacc, sdesc_sw128(sA + j * 32, 16, 1024), sdesc_sw128(sKb + j * 32, 16, 1024),
                        idP, j > 0);
          mma_commit(UB(U_P));
          mma_commit(UB(b == 0 ? U_PD0 : U_PD1));
        }
        if (!ok || !mbar_wait(UB(U_PK), qb & 1, ab)) break;
        tc_fence_after();
        if constexpr (LOSS == 0) {
          if (!mbar_wait(UB(U_D), 0, ab) || (qb == 1 && !mbar_wait(UB(U_E), 0, ab))) break;
          tc_fence_after();
          for (int b = 0; b <= qb; ++b) {
            const uint32_t sKb = b == 0 ? sD : sE;
#pragma unroll
            for (int j = 0; j < 8; ++j)
              mma_bf16_ts(tacc, tmem + L::T_S + 64 * b + 8 * j, sdesc_sw128(sKb + j * 2048, 0, 1024),
                          idN, b > 0 || j > 0);
          }
        }
        mma_commit(UB(U_SK));  // (inner product: no S K, this only orders the R epilogue)
        if (!mbar_wait(UB(U_R), 0, ab) || !mbar_wait(UB(LOSS == 0 ? U_D2 : U_D), 0, ab)) break;
        tc_fence_after();
#pragma unroll
        for (int j = 0; j < VD / 16; ++j)
          mma_bf16_ss(tacc, sdesc_sw128(sA + j * 32, 16, 1024), sdesc_sw128(sD + j * 2048, 0, 1024),
                      idN, j > 0);
        for (int b = 0; b <= qb && ok; ++b) {
          ok = mbar_wait(UB(b == 0 ? U_B2 : U_C2), 0, ab);
          if (!ok) break;
          tc_fence_after();
          const uint32_t sVb = b == 0 ? sB : sC;
#pragma unroll
          for (int j = 0; j < 8; ++j)
            mma_bf16_ts(tacc, tmem + L::T_S + 64 * b + 8 * j, sdesc_sw128(sVb + j * 2048, 0, 1024),
                        idN, 1);
        }
        if (!ok) break;
        mma_commit(UB(U_ZQ));
      } while (0);
    }
  } else {
    // ------------------------------------------------ epilogue: warps 2-5, one row per thread
    const int q = warp & 3;
    const int lrow = q * 32 + lane;
    const uint32_t loff = (uint32_t)(q * 32) << 16;
    const int s = 128 * qb + lrow;
    do {
      // eta of the chunk's keys up to this block, exp(L_m) of this block
      for (int t = threadIdx.x - 64; t < 128 * (qb + 1); t += 128)
        f_eta[t] = eta_of(p.beta, (size_t)tokc + t, p.lr_bias);
      if (threadIdx.x - 64 < VD)
        f_eLm[threadIdx.x - 64] = __ldg(p.Em + ((size_t)bc * NB + qb) * VD + (threadIdx.x - 64));
      // (the four warps meet on the mbarrier below before any thread reads these)
      __syncwarp();
      if (lane == 0) mbar_arrive(UB(U_SCAN));
      if (!mbar_wait(UB(U_SCAN), 0, ab)) break;
      // -------- S blocks: P_b packed out of the accumulator with S_sr = P_sr eta_r (r <= s)
      bool ok = true;
      for (int b = 0; b <= qb; ++b) {
        if (!mbar_wait(UB(U_P), b & 1, ab)) { ok = false; break; }
        __syncwarp();
        tc_fence_after();
        const EWeights w{f_eta, s, 128 * b};
        pack_block_to(tmem + loff + L::T_ACC, tmem + loff + L::T_S + 64 * b, q, b == qb, w);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(UB(U_PK));
      }
      if (!ok) break;
      // -------- R = qtilde exp(L_m) - (S K) (MSE) or qtilde exp(L_m), bf16 over slot A
      if (!mbar_wait(UB(U_SK), 0, ab)) break;
      __syncwarp();
      tc_fence_after();
#pragma unroll 1
      for (int c32 = 0; c32 < VD / 32; ++c32) {
        float x[32];
        ld_row32(sA, lrow, 4 * c32, x);
        if constexpr (LOSS == 0) {
          float sk[32];
          tmem_ld32(tmem + loff + L::T_ACC + 32 * c32, sk);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 32; ++j) x[j] = x[j] * f_eLm[32 * c32 + j] - sk[j];
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) x[j] *= f_eLm[32 * c32 + j];
        }
        st_row32(sA, lrow, 4 * c32, x);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(UB(U_R));
      // -------- O = Zq (identity activation)
      if (!mbar_wait(UB(U_ZQ), 0, ab)) break;
      __syncwarp();
      tc_fence_after();
      __nv_bfloat16* orow = p.O + ((size_t)tokc + s) * VD;
#pragma unroll 1
      for (int c32 = 0; c32 < VD / 32; ++c32) {
        float o[32];
        tmem_ld32(tmem + loff + L::T_ACC + 32 * c32, o);
        tmem_wait_ld();
        st_global_bf16x32(orow + 32 * c32, o);
      }
    } while (0);
  }
#undef UB
  tc_fence_before();
  __syncthreads();
  if (bars->abort_flag) __nanosleep(100000);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

size_t align_up(size_t x) { return (x + 1023) & ~size_t(1023); }

template <int NB>
cudaError_t launch_prep(const LayerArgs& a, const VecPrep& o, cudaStream_t s) {
  PrepParams p{};
  p.NC = a.T / a.C;
  p.gamma = a.gamma;
  p.Q = static_cast<const __nv_bfloat16*>(a.Q);
  p.K = static_cast<const __nv_bfloat16*>(a.K);
  p.Qt = static_cast<__nv_bfloat16*>(o.Qt);
  p.Kh = static_cast<__nv_bfloat16*>(o.Kh);
  p.Kt = static_cast<__nv_bfloat16*>(o.Kt);
  p.GC = o.GC;
  p.Em = o.Em;
  p.Lf = o.Lf;
  p.err = a.err;
  vec_prep_kernel<NB><<<a.B * a.H * p.NC * 2, kPrepThreads, 0, s>>>(p);
  count_launches(1);
  return cudaGetLastError();
}

template <int NB, int LOSS>
cudaError_t launch_vec(const LayerArgs& a, cudaStream_t s) {
  constexpr int C = 128 * NB, NV = NB * (NB + 1) / 2;
  const uint64_t rows = (uint64_t)a.B * a.H * a.T;
  const int BH = a.B * a.H, NC = a.T / C;
  // workspace: the decayed operands, then (without W_chunks) the chunk-start states
  const VecPrep pr = vec_prep_carve(a, a.ws, false);
  __nv_bfloat16* Wc = static_cast<__nv_bfloat16*>(
      a.W_chunks ? a.W_chunks
                 : static_cast<void*>(static_cast<uint8_t*>(a.ws) + vec_prep_bytes(a, false)));
  CUtensorMap tK, tKh, tV, tVc, tQt, tKt, tW, tG;
  if (!make_tmap_bf16(&tK, a.K, VD, rows, VD, 64, 128) ||
      !make_tmap_bf16(&tKh, pr.Kh, VD, rows, VD, 64, 128) ||
      !make_tmap_bf16(&tVc, a.V, VD, rows, VD, 64, C) ||
      !make_tmap_bf16(&tV, a.V, VD, rows, VD, 64, 128) ||
      !make_tmap_bf16(&tQt, pr.Qt, VD, rows, VD, 64, 128) ||
      !make_tmap_bf16(&tKt, pr.Kt, VD, (uint64_t)BH * NC * NV * 128, VD, 64, 128) ||
      !make_tmap_bf16(&tW, Wc, VD, (uint64_t)BH * NC * VD, VD, 64, VD) ||
      (a.G_saved && !make_tmap_bf16(&tG, a.G_saved, VD, rows, VD, 64, C)))
    return cudaErrorInvalidValue;
  if (!a.G_saved) tG = tK;  // never used
  VecParams p{};
  p.BH = BH;
  p.T = a.T;
  p.NC = NC;
  p.lr_bias = a.lr_bias;
  p.beta = a.beta;
  p.W0 = a.W0;
  p.GC = pr.GC;
  p.Em = pr.Em;
  p.W_final = a.W_final;
  p.Wc = Wc;
  p.O = static_cast<__nv_bfloat16*>(a.O);
  p.save_g = a.G_saved != nullptr;
  const size_t sm_s = vs_bytes<NB>() + 1024, sm_o = vo_bytes() + 1024;
  auto ks = fwd_vstate_kernel<NB, LOSS>;
  auto ko = fwd_vout_kernel<NB, LOSS>;
  cudaError_t e;
  if ((e = cudaFuncSetAttribute(ks, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm_s)) ||
      (e = cudaFuncSetAttribute(ko, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm_o)))
    return e;
  if ((e = launch_prep<NB>(a, pr, s))) return e;
  ks<<<BH, kVsThreads, sm_s, s>>>(tK, tKh, tVc, tG, p, a.err);
  ko<<<BH * NC * NB, kVoThreads, sm_o, s>>>(tQt, tKt, tK, tV, tW, p, a.err);
  count_launches(2);
  return cudaGetLastError();
}

}  // namespace

size_t vec_prep_bytes(const LayerArgs& a, bool with_L) {
  const size_t rows = (size_t)a.B * a.H * a.T, BH = (size_t)a.B * a.H, NC = a.T / a.C;
  const size_t NB = a.C / 128, NV = NB * (NB + 1) / 2;
  size_t n = align_up(rows * VD * 2) * 2                // Qt, Kh
             + align_up(BH * NC * NV * 128 * VD * 2)    // Kt
             + align_up(BH * NC * VD * 4)               // GC
             + align_up(BH * NC * NB * VD * 4);         // Em
  if (with_L) n += align_up(rows * VD * 4);
  return n;
}

VecPrep vec_prep_carve(const LayerArgs& a, void* base, bool with_L) {
  const size_t rows = (size_t)a.B * a.H * a.T, BH = (size_t)a.B * a.H, NC = a.T / a.C;
  const size_t NB = a.C / 128, NV = NB * (NB + 1) / 2;
  uint8_t* b = static_cast<uint8_t*>(base);
  VecPrep o{};
  o.Qt = b;
  b += align_up(rows * VD * 2);
  o.Kh = b;
  b += align_up(rows * VD * 2);
  o.Kt = b;
  b += align_up(BH * NC * NV * 128 * VD * 2);
  o.GC = reinterpret_cast<float*>(b);
  b += align_up(BH * NC * VD * 4);
  o.Em = reinterpret_cast<float*>(b);
  b += align_up(BH * NC * NB * VD * 4);
  o.Lf = with_L ? reinterpret_cast<float*>(b) : nullptr;
  return o;
}

cudaError_t vec_prep(const LayerArgs& a, const VecPrep& o, cudaStream_t s) {
  return a.C == 128 ? launch_prep<1>(a, o, s) : launch_prep<2>(a, o, s);
}

bool tc_vec_fwd_supported(const LayerArgs& a) {
  return a.dtype == 1 && a.gvec && a.gamma && a.act == 0 && a.dk == VD && a.dv == VD &&
         (a.C == 128 || a.C == 256) && a.T % a.C == 0;
}

// the decayed operands and room for the chunk-start states when the caller keeps none
size_t tc_vec_fwd_workspace(const LayerArgs& a) {
  return vec_prep_bytes(a, false) + (size_t)a.B * a.H * (a.T / a.C) * VD * VD * 2;
}

cudaError_t tc_vec_fwd(const LayerArgs& a, cudaStream_t s) {
  if (a.C == 128) return a.loss == 0 ? launch_vec<1, 0>(a, s) : launch_vec<1, 1>(a, s);
  return a.loss == 0 ? launch_vec<2, 0>(a, s) : launch_vec<2, 1>(a, s);
}

}  // namespace tttk
