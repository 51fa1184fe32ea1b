// tcgen05 forward and backward of the chunkwise TTT layer with a per-feature (vector) decay,
// identity activation, d_k = d_v = 64 (bf16 operands, fp32 state and accumulators).
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
// Forward, three kernels:
//   prep   : persistent, one CTA per SM over (batch, head, chunk, half of the features) units,
//            the next two units' gamma, q and k in flight to shared memory while the current
//            one runs: the per-feature log-decay scan and every decayed operand (qtilde, ktilde
//            per reference token, Khat) written once as bf16, with exp(L_C) and exp(L_m); the
//            backward reuses it (and keeps L itself).
//   vstate : one CTA per (batch, head) walks the chunks with the fp32 state in TMEM: Z = K W0,
//            -eta G, W = diag(exp(L_C)) W + Khat^T (-eta G); K and Khat arrive by TMA.
//   vout   : one CTA per (batch, head, chunk, 128-query block), two per SM:
//            P = qtilde ktilde^T, S = P * eta (causal), R, O = R W0 + S V.
// Backward (equations above its kernels): prep again (keeping L), vout for R alone, a serial
// adjoint pass, a key-side and a query-side chunk-parallel kernel, and the decay-gradient scan.
#include <cuda_bf16.h>
#include <math.h>

#include <algorithm>

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
  const float* W0;      // [BH, 64, 64] (or [H, 64, 64]: block bh % w0_mod)
  int w0_mod;
  const float* GC;      // [BH, NC, 64] exp(L_C)
  const float* Em;      // [BH, NC, NB, 64] exp(L_m)
  float* W_final;       // nullable
  __nv_bfloat16* Wc;    // [BH, NC, 64, 64]
  __nv_bfloat16* O;
  int save_g;
  int save_r;  // the readout also stores R (for the backward)
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
  __nv_bfloat16* Qt2;  // nullable (C = 256): second-block queries against the first reference
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
__device__ __forceinline__ void prefetch_l2(const void* a) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(a));
}
__device__ __forceinline__ void prefetch_l1(const void* a) {
  asm volatile("prefetch.global.L1 [%0];" ::"l"(a));
}
// Row stores of a warp's 32 rows (this lane's row in v; row r goes to dst0 + r * ld) through a
// 4 KB tile of shared memory: the lanes write their rows in 16-byte groups, then every store
// instruction writes whole rows (four 128-byte float32 rows, or eight 64-byte bf16 rows) instead
// of one 16-byte piece of each of 32 rows. The groups are rotated by the row so that neither the
// row writes nor the reads collide in a bank.
__device__ __forceinline__ void store_rows32_f32(float* tile, const float (&v)[32], float* dst0,
                                                 size_t ld, int lane) {
  float4* t4 = reinterpret_cast<float4*>(tile + lane * 32);
#pragma unroll
  for (int c = 0; c < 8; ++c)
    t4[(c + lane) & 7] = make_float4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
  __syncwarp();
  const int rs = lane >> 3, c = lane & 7;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int r = 4 * i + rs;
    reinterpret_cast<float4*>(dst0 + (size_t)r * ld)[c] =
        reinterpret_cast<const float4*>(tile + r * 32)[(c + r) & 7];
  }
  __syncwarp();
}
__device__ __forceinline__ void store_rows32_bf16(float* tile, const float (&v)[32],
                                                  __nv_bfloat16* dst0, size_t ld, int lane) {
  // row r's four groups sit at (c + 4 (r & 1) + (r >> 1)) & 7 of its 128-byte tile row
  auto slot = [](int c, int r) { return (c + 4 * (r & 1) + (r >> 1)) & 7; };
  uint4* t4 = reinterpret_cast<uint4*>(tile + lane * 32);
#pragma unroll
  for (int c = 0; c < 4; ++c)
    t4[slot(c, lane)] = make_uint4(pack_bf16x2(v[8 * c], v[8 * c + 1]),
                                   pack_bf16x2(v[8 * c + 2], v[8 * c + 3]),
                                   pack_bf16x2(v[8 * c + 4], v[8 * c + 5]),
                                   pack_bf16x2(v[8 * c + 6], v[8 * c + 7]));
  __syncwarp();
  const int rs = lane >> 2, c = lane & 3;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = 8 * i + rs;
    reinterpret_cast<uint4*>(dst0 + (size_t)r * ld)[c] =
        reinterpret_cast<const uint4*>(tile + r * 32)[slot(c, r)];
  }
  __syncwarp();
}

// Eight bf16 of u (x, y, z, w in order) as float32.
__device__ __forceinline__ void unpack_bf16x8(const uint4& u, float* v) {
  v[0] = bf16lo(u.x); v[1] = bf16hi(u.x); v[2] = bf16lo(u.y); v[3] = bf16hi(u.y);
  v[4] = bf16lo(u.z); v[5] = bf16hi(u.z); v[6] = bf16lo(u.w); v[7] = bf16hi(u.w);
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

constexpr int kPrepSeg = 16;  // slices per chunk (decay-gradient scan)
constexpr int kPrepThreads = 128;  // 8 feature quads (32 features) x 16 slices

// 16-byte asynchronous global -> shared copies (no register staging), in commit groups.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// The prep is persistent: one CTA per SM walks units u = (batch, head, chunk, half of the
// features) with a stride of the grid. A unit's gamma, q and k rows reach shared memory through
// asynchronous copies issued two units ahead (three stages), so an SM's DRAM traffic for the
// next units overlaps the exponentials and stores of the current one. Thread (f = four adjacent
// key features, seg = one of 64 slices of the chunk); the slice sums are scanned by eight warps
// (one per feature quad) with shuffles.
constexpr int kPrepNseg = 64;
constexpr int kPrepPThreads = 8 * kPrepNseg;
constexpr int kPrepStages = 3;
template <int NB>
__host__ __device__ constexpr uint32_t prep_stage_bytes() { return 128 * NB * (128 + 2 * 64); }  // gamma, q, k

template <int NB>
__global__ void __launch_bounds__(kPrepPThreads, 1) vec_prep_kernel(const PrepParams p, int nunits) {
  constexpr int C = 128 * NB, SEG = C / kPrepNseg, NV = NB * (NB + 1) / 2;
  constexpr uint32_t GB = C * 128, QB = C * 64, STAGE = prep_stage_bytes<NB>();
  extern __shared__ __align__(16) uint8_t prep_smem[];
  __shared__ float4 tot[kPrepNseg][8];  // per-slice sums of log gamma
  __shared__ float4 pre[kPrepNseg][8];  // their exclusive prefix sums
  const int f = threadIdx.x & 7, seg = threadIdx.x >> 3;
  const uint32_t s_base = smem_u32(prep_smem);
  // unit u into stage st: C rows of 32 gamma (8 x 16 bytes), of 32 q and of 32 k (4 x 16 bytes
  // each); one commit group per call, empty past the last unit
  auto issue = [&](int u, int st) {
    if (u < nunits) {
      const size_t e0 = (size_t)(u >> 1) * C * VD + 32 * (u & 1);
      const uint8_t* g = reinterpret_cast<const uint8_t*>(p.gamma + e0);
      const uint8_t* q = reinterpret_cast<const uint8_t*>(p.Q + e0);
      const uint8_t* k = reinterpret_cast<const uint8_t*>(p.K + e0);
      const uint32_t s0 = s_base + st * STAGE;
      for (int i = threadIdx.x; i < C * 8; i += kPrepPThreads)
        cp_async16(s0 + i * 16, g + (size_t)(i >> 3) * VD * 4 + (i & 7) * 16);
      for (int i = threadIdx.x; i < C * 4; i += kPrepPThreads) {
        const size_t off = (size_t)(i >> 2) * VD * 2 + (i & 3) * 16;
        cp_async16(s0 + GB + i * 16, q + off);
        cp_async16(s0 + GB + QB + i * 16, k + off);
      }
    }
    cp_async_commit();
  };
  bool range = false;
  const int stride = gridDim.x;
  issue(blockIdx.x, 0);
  issue(blockIdx.x + stride, 1);
  int st = 0;
  for (int u = blockIdx.x; u < nunits; u += stride) {
    cp_async_wait<1>();  // this thread's copies of unit u have landed ...
    __syncthreads();     // ... and every thread's
    const uint8_t* sb = prep_smem + st * STAGE;
    const float4* gs = reinterpret_cast<const float4*>(sb) + seg * SEG * 8 + f;
    const uint2* qs = reinterpret_cast<const uint2*>(sb + GB) + seg * SEG * 8 + f;
    const uint2* ks = reinterpret_cast<const uint2*>(sb + GB + QB) + seg * SEG * 8 + f;
    float4 lg[SEG];
    uint2 qv[SEG], kv[SEG];
#pragma unroll
    for (int t = 0; t < SEG; ++t) {
      lg[t] = gs[t * 8];
      qv[t] = qs[t * 8];
      kv[t] = ks[t * 8];
    }
    // the stage of the previous unit: every thread has read it before the barrier above
    issue(u + 2 * stride, st == 0 ? 2 : st - 1);
    st = st == kPrepStages - 1 ? 0 : st + 1;

    const int fq = (u & 1) * 8 + f;        // feature quad 0..15
    const size_t bc = u >> 1;              // bh * NC + c
    const size_t r0 = bc * C + seg * SEG;  // first token row of this slice
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
    if (threadIdx.x < 256) {
      // warp w: exclusive prefix over the 64 slices of feature quad w, two slices a lane
      const int w = threadIdx.x >> 5, j = threadIdx.x & 31;
      const float4 a = tot[2 * j][w], b = tot[2 * j + 1][w];
      float4 inc = add4(a, b);
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) {
        const float4 o = make_float4(__shfl_up_sync(0xffffffffu, inc.x, d),
                                     __shfl_up_sync(0xffffffffu, inc.y, d),
                                     __shfl_up_sync(0xffffffffu, inc.z, d),
                                     __shfl_up_sync(0xffffffffu, inc.w, d));
        if (j >= d) inc = add4(o, inc);
      }
      float4 ex = make_float4(__shfl_up_sync(0xffffffffu, inc.x, 1),
                              __shfl_up_sync(0xffffffffu, inc.y, 1),
                              __shfl_up_sync(0xffffffffu, inc.z, 1),
                              __shfl_up_sync(0xffffffffu, inc.w, 1));
      if (j == 0) ex = make_float4(0.f, 0.f, 0.f, 0.f);
      pre[2 * j][w] = ex;
      pre[2 * j + 1][w] = add4(ex, a);
    }
    __syncthreads();
    // L_t = (prefix of the slice) + (running sum inside it). Slice boundaries fall on the
    // reference tokens' successors (64 and 192 for C = 256, 64 for C = 128), and L_m and L_C are
    // formed as the same two-term sum as L_t at those tokens, so the exponent at the reference
    // token is exactly 0.
    const float4 Lstart = pre[seg][f];
    const float4 LC = add4(pre[kPrepNseg - 1][f], tot[kPrepNseg - 1][f]);
    float4 Lm[NB];
#pragma unroll
    for (int qb = 0; qb < NB; ++qb) {
      const int kk = (128 * qb + 64) / SEG - 1;
      Lm[qb] = add4(pre[kk][f], tot[kk][f]);
    }
    const int kb = seg * SEG / 128;
    float4 l = make_float4(0.f, 0.f, 0.f, 0.f);
    uint2* qt = reinterpret_cast<uint2*>(p.Qt + r0 * VD) + fq;
    uint2* kh = reinterpret_cast<uint2*>(p.Kh + r0 * VD) + fq;
    const float4 lmk = kb ? Lm[NB - 1] : Lm[0];  // kb < NB <= 2
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
      if (NB == 2 && kb == 1 && p.Qt2) {  // exponents <= 0: the reference precedes the token
        const float4 m = Lm[0];
        reinterpret_cast<uint2*>(p.Qt2 + (bc * 128 + tr) * VD)[fq] =
            scale4(qv[t], make_float4(L.x - m.x, L.y - m.y, L.z - m.z, L.w - m.w), range);
      }
    }
    if (seg == 0) {
      reinterpret_cast<float4*>(p.GC + bc * VD)[fq] =
          make_float4(__expf(LC.x), __expf(LC.y), __expf(LC.z), __expf(LC.w));
#pragma unroll
      for (int qb = 0; qb < NB; ++qb)
        reinterpret_cast<float4*>(p.Em + (bc * NB + qb) * VD)[fq] = make_float4(
            __expf(Lm[qb].x), __expf(Lm[qb].y), __expf(Lm[qb].z), __expf(Lm[qb].w));
    }
  }
  cp_async_wait<0>();  // no copy in flight when the CTA exits
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
      const float4* src =
          reinterpret_cast<const float4*>(p.W0 + ((size_t)(bh % p.w0_mod) * VD + lrow) * VD + col);
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

// MODE 0: the forward's O. MODE 1 (backward): R alone, stored through tmR; with the inner-product
// loss R = qtilde exp(L_m) needs no scores at all.
template <int NB, int LOSS, int MODE>
__global__ void __launch_bounds__(kVoThreads, 2)
    fwd_vout_kernel(const __grid_constant__ CUtensorMap tmQt, const __grid_constant__ CUtensorMap tmKt,
                    const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                    const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmR,
                    const VecParams p, unsigned* err) {
  constexpr int C = 128 * NB, NV = NB * (NB + 1) / 2;
  constexpr bool NEED_S = !(MODE == 1 && LOSS == 1);
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
      if (NEED_S) {
        load(sB, &tmKt, U_B, kt_row(0));
        if (qb == 1) load(sC, &tmKt, U_C, kt_row(1));
      }
      if (LOSS == 0) {
        load(sD, &tmK, U_D, tokc);
        if (qb == 1) load(sE, &tmK, U_E, tokc + 128);
      } else if (MODE == 0) {
        load_w(U_D);
      }
      if constexpr (MODE == 0) {
        // slots freed by the score MMAs take the values, the S K slot takes W0
        if (mbar_wait(UB(U_PD0), 0, ab)) load(sB, &tmV, U_B2, tokc);
        if (qb == 1 && mbar_wait(UB(U_PD1), 0, ab)) load(sC, &tmV, U_C2, tokc + 128);
        if (LOSS == 0 && mbar_wait(UB(U_SK), 0, ab)) load_w(U_D2);
      }
      if ((MODE == 1 || p.save_r) && mbar_wait(UB(U_R), 0, ab)) {
        tma_store_2d(&tmR, sA, 0, tokc + 128 * qb);
        bulk_commit();
        bulk_wait0();
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idP = idesc_bf16(128, 128, 0, 0);  // qtilde ktilde^T: both K-major
      const uint32_t idN = idesc_bf16(128, VD, 0, 1);   // S K, S V, R W0: MN-major B
      const uint32_t tacc = tmem + L::T_ACC;
      do {
        if (!NEED_S) break;
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
        if (MODE == 1) break;
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
      for (int b = 0; b <= qb && NEED_S; ++b) {
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
      if (!mbar_wait(UB(NEED_S ? U_SK : U_A), 0, ab)) break;
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
      if (MODE == 1) break;
      // -------- O = Zq (identity activation)
      if (!mbar_wait(UB(U_ZQ), 0, ab)) break;
      __syncwarp();
      tc_fence_after();
      // the rows go out through slot B (V_0, read by no product any more)
      float* otile = reinterpret_cast<float*>(smem + L::OFF_B) + q * 1024;
      __nv_bfloat16* orow0 = p.O + ((size_t)tokc + s - lane) * VD;
#pragma unroll 1
      for (int c32 = 0; c32 < VD / 32; ++c32) {
        float o[32];
        tmem_ld32(tmem + loff + L::T_ACC + 32 * c32, o);
        tmem_wait_ld();
        store_rows32_bf16(otile, o, orow0 + 32 * c32, VD, lane);
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

// ============================================================================== backward
// With Lambda the adjoint of a chunk's end state, dO its output gradient and the forward's
// quantities of that chunk (identity activation):
//   Lambda_prev = diag(exp(L_C)) Lambda + R^T dO - K^T (eta * (Khat Lambda))     (MSE)
//   Lambda_prev = diag(exp(L_C)) Lambda + R^T dO                                 (inner product)
//   dG  = -S^T dO - eta * X,  X = Khat Lambda,   dV = -dG
//   dK  = dG W0^T (MSE) + exp(L_m - L) * ((eta dS)^T qtilde) - eta exp(L_C - L) * (G Lambda^T)
//   dQ  = exp(L - L_m) * (dO (diag(exp(L_m)) W0)^T + (eta dS) ktilde),   dS_sr = -dO_s . G_r
//   deta_r = sum_s dS_sr P_sr - X_r . G_r
// and, L entering every decayed factor, its gradient per token and feature is
//   dL_t = q_t * dQ_t - k_t * (dK_t - (dG W0^T)_t) + [t = C-1] (sum_r k_r * dKhat_r
//          + exp(L_C) * rowsum(W0 * Lambda))
// (dKhat the Khat term of dK), whose reverse running sum over the chunk is d log gamma.

// ------------------------------------------------------------------ serial adjoint pass
template <int NB>
struct VbL {
  static constexpr int C = 128 * NB;
  static constexpr uint32_t KBUF = C * 128;
  static constexpr uint32_t OFF_K = 0;            // two K chunks
  static constexpr uint32_t OFF_KH = 2 * KBUF;    // Khat
  static constexpr uint32_t OFF_R = 3 * KBUF;     // R
  static constexpr uint32_t OFF_DO = 4 * KBUF;    // dO
  static constexpr uint32_t OFF_UX = 5 * KBUF;    // -eta X
  static constexpr uint32_t OFF_L = 6 * KBUF;     // bf16 Lambda, 64 x 64
  static constexpr uint32_t OFF_BAR = OFF_L + VD * 128;
  static constexpr uint32_t T_L = 0, T_X = 64;
};
struct __align__(8) VbBars {
  uint64_t k_full[2], k_free[2], kh_full, kh_free, rd_full, rd_free, x_full, ux_ready, lam_ready,
      acc_full;
  uint32_t tmem_base;
  int abort_flag;
};
template <int NB>
constexpr uint32_t vb_bytes() { return VbL<NB>::OFF_BAR + sizeof(VbBars); }

struct VbParams {
  int T, NC;
  float lr_bias;
  const float* beta;
  const float* GC;             // [BH, NC, 64]
  const float* dW_final;       // nullable
  const __nv_bfloat16* Wc;     // [BH, NC, 64, 64]
  __nv_bfloat16* Lam;          // [BH, NC, 64, 64] chunk-end adjoints
  float* dW0;                  // [BH, 64, 64]
  float* wl;                   // nullable: [BH, NC, 2, 64] half-row sums of W0 * Lambda
};

template <int NB, int LOSS>
__global__ void __launch_bounds__(kVsThreads, 1)
    bwd_vstate_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmKh,
                      const __grid_constant__ CUtensorMap tmR, const __grid_constant__ CUtensorMap tmdO,
                      const VbParams p, unsigned* err) {
  using L = VbL<NB>;
  constexpr int C = L::C;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  const uint32_t sb = smem_u32(smem);
  const uint32_t sK = sb + L::OFF_K, sKH = sb + L::OFF_KH, sR = sb + L::OFF_R, sDO = sb + L::OFF_DO,
                 sUX = sb + L::OFF_UX, sL = sb + L::OFF_L;
  VbBars* bars = reinterpret_cast<VbBars*>(smem + L::OFF_BAR);
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
    mbar_init(BAR(kh_full), 1);
    mbar_init(BAR(kh_free), 1);
    mbar_init(BAR(rd_full), 1);
    mbar_init(BAR(rd_free), 1);
    mbar_init(BAR(x_full), 1);
    mbar_init(BAR(ux_ready), kEpi);
    mbar_init(BAR(lam_ready), kEpi);
    mbar_init(BAR(acc_full), 1);
    bars->abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(BAR(tmem_base), 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  auto row0 = [&](int cc) { return bh * p.T + cc * C; };

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      auto load_k = [&](int cc, int x) {
        mbar_arrive_expect_tx(BAR(k_full[x]), L::KBUF);
        for (int h = 0; h < NB; ++h)
          tma_load_2d(sK + x * L::KBUF + h * PANEL, &tmK, BAR(k_full[x]), 0, row0(cc) + 128 * h);
      };
      auto load_kh = [&](int cc) {
        mbar_arrive_expect_tx(BAR(kh_full), L::KBUF);
        for (int h = 0; h < NB; ++h)
          tma_load_2d(sKH + h * PANEL, &tmKh, BAR(kh_full), 0, row0(cc) + 128 * h);
      };
      auto load_rd = [&](int cc) {
        mbar_arrive_expect_tx(BAR(rd_full), 2 * L::KBUF);
        for (int h = 0; h < NB; ++h) {
          tma_load_2d(sR + h * PANEL, &tmR, BAR(rd_full), 0, row0(cc) + 128 * h);
          tma_load_2d(sDO + h * PANEL, &tmdO, BAR(rd_full), 0, row0(cc) + 128 * h);
        }
      };
      if (LOSS == 0) {
        load_kh(NC - 1);
        load_k(NC - 1, 0);
      }
      load_rd(NC - 1);
      if (LOSS == 0 && NC > 1) load_k(NC - 2, 1);
      for (int j = 0; j < NC; ++j) {
        const int c = NC - 1 - j;
        if (!mbar_wait(BAR(rd_free), j & 1, ab)) break;
        if (c >= 1) load_rd(c - 1);
        if (LOSS == 0) {
          if (!mbar_wait(BAR(kh_free), j & 1, ab)) break;
          if (c >= 1) load_kh(c - 1);
          if (c >= 2) {
            if (!mbar_wait(BAR(k_free[j & 1]), (j >> 1) & 1, ab)) break;
            load_k(c - 2, j & 1);
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------- MMA issue: += R^T dO, X = Khat Lambda, += K^T (-eta X)
    if (lane == 0) {
      const uint32_t idX = idesc_bf16(128, VD, 0, 1);  // K-major A, MN-major B
      const uint32_t idT = idesc_bf16(128, VD, 1, 1);  // MN-major A (R^T, K^T) and B
      auto tok = [&](uint32_t base, int jj) { return base + (jj / 8) * PANEL + (jj % 8) * 2048; };
      for (int j = 0; j < NC; ++j) {
        const int x = j & 1;
        if (!mbar_wait(BAR(lam_ready), j & 1, ab) || !mbar_wait(BAR(rd_full), j & 1, ab)) break;
        tc_fence_after();
        // M = 128 over the 64 key features: the upper half of the result lanes repeats the lower
        for (int jj = 0; jj < C / 16; ++jj)
          mma_bf16_ss(tmem + L::T_L, sdesc_sw128(tok(sR, jj), 0, 1024),
                      sdesc_sw128(tok(sDO, jj), 0, 1024), idT, 1);
        mma_commit(BAR(rd_free));
        if constexpr (LOSS == 0) {
          if (!mbar_wait(BAR(kh_full), j & 1, ab)) break;
          tc_fence_after();
          for (int b = 0; b < NB; ++b) {
#pragma unroll
            for (int jj = 0; jj < VD / 16; ++jj)
              mma_bf16_ss(tmem + L::T_X + VD * b, sdesc_sw128(sKH + b * PANEL + jj * 32, 16, 1024),
                          sdesc_sw128(sL + jj * 2048, 0, 1024), idX, jj > 0);
          }
          mma_commit(BAR(x_full));
          mma_commit(BAR(kh_free));
          if (!mbar_wait(BAR(ux_ready), j & 1, ab) || !mbar_wait(BAR(k_full[x]), (j >> 1) & 1, ab))
            break;
          tc_fence_after();
          for (int jj = 0; jj < C / 16; ++jj)
            mma_bf16_ss(tmem + L::T_L, sdesc_sw128(tok(sK + x * L::KBUF, jj), 0, 1024),
                        sdesc_sw128(tok(sUX, jj), 0, 1024), idT, 1);
          mma_commit(BAR(k_free[x]));
        }
        mma_commit(BAR(acc_full));
      }
    }
  } else {
    // ------------------------------------------------------------------ epilogue
    const int ew = warp - 2, g = ew / 4, q = warp & 3;
    const int lrow = q * 32 + lane;
    const uint32_t loff = (uint32_t)(q * 32) << 16;
    const bool w_rows = q * 32 < VD;
    const int col = 32 * g;
    const size_t bhs = (size_t)bh;
    for (int j = 0; j < NC; ++j) {
      const int c = NC - 1 - j;
      const size_t bc = bhs * NC + c;
      if (w_rows) {
        float lam[32];
        if (j == 0) {
          if (p.dW_final) {
            const float4* src =
                reinterpret_cast<const float4*>(p.dW_final + (bhs * VD + lrow) * VD + col);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              const float4 v = src[k];
              lam[4 * k] = v.x; lam[4 * k + 1] = v.y; lam[4 * k + 2] = v.z; lam[4 * k + 3] = v.w;
            }
          } else {
#pragma unroll
            for (int k = 0; k < 32; ++k) lam[k] = 0.f;
          }
        } else {
          tmem_ld32(tmem + loff + L::T_L + col, lam);
          tmem_wait_ld();
        }
        st_row32(sL, lrow, 4 * g, lam);
        st_global_bf16x32(p.Lam + (bc * VD + lrow) * VD + col, lam);
        if (p.wl) {
          const uint4* w4 = reinterpret_cast<const uint4*>(p.Wc + (bc * VD + lrow) * VD + col);
          float acc = 0.f;
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint4 w = __ldg(w4 + k);
            acc += bf16lo(w.x) * lam[8 * k] + bf16hi(w.x) * lam[8 * k + 1] +
                   bf16lo(w.y) * lam[8 * k + 2] + bf16hi(w.y) * lam[8 * k + 3] +
                   bf16lo(w.z) * lam[8 * k + 4] + bf16hi(w.z) * lam[8 * k + 5] +
                   bf16lo(w.w) * lam[8 * k + 6] + bf16hi(w.w) * lam[8 * k + 7];
          }
          p.wl[(bc * 2 + g) * VD + lrow] = acc;
        }
        const float gc = __ldg(p.GC + bc * VD + lrow);
#pragma unroll
        for (int k = 0; k < 32; ++k) lam[k] *= gc;
        tmem_st32(tmem + loff + L::T_L + col, lam);
        tmem_wait_st();
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(lam_ready));
      if constexpr (LOSS == 0) {
        float eta[NB];
#pragma unroll
        for (int b = 0; b < NB; ++b) eta[b] = eta_of(p.beta, (size_t)row0(c) + 128 * b + lrow, p.lr_bias);
        if (!mbar_wait(BAR(x_full), j & 1, ab)) break;
        __syncwarp();
        tc_fence_after();
#pragma unroll
        for (int b = 0; b < NB; ++b) {
          float xv[32];
          tmem_ld32(tmem + loff + L::T_X + VD * b + col, xv);
          tmem_wait_ld();
          const float ne = -eta[b];
#pragma unroll
          for (int k = 0; k < 32; ++k) xv[k] *= ne;
          st_row32(sUX, 128 * b + lrow, 4 * g, xv);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(BAR(ux_ready));
      }
      if (!mbar_wait(BAR(acc_full), j & 1, ab)) break;
      __syncwarp();
      tc_fence_after();
    }
    if (w_rows && !*ab.flag) {
      float lam[32];
      tmem_ld32(tmem + loff + L::T_L + col, lam);
      tmem_wait_ld();
      float4* dst = reinterpret_cast<float4*>(p.dW0 + (bhs * VD + lrow) * VD + col);
#pragma unroll
      for (int k = 0; k < 8; ++k) dst[k] = make_float4(lam[4 * k], lam[4 * k + 1], lam[4 * k + 2], lam[4 * k + 3]);
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

// Sum over the 32 lanes of each of 32 columns (v[c] of every lane): afterwards lane l holds the
// sum of column l in v[0].
__device__ __forceinline__ void colsum32(float (&v)[32], int lane) {
#pragma unroll
  for (int w = 16; w >= 1; w >>= 1) {
    const bool upper = (lane & w) != 0;
#pragma unroll
    for (int c = 0; c < w; ++c) {
      const float send = upper ? v[c] : v[c + w];
      const float keep = upper ? v[c + w] : v[c];
      v[c] = keep + __shfl_xor_sync(0xffffffffu, send, w);
    }
  }
}

struct VgParams {
  int BH, T, NC;
  float lr_bias;
  const float* beta;
  const float* Lf;        // [BH, T, 64] chunk-local L
  const float* Em;        // [BH, NC, NB, 64]
  const __nv_bfloat16* Q;
  const __nv_bfloat16* K;
  __nv_bfloat16 *dQ, *dK, *dV;
  float* dbeta;
  float* dLk;             // nullable: -k * (dK - dG W0^T), [BH, T, 64]
  float* dLq;             // nullable: q * dQ, [BH, T, 64]
  float* colk;            // nullable: [BH, NC, NB, 4, 64] partial column sums of k * dKhat
};

// ------------------------------------------------------------- key side: dK, dV, dbeta
// One CTA per (batch, head, chunk, 128-key block kb), two per SM. Every query block qb >= kb
// is taken in two halves of 64 queries, with both operands referred to the key block's
// reference token m(kb): ktilde (kb, kb) for the keys and, for the queries, qtilde (qb = kb) or
// the prep pass's second-block copy against m(0) (qb = kb + 1, kb = 0), so one accumulator
// holds (eta dS^T) qtilde' over all query blocks and dK^S = exp(L_m(kb) - L) * that.
// Shared memory (16 KB panels unless stated): K (MSE: the G product; then a query-half slot),
// V (then G, bf16, in place), Khat (then dG, bf16), W0 and Lambda (8 KB each), ktilde (kb, kb),
// a query-half slot (qtilde' half, then dO half, 8 KB each). Query halves alternate between the
// two slots. TMEM (256 columns): [0,64) G (MSE), then the dK^S accumulator; [64,128) X, then
// eta X and the dG accumulator; [128,192) P^T of a half, S^T packed over it; [192,256) G dO^T
// of a half, eta dS^T packed over it; after the last half G Lambda^T and dG W0^T go to
// [128,192) and [192,256).
struct KgL {
  static constexpr uint32_t OFF_K = 0, OFF_V = PANEL, OFF_KH = 2 * PANEL, OFF_KT = 3 * PANEL,
                            OFF_HA = 4 * PANEL, OFF_W = 5 * PANEL, OFF_L = OFF_W + VD * 128;
  static constexpr uint32_t HALF = 64 * 128;               // 64 rows x 64 bf16
  static constexpr uint32_t OFF_F = OFF_L + VD * 128;      // L_m(kb)[64], L_C[64]
  static constexpr uint32_t OFF_BAR = OFF_F + 2 * VD * 4;
  static constexpr uint32_t T_DKS = 0, T_DG = 64, T_P = 128, T_DS = 192;
};
enum { K_LDA, K_LDH0, K_LDH1, K_GA, K_GRDY, K_PS, K_PK, K_ST0, K_ST1, K_GL, K_DGRDY, K_DGW, K_F,
       K_NBARS };
struct __align__(8) KgBars {
  uint64_t b[K_NBARS];
  uint32_t tmem_base;
  int abort_flag;
};
constexpr uint32_t kg_bytes() { return KgL::OFF_BAR + sizeof(KgBars); }

// SG: the tmV operand is the forward's saved G (bf16), so G is neither recomputed nor negated.
template <int NB, int LOSS, bool SG>
__global__ void __launch_bounds__(kVoThreads, 2)
    bwd_vkey_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmKh,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmKt,
                    const __grid_constant__ CUtensorMap tmQh, const __grid_constant__ CUtensorMap tmQ2h,
                    const __grid_constant__ CUtensorMap tmdOh, const __grid_constant__ CUtensorMap tmW,
                    const __grid_constant__ CUtensorMap tmLam, const VgParams p, unsigned* err) {
  constexpr int C = 128 * NB, NV = NB * (NB + 1) / 2;
  using L = KgL;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  const uint32_t sb = smem_u32(smem);
  const uint32_t sK = sb + L::OFF_K, sV = sb + L::OFF_V, sKH = sb + L::OFF_KH,
                 sKT = sb + L::OFF_KT, sW = sb + L::OFF_W, sL = sb + L::OFF_L;
  // query half h lives in slot h & 1: the half slot, or the K panel once K is no longer read
  auto sQh = [&](int h) { return (h & 1) ? sK : sb + L::OFF_HA; };
  auto sDOh = [&](int h) { return sQh(h) + L::HALF; };
  float* f_Lm = reinterpret_cast<float*>(smem + L::OFF_F);
  float* f_LC = f_Lm + VD;
  KgBars* bars = reinterpret_cast<KgBars*>(smem + L::OFF_BAR);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int per_c = p.BH * NB;
  const int c = p.NC - 1 - (int)blockIdx.x / per_c;
  const int rem = (int)blockIdx.x % per_c;
  const int bh = rem / NB, kb = rem % NB;
  const int NH = 2 * (NB - kb);  // query halves at or after this key block
  const int tokc = bh * p.T + c * C;
  const int bc = bh * p.NC + c;
  Abort ab{&bars->abort_flag, err};
#define KB(i) smem_u32(&bars->b[i])
  if (threadIdx.x == 0) {
    for (int i = 0; i < K_NBARS; ++i)
      mbar_init(KB(i), (i == K_GRDY || i == K_PK || i == K_DGRDY || i == K_F) ? 4 : 1);
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

  if (warp == 0) {
    if (lane == 0) {
      const int tk = tokc + 128 * kb;
      constexpr bool kmma = LOSS == 0 && !SG;  // G = K W0 - V by MMA
      mbar_arrive_expect_tx(KB(K_LDA), (kmma ? 4 : 3) * PANEL + 2 * VD * 128);
      if (kmma) tma_load_2d(sK, &tmK, KB(K_LDA), 0, tk);
      tma_load_2d(sKH, &tmKh, KB(K_LDA), 0, tk);
      tma_load_2d(sV, &tmV, KB(K_LDA), 0, tk);
      tma_load_2d(sKT, &tmKt, KB(K_LDA), 0, (bc * NV + kb * (kb + 1) / 2 + kb) * 128);
      tma_load_2d(sW, &tmW, KB(K_LDA), 0, bc * VD);
      tma_load_2d(sL, &tmLam, KB(K_LDA), 0, bc * VD);
      for (int h = 0; h < NH; ++h) {
        const int qb = kb + (h >> 1), half = h & 1, bar = (h & 1) ? K_LDH1 : K_LDH0;
        // the slot is free once the half two before it has been multiplied (or, for the K
        // panel's first use, once G = K W0 has read K)
        if (h >= 2 && !mbar_wait(KB((h & 1) ? K_ST1 : K_ST0), ((h - 2) >> 1) & 1, ab)) break;
        if (h == 1 && kmma && !mbar_wait(KB(K_GA), 0, ab)) break;
        mbar_arrive_expect_tx(KB(bar), 2 * L::HALF);
        if (qb == kb)
          tma_load_2d(sQh(h), &tmQh, KB(bar), 0, tokc + 128 * qb + 64 * half);
        else
          tma_load_2d(sQh(h), &tmQ2h, KB(bar), 0, bc * 128 + 64 * half);
        tma_load_2d(sDOh(h), &tmdOh, KB(bar), 0, tokc + 128 * qb + 64 * half);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idKM = idesc_bf16(128, VD, 0, 1);  // K-major A, MN-major B, N = 64
      const uint32_t idKK = idesc_bf16(128, VD, 0, 0);  // both K-major, N = 64
      do {
        if (!mbar_wait(KB(K_LDA), 0, ab)) break;
        tc_fence_after();
        if constexpr (LOSS == 0 && !SG) {
#pragma unroll
          for (int jj = 0; jj < 4; ++jj)
            mma_bf16_ss(tmem + L::T_DKS, sdesc_sw128(sK + jj * 32, 16, 1024),
                        sdesc_sw128(sW + jj * 2048, 0, 1024), idKM, jj > 0);
        }
#pragma unroll
        for (int jj = 0; jj < 4; ++jj)
          mma_bf16_ss(tmem + L::T_DG, sdesc_sw128(sKH + jj * 32, 16, 1024),
                      sdesc_sw128(sL + jj * 2048, 0, 1024), idKM, jj > 0);
        mma_commit(KB(K_GA));
        if (!mbar_wait(KB(K_GRDY), 0, ab)) break;
        bool ok = true;
        for (int h = 0; h < NH && ok; ++h) {
          if (!(ok = mbar_wait(KB((h & 1) ? K_LDH1 : K_LDH0), (h >> 1) & 1, ab))) break;
          // the previous half's products, which read the packed columns, are complete
          if (h > 0 && !(ok = mbar_wait(KB(((h - 1) & 1) ? K_ST1 : K_ST0), ((h - 1) >> 1) & 1, ab)))
            break;
          tc_fence_after();
          const uint32_t sQ = sQh(h), sD = sDOh(h);
#pragma unroll
          for (int jj = 0; jj < 4; ++jj)
            mma_bf16_ss(tmem + L::T_P, sdesc_sw128(sKT + jj * 32, 16, 1024),
                        sdesc_sw128(sQ + jj * 32, 16, 1024), idKK, jj > 0);
#pragma unroll
          for (int jj = 0; jj < 4; ++jj)
            mma_bf16_ss(tmem + L::T_DS, sdesc_sw128(sV + jj * 32, 16, 1024),
                        sdesc_sw128(sD + jj * 32, 16, 1024), idKK, jj > 0);
          mma_commit(KB(K_PS));
          if (!(ok = mbar_wait(KB(K_PK), h & 1, ab))) break;
          tc_fence_after();
          // dG accumulator += S^T dO and dK^S accumulator += (eta dS^T) qtilde' (A packed in
          // TMEM, K = the half's 64 queries)
#pragma unroll
          for (int jj = 0; jj < 4; ++jj)
            mma_bf16_ts(tmem + L::T_DG, tmem + L::T_P + 8 * jj, sdesc_sw128(sD + jj * 2048, 0, 1024),
                        idKM, 1);
#pragma unroll
          for (int jj = 0; jj < 4; ++jj)
            mma_bf16_ts(tmem + L::T_DKS, tmem + L::T_DS + 8 * jj,
                        sdesc_sw128(sQ + jj * 2048, 0, 1024), idKM, h > 0 || jj > 0);
          mma_commit(KB((h & 1) ? K_ST1 : K_ST0));
        }
        if (!ok) break;
        if (!mbar_wait(KB(((NH - 1) & 1) ? K_ST1 : K_ST0), ((NH - 1) >> 1) & 1, ab)) break;
        tc_fence_after();
        // G Lambda^T over the score columns (all read out by now)
#pragma unroll
        for (int jj = 0; jj < 4; ++jj)
          mma_bf16_ss(tmem + L::T_P, sdesc_sw128(sV + jj * 32, 16, 1024),
                      sdesc_sw128(sL + jj * 32, 16, 1024), idKK, jj > 0);
        mma_commit(KB(K_GL));
        if constexpr (LOSS == 0) {
          if (!mbar_wait(KB(K_DGRDY), 0, ab)) break;
          tc_fence_after();
#pragma unroll
          for (int jj = 0; jj < 4; ++jj)
            mma_bf16_ss(tmem + L::T_DS, sdesc_sw128(sKH + jj * 32, 16, 1024),
                        sdesc_sw128(sW + jj * 32, 16, 1024), idKK, jj > 0);
          mma_commit(KB(K_DGW));
        }
      } while (0);
    }
  } else {
    // ------------------------------------------------ epilogue: warps 2-5, one key per thread
    const int q = warp & 3;
    const int lrow = q * 32 + lane;
    const uint32_t loff = (uint32_t)(q * 32) << 16;
    const size_t tr = (size_t)tokc + 128 * kb + lrow;
    // this key's rows of L (two 128-byte lines) and k (one), read by the last phase: into L2 now
    const float* Lr = p.Lf + tr * VD;
    const __nv_bfloat16* kr = p.K + tr * VD;
    prefetch_l2(Lr);
    prefetch_l2(Lr + 32);
    if (p.colk || p.dLk) prefetch_l2(kr);
    const float sg = sigm(__ldg(p.beta + tr) + p.lr_bias), eta = 2.f * sg;
    float deta = 0.f;
    // this warp's staging tile for row stores, in the K panel (read by no product once the last
    // query half has been multiplied)
    float* ktile = reinterpret_cast<float*>(smem + L::OFF_K) + q * 1024;
    do {
      // L at the key block's reference token and at the chunk's last token
      {
        const int t = threadIdx.x - 64;
        if (t < VD) {
          f_Lm[t] = __ldg(p.Lf + ((size_t)tokc + 128 * kb + 63) * VD + t);
          f_LC[t] = __ldg(p.Lf + ((size_t)tokc + C - 1) * VD + t);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(KB(K_F));
      }
      if (!mbar_wait(KB(K_GA), 0, ab)) break;
      __syncwarp();
      tc_fence_after();
      // G (bf16, over V) and eta X into the dG accumulator; deta's X . G term
#pragma unroll 1
      for (int h = 0; h < 2; ++h) {
        float gv[32], xv[32];
        ld_row32(sV, lrow, 4 * h, gv);
        if constexpr (SG) {
          // G as saved
        } else if constexpr (LOSS == 0) {
          float z[32];
          tmem_ld32(tmem + loff + L::T_DKS + 32 * h, z);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 32; ++k) gv[k] = z[k] - gv[k];
        } else {
#pragma unroll
          for (int k = 0; k < 32; ++k) gv[k] = -gv[k];
        }
        tmem_ld32(tmem + loff + L::T_DG + 32 * h, xv);
        tmem_wait_ld();
#pragma unroll
        for (int k = 0; k < 32; ++k) {
          deta -= xv[k] * gv[k];
          xv[k] *= eta;
        }
        if (!SG) st_row32(sV, lrow, 4 * h, gv);
        tmem_st32(tmem + loff + L::T_DG + 32 * h, xv);
      }
      tmem_wait_st();
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(KB(K_GRDY));
      // -------- per query half: S^T = eta P^T and eta dS^T (s >= r), packed in place
      bool ok = true;
      for (int h = 0; h < NH; ++h) {
        const bool diag = (h >> 1) == 0;  // qb == kb
        if (!mbar_wait(KB(K_PS), h & 1, ab)) {
          ok = false;
          break;
        }
        __syncwarp();
        tc_fence_after();
        // group g (32 queries) of the half is group G = 2 (h & 1) + g of the 128-query block;
        // it is read (columns [32 g, 32 g + 32)) before its packed form goes to [16 g, 16 g + 16)
#pragma unroll 1
        for (int g = 0; g < 2; ++g) {
          const int G = 2 * (h & 1) + g;
          uint32_t pk[16], pa[16];
          if (diag && G < q) {
            // every query of the group precedes every key of the warp: masked
#pragma unroll
            for (int k = 0; k < 16; ++k) pk[k] = pa[k] = 0u;
          } else {
            float pv[32], dv[32];
            tmem_ld32(tmem + loff + L::T_P + 32 * g, pv);
            tmem_ld32(tmem + loff + L::T_DS + 32 * g, dv);
            tmem_wait_ld();
#pragma unroll
            for (int k = 0; k < 32; ++k) {
              const bool keep = !diag || G > q || 32 * G + k >= lrow;
              const float ds = keep ? -dv[k] : 0.f;
              const float pp = keep ? pv[k] : 0.f;
              deta += ds * pp;
              pv[k] = eta * pp;
              dv[k] = eta * ds;
            }
#pragma unroll
            for (int k = 0; k < 16; ++k) {
              pk[k] = pack_bf16x2(pv[2 * k], pv[2 * k + 1]);
              pa[k] = pack_bf16x2(dv[2 * k], dv[2 * k + 1]);
            }
          }
          tmem_st16u(tmem + loff + L::T_P + 16 * g, pk);
          tmem_st16u(tmem + loff + L::T_DS + 16 * g, pa);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(KB(K_PK));
      }
      if (!ok) break;
      // -------- dG, dV; dG (bf16) for dG W0^T
      if (!mbar_wait(KB(((NH - 1) & 1) ? K_ST1 : K_ST0), ((NH - 1) >> 1) & 1, ab)) break;
      __syncwarp();
      tc_fence_after();
#pragma unroll 1
      for (int h = 0; h < 2; ++h) {
        float a[32];
        tmem_ld32(tmem + loff + L::T_DG + 32 * h, a);  // = -dG = dV
        tmem_wait_ld();
        store_rows32_bf16(ktile, a, p.dV + (tr - lane) * VD + 32 * h, VD, lane);
        if constexpr (LOSS == 0) {
#pragma unroll
          for (int k = 0; k < 32; ++k) a[k] = -a[k];
          st_row32(sKH, lrow, 4 * h, a);
        }
      }
      if constexpr (LOSS == 0) {
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(KB(K_DGRDY));
      }
      // -------- dK
      // the first half's L and k go out before the last products are waited for, the second
      // half's into L1, so no tensor-memory read below waits on global memory
      float4 Lq[8];
      uint4 kq[4];
      const bool want_k = p.colk || p.dLk;
#pragma unroll
      for (int k = 0; k < 8; ++k) Lq[k] = __ldg(reinterpret_cast<const float4*>(Lr) + k);
      if (want_k) {
#pragma unroll
        for (int k = 0; k < 4; ++k) kq[k] = __ldg(reinterpret_cast<const uint4*>(kr) + k);
      }
      prefetch_l1(Lr + 32);
      if (!mbar_wait(KB(K_F), 0, ab) || !mbar_wait(KB(K_GL), 0, ab) ||
          (LOSS == 0 && !mbar_wait(KB(K_DGW), 0, ab)))
        break;
      __syncwarp();
      tc_fence_after();
      bool range = false;
#pragma unroll 1
      for (int h = 0; h < 2; ++h) {
        float dk[32], t32[32], Lv[32];
        if (h == 1) {
#pragma unroll
          for (int k = 0; k < 8; ++k) Lq[k] = __ldg(reinterpret_cast<const float4*>(Lr + 32) + k);
          if (want_k) {
#pragma unroll
            for (int k = 0; k < 4; ++k) kq[k] = __ldg(reinterpret_cast<const uint4*>(kr + 32) + k);
          }
        }
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          Lv[4 * k] = Lq[k].x; Lv[4 * k + 1] = Lq[k].y; Lv[4 * k + 2] = Lq[k].z; Lv[4 * k + 3] = Lq[k].w;
        }
        tmem_ld32(tmem + loff + L::T_P + 32 * h, t32);  // G Lambda^T
        tmem_wait_ld();
        const float* LC = f_LC + 32 * h;
#pragma unroll
        for (int k = 0; k < 32; ++k) dk[k] = -eta * __expf(LC[k] - Lv[k]) * t32[k];
        if (p.colk) {
#pragma unroll
          for (int k = 0; k < 4; ++k) unpack_bf16x8(kq[k], t32 + 8 * k);
#pragma unroll
          for (int k = 0; k < 32; ++k) t32[k] *= dk[k];
          colsum32(t32, lane);
          p.colk[(((size_t)bc * NB + kb) * 4 + q) * VD + 32 * h + lane] = t32[0];
        }
        tmem_ld32(tmem + loff + L::T_DKS + 32 * h, t32);
        tmem_wait_ld();
        const float* Lm = f_Lm + 32 * h;
#pragma unroll
        for (int k = 0; k < 32; ++k) dk[k] += clamped_exp(Lm[k] - Lv[k], range) * t32[k];
        if (p.dLk) {
#pragma unroll
          for (int k = 0; k < 4; ++k) unpack_bf16x8(kq[k], t32 + 8 * k);
#pragma unroll
          for (int k = 0; k < 32; ++k) t32[k] = -t32[k] * dk[k];
          store_rows32_f32(ktile, t32, p.dLk + (tr - lane) * VD + 32 * h, VD, lane);
        }
        if constexpr (LOSS == 0) {
          tmem_ld32(tmem + loff + L::T_DS + 32 * h, t32);  // dG W0^T
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 32; ++k) dk[k] += t32[k];
        }
        store_rows32_bf16(ktile, dk, p.dK + (tr - lane) * VD + 32 * h, VD, lane);
      }
      p.dbeta[tr] = deta * 2.f * sg * (1.f - sg);
      if (range) atomicOr(err, ERR_RANGE);
    } while (0);
  }
#undef KB
  tc_fence_before();
  __syncthreads();
  if (bars->abort_flag) __nanosleep(100000);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

// ----------------------------------------------------------------------- query side: dQ
// One CTA per (batch, head, chunk, 128-query block qb), two per SM. Shared memory (16 KB
// panels): 0, 1: K_kb, then ktilde (qb, kb); 2, 3: V_kb, then G_kb (bf16, in place); 4: dO_qb;
// then W0 and diag(exp(L_m)) W0 (64 x 64 bf16). TMEM (256 columns): [0, 128) G_kb, then the dQ
// accumulator [0, 64) and the packed eta dS block [64, 128); [128, 256) dO G^T.
struct QgL {
  static constexpr uint32_t OFF_W = 5 * PANEL, OFF_WS = OFF_W + VD * 128;
  static constexpr uint32_t OFF_F = OFF_WS + VD * 128;  // -eta[256], L_m[64], exp(L_m)[64]
  static constexpr uint32_t OFF_BAR = OFF_F + (256 + 128) * 4;
  static constexpr uint32_t T_G = 0, T_DQ = 0, T_A = 64, T_DS = 128;
};
enum { Q_LDA, Q_KT, Q_GF, Q_GRDY, Q_DS0, Q_DS1, Q_PK0, Q_PK1, Q_DQS0, Q_DQS1, Q_DQ, Q_F,
       Q_NBARS };
struct __align__(8) QgBars {
  uint64_t b[Q_NBARS];
  uint32_t tmem_base;
  int abort_flag;
};
constexpr uint32_t qg_bytes() { return QgL::OFF_BAR + sizeof(QgBars); }

// SG: the tmV operand is the forward's saved G (bf16), so G is neither recomputed nor negated.
template <int NB, int LOSS, bool SG>
__global__ void __launch_bounds__(kVoThreads, 2)
    bwd_vquery_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                      const __grid_constant__ CUtensorMap tmKt, const __grid_constant__ CUtensorMap tmdO,
                      const __grid_constant__ CUtensorMap tmW, const VgParams p, unsigned* err) {
  constexpr int C = 128 * NB, NV = NB * (NB + 1) / 2;
  using L = QgL;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  const uint32_t sb = smem_u32(smem);
  const uint32_t sDO = sb + 4 * PANEL, sW = sb + L::OFF_W, sWS = sb + L::OFF_WS;
  auto sKb = [&](int kb) { return sb + kb * PANEL; };
  auto sVb = [&](int kb) { return sb + (2 + kb) * PANEL; };
  float* f_neta = reinterpret_cast<float*>(smem + L::OFF_F);
  float* f_Lm = f_neta + 256;
  float* f_eLm = f_Lm + VD;
  QgBars* bars = reinterpret_cast<QgBars*>(smem + L::OFF_BAR);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int per_c = p.BH * NB;
  const int c = p.NC - 1 - (int)blockIdx.x / per_c;
  const int rem = (int)blockIdx.x % per_c;
  const int bh = rem / NB, qb = NB - 1 - rem % NB;
  const int tokc = bh * p.T + c * C;
  const int bc = bh * p.NC + c;
  Abort ab{&bars->abort_flag, err};
#define QB(i) smem_u32(&bars->b[i])
  if (threadIdx.x == 0) {
    for (int i = 0; i < Q_NBARS; ++i)
      mbar_init(QB(i), (i == Q_GRDY || i == Q_PK0 || i == Q_PK1 || i == Q_F) ? 4 : 1);
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

  if (warp == 0) {
    if (lane == 0) {
      const int nk = qb + 1;
      constexpr bool kmma = LOSS == 0 && !SG;  // G = K W0 - V by MMA
      mbar_arrive_expect_tx(QB(Q_LDA), (kmma ? 2 : 1) * nk * PANEL + PANEL + VD * 128);
      for (int kb = 0; kb < nk; ++kb) {
        if (kmma) tma_load_2d(sKb(kb), &tmK, QB(Q_LDA), 0, tokc + 128 * kb);
        tma_load_2d(sVb(kb), &tmV, QB(Q_LDA), 0, tokc + 128 * kb);
      }
      tma_load_2d(sDO, &tmdO, QB(Q_LDA), 0, tokc + 128 * qb);
      tma_load_2d(sW, &tmW, QB(Q_LDA), 0, bc * VD);
      // ktilde over the K slots once K W0 is done
      if (!kmma || mbar_wait(QB(Q_GF), 0, ab)) {
        mbar_arrive_expect_tx(QB(Q_KT), nk * PANEL);
        for (int kb = 0; kb < nk; ++kb)
          tma_load_2d(sKb(kb), &tmKt, QB(Q_KT), 0, (bc * NV + qb * (qb + 1) / 2 + kb) * 128);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idKM = idesc_bf16(128, VD, 0, 1);   // K-major A, MN-major B, N = 64
      const uint32_t idPP = idesc_bf16(128, 128, 0, 0);  // both K-major, N = 128
      const uint32_t idKK = idesc_bf16(128, VD, 0, 0);   // both K-major, N = 64
      do {
        if (!mbar_wait(QB(Q_LDA), 0, ab)) break;
        tc_fence_after();
        if constexpr (LOSS == 0 && !SG) {
          for (int kb = 0; kb <= qb; ++kb) {
#pragma unroll
            for (int jj = 0; jj < 4; ++jj)
              mma_bf16_ss(tmem + L::T_G + VD * kb, sdesc_sw128(sKb(kb) + jj * 32, 16, 1024),
                          sdesc_sw128(sW + jj * 2048, 0, 1024), idKM, jj > 0);
          }
          mma_commit(QB(Q_GF));
        }
        if (!mbar_wait(QB(Q_GRDY), 0, ab)) break;
        tc_fence_after();
        // dQ accumulator = dO (diag(exp(L_m)) W0)^T
#pragma unroll
        for (int jj = 0; jj < 4; ++jj)
          mma_bf16_ss(tmem + L::T_DQ, sdesc_sw128(sDO + jj * 32, 16, 1024),
                      sdesc_sw128(sWS + jj * 32, 16, 1024), idKK, jj > 0);
        bool ok = true;
        for (int kb = 0; kb <= qb && ok; ++kb) {
          if (kb > 0 && !(ok = mbar_wait(QB(Q_PK0), 0, ab))) break;  // dO G_0^T read out
          tc_fence_after();
#pragma unroll
          for (int jj = 0; jj < 4; ++jj)
            mma_bf16_ss(tmem + L::T_DS, sdesc_sw128(sDO + jj * 32, 16, 1024),
                        sdesc_sw128(sVb(kb) + jj * 32, 16, 1024), idPP, jj > 0);
          mma_commit(QB(kb == 0 ? Q_DS0 : Q_DS1));
          if (!(ok = mbar_wait(QB(kb == 0 ? Q_PK0 : Q_PK1), 0, ab))) break;
          if (kb == 0 && !(ok = mbar_wait(QB(Q_KT), 0, ab))) break;
          tc_fence_after();
#pragma unroll
          for (int jj = 0; jj < 8; ++jj)
            mma_bf16_ts(tmem + L::T_DQ, tmem + L::T_A + 8 * jj, sdesc_sw128(sKb(kb) + jj * 2048, 0, 1024),
                        idKM, 1);
          mma_commit(QB(kb == 0 ? Q_DQS0 : Q_DQS1));
        }
        if (!ok) break;
        mma_commit(QB(Q_DQ));
      } while (0);
    }
  } else {
    // ------------------------------------------------ epilogue: warps 2-5, one query per thread
    const int q = warp & 3;
    const int lrow = q * 32 + lane;
    const uint32_t loff = (uint32_t)(q * 32) << 16;
    const int s = 128 * qb + lrow;
    const size_t ts = (size_t)tokc + s;
    // this query's rows of L (two 128-byte lines) and q (one), read by the last phase: into L2 now
    const float* Ls = p.Lf + ts * VD;
    prefetch_l2(Ls);
    prefetch_l2(Ls + 32);
    if (p.dLq) prefetch_l2(p.Q + ts * VD);
    do {
      for (int t = threadIdx.x - 64; t < 128 * (qb + 1); t += 128)
        f_neta[t] = -eta_of(p.beta, (size_t)tokc + t, p.lr_bias);
      if (threadIdx.x - 64 < VD) {
        const int i = threadIdx.x - 64;
        f_Lm[i] = __ldg(p.Lf + ((size_t)tokc + 128 * qb + 63) * VD + i);
        f_eLm[i] = __ldg(p.Em + ((size_t)bc * NB + qb) * VD + i);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(QB(Q_F));
      if (!mbar_wait(QB(Q_F), 0, ab) || !mbar_wait(QB(Q_LDA), 0, ab) ||
          (LOSS == 0 && !SG && !mbar_wait(QB(Q_GF), 0, ab)))
        break;
      __syncwarp();
      tc_fence_after();
      // G_kb (bf16, over V_kb) for every key block up to this one (as saved: nothing to do)
      for (int kb = 0; kb <= qb && !SG; ++kb) {
#pragma unroll 1
        for (int h = 0; h < 2; ++h) {
          float gv[32];
          ld_row32(sVb(kb), lrow, 4 * h, gv);
          if constexpr (LOSS == 0) {
            float z[32];
            tmem_ld32(tmem + loff + L::T_G + VD * kb + 32 * h, z);
            tmem_wait_ld();
#pragma unroll
            for (int k = 0; k < 32; ++k) gv[k] = z[k] - gv[k];
          } else {
#pragma unroll
            for (int k = 0; k < 32; ++k) gv[k] = -gv[k];
          }
          st_row32(sVb(kb), lrow, 4 * h, gv);
        }
      }
      // diag(exp(L_m)) W0 (rows = key features)
      if (lrow < VD) {
#pragma unroll 1
        for (int h = 0; h < 2; ++h) {
          float w[32];
          ld_row32(sW, lrow, 4 * h, w);
          const float e = f_eLm[lrow];
#pragma unroll
          for (int k = 0; k < 32; ++k) w[k] *= e;
          st_row32(sWS, lrow, 4 * h, w);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(QB(Q_GRDY));
      // -------- eta dS blocks (dS' = dO G^T, the sign is in f_neta), packed to bf16
      bool ok = true;
      for (int kb = 0; kb <= qb; ++kb) {
        if (!mbar_wait(QB(kb == 0 ? Q_DS0 : Q_DS1), 0, ab) ||
            (kb > 0 && !mbar_wait(QB(Q_DQS0), 0, ab))) {
          ok = false;
          break;
        }
        __syncwarp();
        tc_fence_after();
        const EWeights w{f_neta, s, 128 * kb};
        pack_block_to(tmem + loff + L::T_DS, tmem + loff + L::T_A, q, kb == qb, w);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(QB(kb == 0 ? Q_PK0 : Q_PK1));
      }
      if (!ok) break;
      // -------- dQ = exp(L_s - L_m) * accumulator; q * dQ for the decay gradient
      // the first half's L and q go out before the accumulator is waited for, the second half's
      // into L1
      float4 Lq[8];
      uint4 qq[4];
      const uint4* q4 = reinterpret_cast<const uint4*>(p.Q + ts * VD);
#pragma unroll
      for (int k = 0; k < 8; ++k) Lq[k] = __ldg(reinterpret_cast<const float4*>(Ls) + k);
      if (p.dLq) {
#pragma unroll
        for (int k = 0; k < 4; ++k) qq[k] = __ldg(q4 + k);
      }
      prefetch_l1(Ls + 32);
      if (!mbar_wait(QB(Q_DQ), 0, ab)) break;
      __syncwarp();
      tc_fence_after();
      bool range = false;
#pragma unroll 1
      for (int h = 0; h < 2; ++h) {
        float a[32];
        if (h == 1) {
#pragma unroll
          for (int k = 0; k < 8; ++k) Lq[k] = __ldg(reinterpret_cast<const float4*>(Ls + 32) + k);
          if (p.dLq) {
#pragma unroll
            for (int k = 0; k < 4; ++k) qq[k] = __ldg(q4 + 4 + k);
          }
        }
        tmem_ld32(tmem + loff + L::T_DQ + 32 * h, a);
        tmem_wait_ld();
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const float4 v = Lq[k];
          a[4 * k] *= clamped_exp(v.x - f_Lm[32 * h + 4 * k], range);
          a[4 * k + 1] *= clamped_exp(v.y - f_Lm[32 * h + 4 * k + 1], range);
          a[4 * k + 2] *= clamped_exp(v.z - f_Lm[32 * h + 4 * k + 2], range);
          a[4 * k + 3] *= clamped_exp(v.w - f_Lm[32 * h + 4 * k + 3], range);
        }
        // the first K panel, read by no product any more, stages the row stores
        float* qtile = reinterpret_cast<float*>(smem) + q * 1024;
        store_rows32_bf16(qtile, a, p.dQ + (ts - lane) * VD + 32 * h, VD, lane);
        if (p.dLq) {
          float qv[32];
#pragma unroll
          for (int k = 0; k < 4; ++k) unpack_bf16x8(qq[k], qv + 8 * k);
#pragma unroll
          for (int k = 0; k < 32; ++k) a[k] *= qv[k];
          store_rows32_f32(qtile, a, p.dLq + (ts - lane) * VD + 32 * h, VD, lane);
        }
      }
      if (range) atomicOr(err, ERR_RANGE);
    } while (0);
  }
#undef QB
  tc_fence_before();
  __syncthreads();
  if (bars->abort_flag) __nanosleep(100000);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

// ------------------------------------------------------------------- decay gradient
// d log gamma_t = sum_{t' >= t} dL_t' (within the chunk), dL_C added at the chunk's last token;
// dgamma = d log gamma / gamma. Thread layout as in the prep kernel.
struct DgParams {
  int NB;
  const float* gamma;
  const float* dLq;
  const float* dLk;
  const float* colk;   // [BH, NC, NB, 4, 64]
  const float* wl;     // [BH, NC, 2, 64]
  const float* GC;     // [BH, NC, 64]
  float* dgamma;
};

template <int NB>
__global__ void __launch_bounds__(kPrepThreads) vec_dgamma_kernel(const DgParams p) {
  constexpr int C = 128 * NB, SEG = C / kPrepSeg;
  __shared__ float4 tot[kPrepSeg][8];
  const int f = threadIdx.x & 7, seg = threadIdx.x >> 3;
  const int fq = (blockIdx.x & 1) * 8 + f;
  const size_t bc = blockIdx.x >> 1;
  const size_t r0 = bc * C + seg * SEG;
  const float4* dq = reinterpret_cast<const float4*>(p.dLq + r0 * VD) + fq;
  const float4* dk = reinterpret_cast<const float4*>(p.dLk + r0 * VD) + fq;
  // every load of the thread (its slice of dLq, dLk and gamma) in flight before any arithmetic
  const float4* g = reinterpret_cast<const float4*>(p.gamma + r0 * VD) + fq;
  float4 d[SEG], gv[SEG];
#pragma unroll
  for (int t = 0; t < SEG; ++t) d[t] = add4(__ldg(dq + t * (VD / 4)), __ldg(dk + t * (VD / 4)));
#pragma unroll
  for (int t = 0; t < SEG; ++t) gv[t] = __ldg(g + t * (VD / 4));
  float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int t = 0; t < SEG; ++t) s = add4(s, d[t]);
  tot[seg][f] = s;
  // the chunk-end term: k * dKhat summed over the chunk's keys, and exp(L_C) rowsum(W0 * Lambda)
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  {
    const float4 w0 = __ldg(reinterpret_cast<const float4*>(p.wl + bc * 2 * VD) + fq);
    const float4 w1 = __ldg(reinterpret_cast<const float4*>(p.wl + (bc * 2 + 1) * VD) + fq);
    const float4 gc = __ldg(reinterpret_cast<const float4*>(p.GC + bc * VD) + fq);
    acc = make_float4(gc.x * (w0.x + w1.x), gc.y * (w0.y + w1.y), gc.z * (w0.z + w1.z),
                      gc.w * (w0.w + w1.w));
#pragma unroll
    for (int j = 0; j < NB * 4; ++j)
      acc = add4(acc, __ldg(reinterpret_cast<const float4*>(p.colk + (bc * NB * 4 + j) * VD) + fq));
  }
  __syncthreads();
#pragma unroll
  for (int k = kPrepSeg - 1; k >= 0; --k)
    if (k > seg) acc = add4(acc, tot[k][f]);
  float4* out = reinterpret_cast<float4*>(p.dgamma + r0 * VD) + fq;
#pragma unroll
  for (int t = SEG - 1; t >= 0; --t) {
    acc = add4(acc, d[t]);
    out[t * (VD / 4)] = make_float4(__fdividef(acc.x, gv[t].x), __fdividef(acc.y, gv[t].y),
                                    __fdividef(acc.z, gv[t].z), __fdividef(acc.w, gv[t].w));
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
  p.Qt2 = static_cast<__nv_bfloat16*>(o.Qt2);
  p.err = a.err;
  const int nunits = a.B * a.H * p.NC * 2;
  int dev = 0, sms = 0;
  cudaError_t e;
  if ((e = cudaGetDevice(&dev)) || (e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)))
    return e;
  const size_t smem = kPrepStages * prep_stage_bytes<NB>();
  if ((e = cudaFuncSetAttribute(vec_prep_kernel<NB>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)smem)))
    return e;
  vec_prep_kernel<NB><<<std::min(nunits, sms), kPrepPThreads, smem, s>>>(p, nunits);
  count_launches(1);
  return cudaGetLastError();
}

// The forward's saved buffer on this path: G [B H T, 64], then the decayed operands with L,
// then R [B H T, 64] (bf16).
struct SavedVec {
  VecPrep pr;
  __nv_bfloat16* R;
};
size_t g_plane(const LayerArgs& a) { return align_up((size_t)a.B * a.H * a.T * VD * 2); }
SavedVec saved_vec(const LayerArgs& a) {
  SavedVec v{};
  if (!a.G_saved) return v;
  uint8_t* base = static_cast<uint8_t*>(a.G_saved) + g_plane(a);
  v.pr = vec_prep_carve(a, base, true);
  v.R = reinterpret_cast<__nv_bfloat16*>(base + vec_prep_bytes(a, true));
  return v;
}

template <int NB, int LOSS>
cudaError_t launch_vec(const LayerArgs& a, cudaStream_t s) {
  constexpr int C = 128 * NB, NV = NB * (NB + 1) / 2;
  const uint64_t rows = (uint64_t)a.B * a.H * a.T;
  const int BH = a.B * a.H, NC = a.T / C;
  // workspace: the decayed operands, then (without W_chunks) the chunk-start states; with
  // G_saved the decayed operands (L included) and R go to the saved buffer after G instead,
  // for the backward
  const SavedVec sv = saved_vec(a);
  const VecPrep pr = a.G_saved ? sv.pr : vec_prep_carve(a, a.ws, false);
  __nv_bfloat16* Wc = static_cast<__nv_bfloat16*>(
      a.W_chunks ? a.W_chunks
                 : static_cast<void*>(static_cast<uint8_t*>(a.ws) + vec_prep_bytes(a, false)));
  CUtensorMap tK, tKh, tV, tVc, tQt, tKt, tW, tG, tR;
  if (!make_tmap_bf16(&tK, a.K, VD, rows, VD, 64, 128) ||
      !make_tmap_bf16(&tKh, pr.Kh, VD, rows, VD, 64, 128) ||
      !make_tmap_bf16(&tVc, a.V, VD, rows, VD, 64, C) ||
      !make_tmap_bf16(&tV, a.V, VD, rows, VD, 64, 128) ||
      !make_tmap_bf16(&tQt, pr.Qt, VD, rows, VD, 64, 128) ||
      !make_tmap_bf16(&tKt, pr.Kt, VD, (uint64_t)BH * NC * NV * 128, VD, 64, 128) ||
      !make_tmap_bf16(&tW, Wc, VD, (uint64_t)BH * NC * VD, VD, 64, VD) ||
      (a.G_saved && !make_tmap_bf16(&tG, a.G_saved, VD, rows, VD, 64, C)) ||
      (a.G_saved && !make_tmap_bf16(&tR, sv.R, VD, rows, VD, 64, 128)))
    return cudaErrorInvalidValue;
  if (!a.G_saved) tG = tR = tK;  // never used
  VecParams p{};
  p.BH = BH;
  p.T = a.T;
  p.NC = NC;
  p.lr_bias = a.lr_bias;
  p.beta = a.beta;
  p.W0 = a.W0;
  p.w0_mod = a.w0_mod;
  p.GC = pr.GC;
  p.Em = pr.Em;
  p.W_final = a.W_final;
  p.Wc = Wc;
  p.O = static_cast<__nv_bfloat16*>(a.O);
  p.save_g = a.G_saved != nullptr;
  p.save_r = a.G_saved != nullptr;
  const size_t sm_s = vs_bytes<NB>() + 1024, sm_o = vo_bytes() + 1024;
  auto ks = fwd_vstate_kernel<NB, LOSS>;
  auto ko = fwd_vout_kernel<NB, LOSS, 0>;
  cudaError_t e;
  if ((e = cudaFuncSetAttribute(ks, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm_s)) ||
      (e = cudaFuncSetAttribute(ko, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm_o)))
    return e;
  if ((e = launch_prep<NB>(a, pr, s))) return e;
  ks<<<BH, kVsThreads, sm_s, s>>>(tK, tKh, tVc, tG, p, a.err);
  ko<<<BH * NC * NB, kVoThreads, sm_o, s>>>(tQt, tKt, tK, tV, tW, tR, p, a.err);
  count_launches(2);
  return cudaGetLastError();
}


template <int NB, int LOSS>
cudaError_t launch_vec_bwd(const LayerArgs& a, cudaStream_t s) {
  constexpr int C = 128 * NB, NV = NB * (NB + 1) / 2;
  const uint64_t rows = (uint64_t)a.B * a.H * a.T;
  const int BH = a.B * a.H, NC = a.T / C;
  // the decayed operands and R: from the forward's saved buffer when given, else formed here
  const bool saved = a.G_saved != nullptr;
  const SavedVec sv = saved_vec(a);
  const VecPrep pr = saved ? sv.pr : vec_prep_carve(a, a.ws, true);
  uint8_t* b = static_cast<uint8_t*>(a.ws) + (saved ? 0 : vec_prep_bytes(a, true));
  auto take = [&](size_t n) {
    uint8_t* r = b;
    b += align_up(n);
    return r;
  };
  __nv_bfloat16* R =
      saved ? sv.R : reinterpret_cast<__nv_bfloat16*>(take(rows * VD * 2));
  __nv_bfloat16* Lam = reinterpret_cast<__nv_bfloat16*>(take((size_t)BH * NC * VD * VD * 2));
  float* wl = reinterpret_cast<float*>(take((size_t)BH * NC * 2 * VD * 4));
  float* colk = reinterpret_cast<float*>(take((size_t)BH * NC * NB * 4 * VD * 4));
  float* dLq = reinterpret_cast<float*>(take(rows * VD * 4));
  float* dLk = reinterpret_cast<float*>(take(rows * VD * 4));
  const bool dg = a.dgamma != nullptr;
  // (with the saved buffer, the gradient kernels take its G through tV instead of V)
  CUtensorMap tK, tKh, tV, tR, tdO, tQt, tKt, tW, tLam, tQh, tQ2h, tdOh;
  if (!make_tmap_bf16(&tK, a.K, VD, rows, VD, 64, 128) ||
      !make_tmap_bf16(&tKh, pr.Kh, VD, rows, VD, 64, 128) ||
      !make_tmap_bf16(&tV, saved ? a.G_saved : a.V, VD, rows, VD, 64, 128) ||
      !make_tmap_bf16(&tR, R, VD, rows, VD, 64, 128) ||
      !make_tmap_bf16(&tdO, a.dO, VD, rows, VD, 64, 128) ||
      !make_tmap_bf16(&tQt, pr.Qt, VD, rows, VD, 64, 128) ||
      !make_tmap_bf16(&tKt, pr.Kt, VD, (uint64_t)BH * NC * NV * 128, VD, 64, 128) ||
      !make_tmap_bf16(&tW, a.W_chunks, VD, (uint64_t)BH * NC * VD, VD, 64, VD) ||
      !make_tmap_bf16(&tLam, Lam, VD, (uint64_t)BH * NC * VD, VD, 64, VD) ||
      !make_tmap_bf16(&tQh, pr.Qt, VD, rows, VD, 64, 64) ||
      !make_tmap_bf16(&tdOh, a.dO, VD, rows, VD, 64, 64) ||
      (NB == 2 && !make_tmap_bf16(&tQ2h, pr.Qt2, VD, (uint64_t)BH * NC * 128, VD, 64, 64)))
    return cudaErrorInvalidValue;
  if (NB == 1) tQ2h = tQh;  // never used
  VecParams vp{};
  vp.BH = BH;
  vp.T = a.T;
  vp.NC = NC;
  vp.lr_bias = a.lr_bias;
  vp.beta = a.beta;
  vp.GC = pr.GC;
  vp.Em = pr.Em;
  VbParams bp{};
  bp.T = a.T;
  bp.NC = NC;
  bp.lr_bias = a.lr_bias;
  bp.beta = a.beta;
  bp.GC = pr.GC;
  bp.dW_final = a.dW_final;
  bp.Wc = static_cast<const __nv_bfloat16*>(a.W_chunks);
  bp.Lam = Lam;
  bp.dW0 = a.dW0;
  bp.wl = dg ? wl : nullptr;
  VgParams gp{};
  gp.BH = BH;
  gp.T = a.T;
  gp.NC = NC;
  gp.lr_bias = a.lr_bias;
  gp.beta = a.beta;
  gp.Lf = pr.Lf;
  gp.Em = pr.Em;
  gp.Q = static_cast<const __nv_bfloat16*>(a.Q);
  gp.K = static_cast<const __nv_bfloat16*>(a.K);
  gp.dQ = static_cast<__nv_bfloat16*>(a.dQ);
  gp.dK = static_cast<__nv_bfloat16*>(a.dK);
  gp.dV = static_cast<__nv_bfloat16*>(a.dV);
  gp.dbeta = a.dbeta;
  gp.dLk = dg ? dLk : nullptr;
  gp.dLq = dg ? dLq : nullptr;
  gp.colk = dg ? colk : nullptr;
  const size_t sm_r = vo_bytes() + 1024, sm_b = vb_bytes<NB>() + 1024, sm_k = kg_bytes() + 1024,
               sm_q = qg_bytes() + 1024;
  auto kr = fwd_vout_kernel<NB, LOSS, 1>;
  auto kb = bwd_vstate_kernel<NB, LOSS>;
  const bool sg = saved;
  auto kk = sg ? bwd_vkey_kernel<NB, LOSS, true> : bwd_vkey_kernel<NB, LOSS, false>;
  auto kq = sg ? bwd_vquery_kernel<NB, LOSS, true> : bwd_vquery_kernel<NB, LOSS, false>;
  cudaError_t e;
  if ((e = cudaFuncSetAttribute(kr, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm_r)) ||
      (e = cudaFuncSetAttribute(kb, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm_b)) ||
      (e = cudaFuncSetAttribute(kk, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm_k)) ||
      (e = cudaFuncSetAttribute(kq, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm_q)))
    return e;
  if (!saved) {
    if ((e = launch_prep<NB>(a, pr, s))) return e;
    kr<<<BH * NC * NB, kVoThreads, sm_r, s>>>(tQt, tKt, tK, tK, tK, tR, vp, a.err);
    count_launches(1);
  }
  // The query side needs no adjoint: it runs on the lower-priority stream beside the serial
  // adjoint chain (one CTA per head, leaving SMs free) and the key side that follows it.
  std::lock_guard<std::mutex> lk(fork_mutex());
  ForkSet* f = fork_set();
  if (!f) return cudaErrorInitializationError;
  if ((e = cudaEventRecord(f->e0, s)) || (e = cudaStreamWaitEvent(f->hi, f->e0, 0)) ||
      (e = cudaStreamWaitEvent(f->lo, f->e0, 0)))
    return e;
  kb<<<BH, kVsThreads, sm_b, f->hi>>>(tK, tKh, tR, tdO, bp, a.err);
  kq<<<BH * NC * NB, kVoThreads, sm_q, f->lo>>>(tK, tV, tKt, tdO, tW, gp, a.err);
  kk<<<BH * NC * NB, kVoThreads, sm_k, f->hi>>>(tK, tKh, tV, tKt, tQh, tQ2h, tdOh, tW, tLam, gp,
                                                a.err);
  if ((e = cudaEventRecord(f->elo, f->lo)) || (e = cudaEventRecord(f->ehi, f->hi)) ||
      (e = cudaStreamWaitEvent(s, f->ehi, 0)) || (e = cudaStreamWaitEvent(s, f->elo, 0)))
    return e;
  count_launches(3);
  if (dg) {
    DgParams dp{};
    dp.NB = NB;
    dp.gamma = a.gamma;
    dp.dLq = dLq;
    dp.dLk = dLk;
    dp.colk = colk;
    dp.wl = wl;
    dp.GC = pr.GC;
    dp.dgamma = a.dgamma;
    vec_dgamma_kernel<NB><<<BH * NC * 2, kPrepThreads, 0, s>>>(dp);
    count_launches(1);
  }
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
  if (with_L) n += align_up(rows * VD * 4) + (NB == 2 ? align_up(BH * NC * 128 * VD * 2) : 0);
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
  if (with_L && NB == 2) o.Qt2 = b + align_up(rows * VD * 4);
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

size_t tc_vec_bwd_workspace(const LayerArgs& a, bool g_saved) {
  const size_t rows = (size_t)a.B * a.H * a.T, BH = (size_t)a.B * a.H, NC = a.T / a.C;
  const size_t NB = a.C / 128;
  return (g_saved ? 0 : vec_prep_bytes(a, true) + align_up(rows * VD * 2)) +
         align_up(BH * NC * VD * VD * 2) + align_up(BH * NC * 2 * VD * 4) +
         align_up(BH * NC * NB * 4 * VD * 4) + 2 * align_up(rows * VD * 4);
}

size_t tc_vec_saved_bytes(const LayerArgs& a) {
  return g_plane(a) + vec_prep_bytes(a, true) + align_up((size_t)a.B * a.H * a.T * VD * 2);
}

cudaError_t tc_vec_bwd(const LayerArgs& a, cudaStream_t s) {
  if (a.C == 128) return a.loss == 0 ? launch_vec_bwd<1, 0>(a, s) : launch_vec_bwd<1, 1>(a, s);
  return a.loss == 0 ? launch_vec_bwd<2, 0>(a, s) : launch_vec_bwd<2, 1>(a, s);
}

}  // namespace tttk
