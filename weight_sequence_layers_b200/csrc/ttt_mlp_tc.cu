// TTT-MLP on the tensor cores: the two-layer fast weight vhat = act(k W1) W2 (page "Modular TTT:
// Rethinking Test-Time Training as Composable Modules", TTT-MLP, the second workload of its
// throughput table) in the chunk dual form of section "方法步骤详情", as a program of batched
// tcgen05 GEMMs with fused epilogues (bgemm_tc.cuh). bf16 operands, fp32 accumulation and fp32
// master weights; d_k = d_v = 64, hidden width h in {128, 256}, C in {128, 256}.
//
// Per chunk, with W1, W2 the chunk-start weights, w_sr = eta_r exp(L_s - L_r) (r <= s),
// u_r = eta_r exp(L_C - L_r), Gamma_s = exp(L_s):
//   Z1 = K W1, A1 = act(Z1), G2 = A1 W2 - V (MSE) or -V (inner product),
//   G1 = (G2 W2^T) * act'(Z1),
//   W1 <- Gamma_C W1 - K^T (u G1),   W2 <- Gamma_C W2 - A1^T (u G2)          (serial)
//   Zq = diag(Gamma) Q W1 - S1 G1, S1 = w * (Q K^T);  Aq = act(Zq)
//   O  = diag(Gamma) Aq W2 - S2 G2, S2 = w * (Aq A1^T)                      (chunk-parallel)
// The serial part runs chunk by chunk, each step one launch batched over the B H heads (its
// intermediates, a few MB per step, stay in L2); the readout runs once over every chunk of
// every head. Operands that a later step reads along the token axis as a K-major A, or as the
// K-major B of a product over tokens, are written transposed by the step that produces them.
#include <cuda_bf16.h>
#include <math.h>

#include <mutex>

#include "bgemm_tc.cuh"
#include "kernels.h"
#include "tc_util.cuh"

namespace tttk {
namespace {

constexpr int D = 64;  // d_k = d_v

struct MCtx {
  int T, C, NC, h;
  float lr_bias;
  int loss;
  const float* beta;
  const float* Lb;  // [BH, T] chunk-local L (zeros without a decay)
};
__device__ __forceinline__ float eta_at(const MCtx& x, size_t tok) {
  return 2.f * sigm(__ldg(x.beta + tok) + x.lr_bias);
}
// u_r = eta_r exp(L_C - L_r) of token tok of the chunk starting at tok0
__device__ __forceinline__ float u_at(const MCtx& x, size_t tok0, size_t tok) {
  return eta_at(x, tok) * __expf(__ldg(x.Lb + tok0 + x.C - 1) - __ldg(x.Lb + tok));
}
__device__ __forceinline__ void ld_bf16x32(const __nv_bfloat16* src, float (&v)[32]) {
  const uint4* s = reinterpret_cast<const uint4*>(src);
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const uint4 u = __ldg(s + k);
    v[8 * k] = bf16lo(u.x); v[8 * k + 1] = bf16hi(u.x);
    v[8 * k + 2] = bf16lo(u.y); v[8 * k + 3] = bf16hi(u.y);
    v[8 * k + 4] = bf16lo(u.z); v[8 * k + 5] = bf16hi(u.z);
    v[8 * k + 6] = bf16lo(u.w); v[8 * k + 7] = bf16hi(u.w);
  }
}
__device__ __forceinline__ void st_f32x32(float* dst, const float (&v)[32]) {
  float4* d = reinterpret_cast<float4*>(dst);
#pragma unroll
  for (int k = 0; k < 8; ++k) d[k] = make_float4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
}
__device__ __forceinline__ void ld_f32x32(const float* src, float (&v)[32]) {
  const float4* s = reinterpret_cast<const float4*>(src);
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const float4 f = s[k];
    v[4 * k] = f.x; v[4 * k + 1] = f.y; v[4 * k + 2] = f.z; v[4 * k + 3] = f.w;
  }
}
// column j of a transposed [cols][ld] bf16 matrix at row r: dst[(col0 + j) ld + r]
__device__ __forceinline__ void st_bf16_cols(__nv_bfloat16* dst, size_t ld, const float (&v)[32]) {
#pragma unroll
  for (int j = 0; j < 32; ++j) dst[(size_t)j * ld] = __float2bfloat16_rn(v[j]);
}

struct Row {
  int b, r;
};

// ---------------------------------------------------------------- forward, serial steps
// Z1 = K W1 of chunk c: Z1 (fp32, per head), A1 = act(Z1) for the whole sequence and A1^T of
// the chunk.
template <int ACT>
struct EpiZ1 {
  MCtx x;
  int c;
  float* Zs;             // [BH, C, h]
  __nv_bfloat16* A1;     // [BH, T, h]
  __nv_bfloat16* A1T;    // [BH, h, C]
  __device__ Row begin(int b, int r) const { return {b, r}; }
  __device__ void chunk(Row& s, int col0, float (&v)[32]) const {
    st_f32x32(Zs + ((size_t)s.b * x.C + s.r) * x.h + col0, v);
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] = act_f<ACT>(v[j]);
    st_global_bf16x32(A1 + ((size_t)s.b * x.T + (size_t)c * x.C + s.r) * x.h + col0, v);
    st_bf16_cols(A1T + ((size_t)s.b * x.h + col0) * x.C + s.r, x.C, v);
  }
  __device__ void end(Row&) const {}
};

// G2 = A1 W2 - V (MSE) or -V; u G2 for the W2 update
struct EpiG2 {
  MCtx x;
  int c;
  const __nv_bfloat16* V;
  __nv_bfloat16* G2;     // [BH, T, 64]
  __nv_bfloat16* uG2;    // [BH, C, 64]
  struct St {
    int b, r;
    size_t tok;
    float u;
  };
  __device__ St begin(int b, int r) const {
    const size_t tok0 = (size_t)b * x.T + (size_t)c * x.C;
    return {b, r, tok0 + r, u_at(x, tok0, tok0 + r)};
  }
  __device__ void chunk(St& s, int col0, float (&v)[32]) const {
    float vv[32];
    ld_bf16x32(V + s.tok * D + col0, vv);
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] = x.loss == 0 ? v[j] - vv[j] : -vv[j];
    st_global_bf16x32(G2 + s.tok * D + col0, v);
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] *= s.u;
    st_global_bf16x32(uG2 + ((size_t)s.b * x.C + s.r) * D + col0, v);
  }
  __device__ void end(St&) const {}
};

// G1 = (G2 W2^T) * act'(Z1): G1^T of the chunk (kept for the readout) and (u G1)^T
template <int ACT>
struct EpiG1 {
  MCtx x;
  int c;
  const float* Zs;
  __nv_bfloat16* G1T;    // [BH, NC, h, C]
  __nv_bfloat16* uG1T;   // [BH, h, C]
  struct St {
    int b, r;
    float u;
  };
  __device__ St begin(int b, int r) const {
    const size_t tok0 = (size_t)b * x.T + (size_t)c * x.C;
    return {b, r, u_at(x, tok0, tok0 + r)};
  }
  __device__ void chunk(St& s, int col0, float (&v)[32]) const {
    float z[32];
    ld_f32x32(Zs + ((size_t)s.b * x.C + s.r) * x.h + col0, z);
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      float f, d1;
      act_both<ACT>(z[j], f, d1);
      v[j] *= d1;
    }
    st_bf16_cols(G1T + (((size_t)s.b * x.NC + c) * x.h + col0) * x.C + s.r, x.C, v);
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] *= s.u;
    st_bf16_cols(uG1T + ((size_t)s.b * x.h + col0) * x.C + s.r, x.C, v);
  }
  __device__ void end(St&) const {}
};

// W1^T <- Gamma_C W1^T - (u G1)^T K: the fp32 master, the bf16 operand copy of the next chunk,
// the caller's W1_chunks / W1_final (not transposed)
struct EpiW1 {
  MCtx x;
  int c;
  float* W1Tm;           // [BH, h, 64]
  __nv_bfloat16* W1Tc;   // [BH, NC, h, 64]
  float* W1c;            // nullable [BH, NC, 64, h]
  float* W1f;            // nullable [BH, 64, h]
  struct St {
    int b, i;
    float g;
  };
  __device__ St begin(int b, int i) const {
    return {b, i, __expf(__ldg(x.Lb + (size_t)b * x.T + (size_t)c * x.C + x.C - 1))};
  }
  __device__ void chunk(St& s, int col0, float (&v)[32]) const {
    float w[32];
    float* m = W1Tm + ((size_t)s.b * x.h + s.i) * D + col0;
    ld_f32x32(m, w);
#pragma unroll
    for (int j = 0; j < 32; ++j) w[j] = s.g * w[j] - v[j];
    st_f32x32(m, w);
    if (c + 1 < x.NC) {
      st_global_bf16x32(W1Tc + (((size_t)s.b * x.NC + c + 1) * x.h + s.i) * D + col0, w);
      if (W1c) {
        float* dst = W1c + (((size_t)s.b * x.NC + c + 1) * D + col0) * x.h + s.i;
#pragma unroll
        for (int j = 0; j < 32; ++j) dst[(size_t)j * x.h] = w[j];
      }
    } else if (W1f) {
      float* dst = W1f + ((size_t)s.b * D + col0) * x.h + s.i;
#pragma unroll
      for (int j = 0; j < 32; ++j) dst[(size_t)j * x.h] = w[j];
    }
  }
  __device__ void end(St&) const {}
};

// W2 <- Gamma_C W2 - A1^T (u G2): the master, bf16 W2 and W2^T of the next chunk, the caller's
// W2_chunks / W2_final
struct EpiW2 {
  MCtx x;
  int c;
  float* W2m;            // [BH, h, 64]
  __nv_bfloat16* W2c;    // [BH, NC, h, 64]
  __nv_bfloat16* W2Tc;   // [BH, NC, 64, h]
  float* W2c_out;        // nullable [BH, NC, h, 64]
  float* W2f;            // nullable [BH, h, 64]
  struct St {
    int b, i;
    float g;
  };
  __device__ St begin(int b, int i) const {
    return {b, i, __expf(__ldg(x.Lb + (size_t)b * x.T + (size_t)c * x.C + x.C - 1))};
  }
  __device__ void chunk(St& s, int col0, float (&v)[32]) const {
    float w[32];
    float* m = W2m + ((size_t)s.b * x.h + s.i) * D + col0;
    ld_f32x32(m, w);
#pragma unroll
    for (int j = 0; j < 32; ++j) w[j] = s.g * w[j] - v[j];
    st_f32x32(m, w);
    if (c + 1 < x.NC) {
      const size_t bc = (size_t)s.b * x.NC + c + 1;
      st_global_bf16x32(W2c + (bc * x.h + s.i) * D + col0, w);
      st_bf16_cols(W2Tc + (bc * D + col0) * x.h + s.i, x.h, w);
      if (W2c_out) st_f32x32(W2c_out + (bc * x.h + s.i) * D + col0, w);
    } else if (W2f) {
      st_f32x32(W2f + ((size_t)s.b * x.h + s.i) * D + col0, w);
    }
  }
  __device__ void end(St&) const {}
};

// ------------------------------------------------------------ forward, chunk-parallel steps
// (batch index = b h NC + c; its tokens are rows [b C, b C + C) of the [B H T] token axis)
// -S_sr = -eta_r exp(L_s - L_r) P_sr for r <= s, else 0
struct EpiScore {
  MCtx x;
  __nv_bfloat16* S;      // [BH NC, C, C]
  struct St {
    size_t tok0;
    int s;
    float Ls;
  };
  __device__ St begin(int b, int s) const {
    const size_t tok0 = (size_t)b * x.C;
    return {tok0, s, __ldg(x.Lb + tok0 + s)};
  }
  __device__ void chunk(St& st, int col0, float (&v)[32]) const {
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const int r = col0 + j;
      v[j] = r <= st.s ? -eta_at(x, st.tok0 + r) * __expf(st.Ls - __ldg(x.Lb + st.tok0 + r)) * v[j]
                       : 0.f;
    }
    st_global_bf16x32(S + (st.tok0 + st.s) * x.C + col0, v);
  }
  __device__ void end(St&) const {}
};

// Aq = act(Zq) and diag(Gamma) Aq
template <int ACT>
struct EpiAq {
  MCtx x;
  __nv_bfloat16* Aq;     // [BH, T, h]
  __nv_bfloat16* Ahq;    // [BH, T, h]
  struct St {
    size_t tok;
    float g;
  };
  __device__ St begin(int b, int s) const {
    const size_t tok = (size_t)b * x.C + s;
    return {tok, __expf(__ldg(x.Lb + tok))};
  }
  __device__ void chunk(St& st, int col0, float (&v)[32]) const {
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] = act_f<ACT>(v[j]);
    st_global_bf16x32(Aq + st.tok * x.h + col0, v);
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] *= st.g;
    st_global_bf16x32(Ahq + st.tok * x.h + col0, v);
  }
  __device__ void end(St&) const {}
};

struct EpiOut {
  MCtx x;
  __nv_bfloat16* O;
  __device__ size_t begin(int b, int s) const { return (size_t)b * x.C + s; }
  __device__ void chunk(size_t& tok, int col0, float (&v)[32]) const {
    st_global_bf16x32(O + tok * D + col0, v);
  }
  __device__ void end(size_t&) const {}
};

// ------------------------------------------------------------------------- helpers
// Chunk-local L of every token (one block per chunk, a warp scan) and Qhat = Gamma_s q_s.
__global__ void __launch_bounds__(256) mlp_scan_kernel(int C, const float* gamma,
                                                       const __nv_bfloat16* Q, float* Lb,
                                                       __nv_bfloat16* Qh) {
  __shared__ float sL[256];
  const size_t tok0 = (size_t)blockIdx.x * C;
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x, per = C / 32;
    float s = 0.f;
    float loc[8];
    for (int k = 0; k < per; ++k) {
      s += gamma ? __logf(__ldg(gamma + tok0 + lane * per + k)) : 0.f;
      loc[k] = s;
    }
    float incl = s;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const float y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    const float excl = incl - s;
    for (int k = 0; k < per; ++k) sL[lane * per + k] = excl + loc[k];
  }
  __syncthreads();
  for (int t = threadIdx.x; t < C; t += blockDim.x) Lb[tok0 + t] = sL[t];
  for (int e = threadIdx.x; e < C * D / 8; e += blockDim.x) {
    const int t = e / (D / 8), q8 = e % (D / 8);
    const float g = __expf(sL[t]);
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(Q + (tok0 + t) * D) + q8);
    uint4 o;
    o.x = pack_bf16x2(bf16lo(u.x) * g, bf16hi(u.x) * g);
    o.y = pack_bf16x2(bf16lo(u.y) * g, bf16hi(u.y) * g);
    o.z = pack_bf16x2(bf16lo(u.z) * g, bf16hi(u.z) * g);
    o.w = pack_bf16x2(bf16lo(u.w) * g, bf16hi(u.w) * g);
    reinterpret_cast<uint4*>(Qh + (tok0 + t) * D)[q8] = o;
  }
}

// Chunk-0 weights: the masters and operand copies from W1_0 [64, h] and W2_0 [h, 64].
__global__ void mlp_init_kernel(int h, int NC, const float* W1_0, const float* W2_0, float* W1Tm,
                                float* W2m, __nv_bfloat16* W1Tc, __nv_bfloat16* W2c,
                                __nv_bfloat16* W2Tc, float* W1c, float* W2c_out) {
  const size_t b = blockIdx.x, n = (size_t)h * D;
  for (size_t e = threadIdx.x; e < n; e += blockDim.x) {
    const int i = (int)(e / D), k = (int)(e % D);  // row i of the [h, 64] matrices
    const float w1 = W1_0[b * n + (size_t)k * h + i];
    const float w2 = W2_0[b * n + e];
    W1Tm[b * n + e] = w1;
    W2m[b * n + e] = w2;
    W1Tc[b * NC * n + e] = __float2bfloat16_rn(w1);
    W2c[b * NC * n + e] = __float2bfloat16_rn(w2);
    W2Tc[b * NC * n + (size_t)k * h + i] = __float2bfloat16_rn(w2);
    if (W1c) W1c[b * NC * n + (size_t)k * h + i] = w1;
    if (W2c_out) W2c_out[b * NC * n + e] = w2;
  }
}

// ---------------------------------------------------------------------------- host side
bool tm3(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint64_t batch,
         uint64_t row_stride, uint64_t batch_stride, uint32_t box_rows) {
  return make_tmap3_bf16(m, base, inner, rows, batch, row_stride, batch_stride, 64, box_rows);
}

template <int N, int MN0, int MN1, int MN2, typename Epi>
cudaError_t gemm(dim3 grid, const CUtensorMap* m, const bg::Prob& pr, const Epi& e,
                 unsigned* err, cudaStream_t s) {
  auto k = bg::gemm_kernel<N, MN0, MN1, MN2, Epi>;
  static std::once_flag once;
  static cudaError_t attr = cudaSuccess;
  std::call_once(once, [&] {
    attr = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)bg::smem_bytes<N>());
  });
  if (attr != cudaSuccess) return attr;
  k<<<grid, bg::kThreads, bg::smem_bytes<N>(), s>>>(m[0], m[1], m[2], m[3], m[4], m[5], pr, e, err);
  count_launches(1);
  return cudaGetLastError();
}

bg::Prob prob1(int K, int a_k0, int a_row, int b_k0, int b_row) {
  bg::Prob p{};
  p.nterm = 1;
  p.t[0] = bg::Term{K, a_k0, a_row, b_k0, b_row};
  return p;
}

struct FwdBufs {
  float *Lb, *W1Tm, *W2m, *Zs;
  __nv_bfloat16 *Qh, *W1Tc, *W2c, *W2Tc, *A1, *A1T, *G2, *uG2, *G1T, *uG1T, *S1, *Aq, *Ahq, *S2;
};

size_t up(size_t x) { return (x + 1023) & ~size_t(1023); }

// Carves the forward's buffers from the workspace (nullptr base: sizes only); returns the bytes.
size_t carve_fwd(const LayerArgs& a, int h, void* base, FwdBufs* f) {
  const size_t BH = (size_t)a.B * a.H, T = a.T, C = a.C, NC = T / C, rows = BH * T;
  uint8_t* p = static_cast<uint8_t*>(base);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    void* r = p ? p + off : nullptr;
    off += up(bytes);
    return r;
  };
  FwdBufs b{};
  b.Lb = (float*)take(rows * 4);
  b.W1Tm = (float*)take(BH * h * D * 4);
  b.W2m = (float*)take(BH * h * D * 4);
  b.Zs = (float*)take(BH * C * h * 4);
  b.Qh = (__nv_bfloat16*)take(rows * D * 2);
  b.W1Tc = (__nv_bfloat16*)take(BH * NC * h * D * 2);
  b.W2c = (__nv_bfloat16*)take(BH * NC * h * D * 2);
  b.W2Tc = (__nv_bfloat16*)take(BH * NC * h * D * 2);
  b.A1 = (__nv_bfloat16*)take(rows * h * 2);
  b.A1T = (__nv_bfloat16*)take(BH * h * C * 2);
  b.G2 = (__nv_bfloat16*)take(rows * D * 2);
  b.uG2 = (__nv_bfloat16*)take(BH * C * D * 2);
  b.G1T = (__nv_bfloat16*)take(rows * h * 2);
  b.uG1T = (__nv_bfloat16*)take(BH * h * C * 2);
  b.S1 = (__nv_bfloat16*)take(rows * C * 2);
  b.Aq = (__nv_bfloat16*)take(rows * h * 2);
  b.Ahq = (__nv_bfloat16*)take(rows * h * 2);
  b.S2 = (__nv_bfloat16*)take(rows * C * 2);
  if (f) *f = b;
  return off;
}

template <int ACT>
cudaError_t mlp_tc_fwd_impl(const LayerArgs& a, int h, const float* W1_0, const float* W2_0,
                            float* W1f, float* W2f, float* W1c, float* W2c_out, cudaStream_t s) {
  const int BH = a.B * a.H, T = a.T, C = a.C, NC = T / C;
  FwdBufs f;
  carve_fwd(a, h, a.ws, &f);
  const auto* Q = static_cast<const __nv_bfloat16*>(a.Q);
  const auto* K = static_cast<const __nv_bfloat16*>(a.K);
  const auto* V = static_cast<const __nv_bfloat16*>(a.V);
  MCtx x{T, C, NC, h, a.lr_bias, a.loss, a.beta, f.Lb};
  cudaError_t e;
  mlp_scan_kernel<<<BH * NC, 256, 0, s>>>(C, a.gamma, Q, f.Lb, f.Qh);
  mlp_init_kernel<<<BH, 256, 0, s>>>(h, NC, W1_0, W2_0, f.W1Tm, f.W2m, f.W1Tc, f.W2c, f.W2Tc,
                                      W1c, W2c_out);
  count_launches(2);
  if ((e = cudaGetLastError())) return e;
  // maps that do not move with the chunk
  CUtensorMap mK, mKmn, mA1, mG2, mUG1T, mA1T, mUG2;
  bool ok = tm3(&mK, K, D, T, BH, D, (uint64_t)T * D, 128) &&
            tm3(&mKmn, K, D, T, BH, D, (uint64_t)T * D, 64) &&
            tm3(&mA1, f.A1, h, T, BH, h, (uint64_t)T * h, 128) &&
            tm3(&mG2, f.G2, D, T, BH, D, (uint64_t)T * D, 128) &&
            tm3(&mUG1T, f.uG1T, C, h, BH, C, (uint64_t)h * C, 128) &&
            tm3(&mA1T, f.A1T, C, h, BH, C, (uint64_t)h * C, 128) &&
            tm3(&mUG2, f.uG2, D, C, BH, D, (uint64_t)C * D, 64);
  if (!ok) return cudaErrorInvalidValue;
  const dim3 gC(C / 128, BH), gH(h / 128, BH);
  const uint64_t wst = (uint64_t)NC * h * D;  // per-head stride of the per-chunk weight copies
  for (int c = 0; c < NC; ++c) {
    CUtensorMap mW1T, mW2T, mW2;
    ok = tm3(&mW1T, f.W1Tc + (size_t)c * h * D, D, h, BH, D, wst, h) &&
         tm3(&mW2T, f.W2Tc + (size_t)c * h * D, h, D, BH, h, wst, D) &&
         tm3(&mW2, f.W2c + (size_t)c * h * D, D, h, BH, D, wst, h);
    if (!ok) return cudaErrorInvalidValue;
    {  // Z1 = K W1
      const CUtensorMap m[6] = {mK, mW1T, mK, mK, mK, mK};
      const EpiZ1<ACT> ep{x, c, f.Zs, f.A1, f.A1T};
      if (h == 256) e = gemm<256, 0, 0, 0>(gC, m, prob1(D, 0, c * C, 0, 0), ep, a.err, s);
      else e = gemm<128, 0, 0, 0>(gC, m, prob1(D, 0, c * C, 0, 0), ep, a.err, s);
      if (e) return e;
    }
    {  // G2 = A1 W2 - V
      const CUtensorMap m[6] = {mA1, mW2T, mK, mK, mK, mK};
      const EpiG2 ep{x, c, V, f.G2, f.uG2};
      if ((e = gemm<64, 0, 0, 0>(gC, m, prob1(h, 0, c * C, 0, 0), ep, a.err, s))) return e;
    }
    {  // G1 = (G2 W2^T) * act'(Z1)
      const CUtensorMap m[6] = {mG2, mW2, mK, mK, mK, mK};
      const EpiG1<ACT> ep{x, c, f.Zs, f.G1T, f.uG1T};
      if (h == 256) e = gemm<256, 0, 0, 0>(gC, m, prob1(D, 0, c * C, 0, 0), ep, a.err, s);
      else e = gemm<128, 0, 0, 0>(gC, m, prob1(D, 0, c * C, 0, 0), ep, a.err, s);
      if (e) return e;
    }
    {  // W1^T <- Gamma_C W1^T - (u G1)^T K
      const CUtensorMap m[6] = {mUG1T, mKmn, mK, mK, mK, mK};
      const EpiW1 ep{x, c, f.W1Tm, f.W1Tc, W1c, W1f};
      if ((e = gemm<64, 1, 0, 0>(gH, m, prob1(C, 0, 0, 0, c * C), ep, a.err, s))) return e;
    }
    {  // W2 <- Gamma_C W2 - A1^T (u G2)
      const CUtensorMap m[6] = {mA1T, mUG2, mK, mK, mK, mK};
      const EpiW2 ep{x, c, f.W2m, f.W2c, f.W2Tc, W2c_out, W2f};
      if ((e = gemm<64, 1, 0, 0>(gH, m, prob1(C, 0, 0, 0, 0), ep, a.err, s))) return e;
    }
  }
  // ----------------------------------------------------- readout over every chunk at once
  const int NB = BH * NC;
  const dim3 gR(C / 128, NB);
  CUtensorMap mQ, mKc, mQh, mW1Tall, mS1, mG1T, mAq, mA1c, mAhq, mW2Tall, mS2, mG2mn;
  ok = tm3(&mQ, Q, D, C, NB, D, (uint64_t)C * D, 128) &&
       tm3(&mKc, K, D, C, NB, D, (uint64_t)C * D, C) &&
       tm3(&mQh, f.Qh, D, C, NB, D, (uint64_t)C * D, 128) &&
       tm3(&mW1Tall, f.W1Tc, D, h, NB, D, (uint64_t)h * D, h) &&
       tm3(&mS1, f.S1, C, C, NB, C, (uint64_t)C * C, 128) &&
       tm3(&mG1T, f.G1T, C, h, NB, C, (uint64_t)h * C, h) &&
       tm3(&mAq, f.Aq, h, C, NB, h, (uint64_t)C * h, 128) &&
       tm3(&mA1c, f.A1, h, C, NB, h, (uint64_t)C * h, C) &&
       tm3(&mAhq, f.Ahq, h, C, NB, h, (uint64_t)C * h, 128) &&
       tm3(&mW2Tall, f.W2Tc, h, D, NB, h, (uint64_t)h * D, D) &&
       tm3(&mS2, f.S2, C, C, NB, C, (uint64_t)C * C, 128) &&
       tm3(&mG2mn, f.G2, D, C, NB, D, (uint64_t)C * D, 64);
  if (!ok) return cudaErrorInvalidValue;
  {  // -S1 = -w * (Q K^T)
    const CUtensorMap m[6] = {mQ, mKc, mQ, mQ, mQ, mQ};
    const EpiScore ep{x, f.S1};
    if (C == 256) e = gemm<256, 0, 0, 0>(gR, m, prob1(D, 0, 0, 0, 0), ep, a.err, s);
    else e = gemm<128, 0, 0, 0>(gR, m, prob1(D, 0, 0, 0, 0), ep, a.err, s);
    if (e) return e;
  }
  {  // Zq = Qhat W1 + (-S1) G1 -> Aq, Gamma Aq
    const CUtensorMap m[6] = {mQh, mW1Tall, mS1, mG1T, mQ, mQ};
    bg::Prob pr{};
    pr.nterm = 2;
    pr.t[0] = bg::Term{D, 0, 0, 0, 0};
    pr.t[1] = bg::Term{C, 0, 0, 0, 0};
    const EpiAq<ACT> ep{x, f.Aq, f.Ahq};
    if (h == 256) e = gemm<256, 0, 0, 0>(gR, m, pr, ep, a.err, s);
    else e = gemm<128, 0, 0, 0>(gR, m, pr, ep, a.err, s);
    if (e) return e;
  }
  {  // -S2 = -w * (Aq A1^T)
    const CUtensorMap m[6] = {mAq, mA1c, mQ, mQ, mQ, mQ};
    const EpiScore ep{x, f.S2};
    if (C == 256) e = gemm<256, 0, 0, 0>(gR, m, prob1(h, 0, 0, 0, 0), ep, a.err, s);
    else e = gemm<128, 0, 0, 0>(gR, m, prob1(h, 0, 0, 0, 0), ep, a.err, s);
    if (e) return e;
  }
  {  // O = (Gamma Aq) W2 + (-S2) G2
    const CUtensorMap m[6] = {mAhq, mW2Tall, mS2, mG2mn, mQ, mQ};
    bg::Prob pr{};
    pr.nterm = 2;
    pr.t[0] = bg::Term{h, 0, 0, 0, 0};
    pr.t[1] = bg::Term{C, 0, 0, 0, 0};
    const EpiOut ep{x, static_cast<__nv_bfloat16*>(a.O)};
    if ((e = gemm<64, 0, 1, 0>(gR, m, pr, ep, a.err, s))) return e;
  }
  return cudaSuccess;
}

}  // namespace

bool mlp_tc_supported(const LayerArgs& a, int hidden) {
  return a.dtype == 1 && !a.gvec && a.dk == D && a.dv == D && (hidden == 128 || hidden == 256) &&
         (a.C == 128 || a.C == 256) && a.T % a.C == 0;
}

size_t mlp_tc_fwd_workspace(const LayerArgs& a, int hidden) {
  return carve_fwd(a, hidden, nullptr, nullptr);
}

cudaError_t mlp_tc_fwd(const LayerArgs& a, int hidden, const float* W1_0, const float* W2_0,
                       float* W1f, float* W2f, float* W1c, float* W2c, cudaStream_t s) {
  return a.act == 1 ? mlp_tc_fwd_impl<1>(a, hidden, W1_0, W2_0, W1f, W2f, W1c, W2c, s)
                    : mlp_tc_fwd_impl<0>(a, hidden, W1_0, W2_0, W1f, W2f, W1c, W2c, s);
}

}  // namespace tttk
