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
  int loss;
  const float* Eb;  // [BH, T] eta_t = 2 sigmoid(beta_t + b)
  const float* Lb;  // [BH, T] chunk-local L (zeros without a decay)
  // with g(t) the first token of t's 32-token group: Cr_t = eta_t exp(L_g(t) - L_t) and
  // Cf_t = exp(L_t - L_g(t)), so that a score weight eta_r exp(L_s - L_r) over a group of 32
  // keys (or queries) costs one exponential per row and group
  const float* Cr;
  const float* Cf;
};
__device__ __forceinline__ float eta_at(const MCtx& x, size_t tok) { return __ldg(x.Eb + tok); }
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
    if (col0 <= st.s) {  // else every key of the group follows the query: zeros
      float c[32];
      ld_f32x32(x.Cr + st.tok0 + col0, c);
      const float rho = -__expf(st.Ls - __ldg(x.Lb + st.tok0 + col0));
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] = col0 + j <= st.s ? rho * c[j] * v[j] : 0.f;
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] = 0.f;
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
// Chunk-local L of every token (one block per chunk, a warp scan), eta, Qhat = Gamma_s q_s and,
// when given, Gamma_s dO_s.
__global__ void __launch_bounds__(256) mlp_scan_kernel(int C, const float* gamma,
                                                       const float* beta, float lr_bias,
                                                       const __nv_bfloat16* Q, float* Lb,
                                                       float* Eb, float* Cr, float* Cf,
                                                       __nv_bfloat16* Qh,
                                                       const __nv_bfloat16* dO = nullptr,
                                                       __nv_bfloat16* dOh = nullptr) {
  __shared__ float sL[256];
  const size_t tok0 = (size_t)blockIdx.x * C;
  for (int t = threadIdx.x; t < C; t += blockDim.x)
    Eb[tok0 + t] = 2.f * sigm(__ldg(beta + tok0 + t) + lr_bias);
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
  for (int t = threadIdx.x; t < C; t += blockDim.x) {
    Lb[tok0 + t] = sL[t];
    const float e = sL[t] - sL[t & ~31];
    Cr[tok0 + t] = 2.f * sigm(__ldg(beta + tok0 + t) + lr_bias) * __expf(-e);
    Cf[tok0 + t] = __expf(e);
  }
  auto scale = [&](const __nv_bfloat16* src, __nv_bfloat16* dst) {
    for (int e = threadIdx.x; e < C * D / 8; e += blockDim.x) {
      const int t = e / (D / 8), q8 = e % (D / 8);
      const float g = __expf(sL[t]);
      const uint4 u = __ldg(reinterpret_cast<const uint4*>(src + (tok0 + t) * D) + q8);
      uint4 o;
      o.x = pack_bf16x2(bf16lo(u.x) * g, bf16hi(u.x) * g);
      o.y = pack_bf16x2(bf16lo(u.y) * g, bf16hi(u.y) * g);
      o.z = pack_bf16x2(bf16lo(u.z) * g, bf16hi(u.z) * g);
      o.w = pack_bf16x2(bf16lo(u.w) * g, bf16hi(u.w) * g);
      reinterpret_cast<uint4*>(dst + (tok0 + t) * D)[q8] = o;
    }
  };
  scale(Q, Qh);
  if (dO) scale(dO, dOh);
}

// dst[c][r] = src[r][c] for an R x Cc float32 matrix (R, Cc multiples of 32; src NULL: zeros),
// through 32 x 32 shared-memory tiles, one block of 256 threads; float or bf16 destinations.
__device__ __forceinline__ void put(float* p, float v) { *p = v; }
__device__ __forceinline__ void put(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }
template <typename TA, typename TB>
__device__ void transpose_to(const float* src, int R, int Cc, TA* dst, TB* dst2,
                             float (*tile)[33]) {
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  for (int r0 = 0; r0 < R; r0 += 32)
    for (int c0 = 0; c0 < Cc; c0 += 32) {
      for (int k = ty; k < 32; k += 8)
        tile[k][tx] = src ? src[(size_t)(r0 + k) * Cc + c0 + tx] : 0.f;
      __syncthreads();
      for (int k = ty; k < 32; k += 8) {
        const size_t o = (size_t)(c0 + k) * R + r0 + tx;
        put(dst + o, tile[tx][k]);
        if (dst2) put(dst2 + o, tile[tx][k]);
      }
      __syncthreads();
    }
}
// element-wise copies of an n-element float32 array (src NULL: zeros)
template <typename TA, typename TB>
__device__ void copy_to(const float* src, size_t n, TA* dst, TB* dst2) {
  for (size_t e = threadIdx.x; e < n; e += blockDim.x) {
    const float v = src ? src[e] : 0.f;
    if (dst) put(dst + e, v);
    if (dst2) put(dst2 + e, v);
  }
}

// Chunk-0 weights: the masters and operand copies from W1_0 [64, h] and W2_0 [h, 64].
// (initial weights of head b are block b % w0_mod of W1_0 / W2_0)
__global__ void __launch_bounds__(256)
    mlp_init_kernel(int h, int NC, int w0_mod, const float* W1_0, const float* W2_0, float* W1Tm,
                    float* W2m, __nv_bfloat16* W1Tc, __nv_bfloat16* W2c, __nv_bfloat16* W2Tc,
                    float* W1c, float* W2c_out) {
  __shared__ float tile[32][33];
  const size_t b = blockIdx.x, n = (size_t)h * D, b0 = b % w0_mod;
  transpose_to(W1_0 + b0 * n, D, h, W1Tm + b * n, W1Tc + b * NC * n, tile);
  transpose_to(W2_0 + b0 * n, h, D, W2Tc + b * NC * n, (float*)nullptr, tile);
  copy_to(W2_0 + b0 * n, n, W2m + b * n, W2c + b * NC * n);
  copy_to(W1_0 + b0 * n, n, W1c ? W1c + b * NC * n : nullptr, (float*)nullptr);
  copy_to(W2_0 + b0 * n, n, W2c_out ? W2c_out + b * NC * n : nullptr, (float*)nullptr);
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
  float *Lb, *Eb, *Cr, *Cf, *W1Tm, *W2m, *Zs;
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
  b.Eb = (float*)take(rows * 4);
  b.Cr = (float*)take(rows * 4);
  b.Cf = (float*)take(rows * 4);
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
  MCtx x{T, C, NC, h, a.loss, f.Eb, f.Lb, f.Cr, f.Cf};
  cudaError_t e;
  mlp_scan_kernel<<<BH * NC, 256, 0, s>>>(C, a.gamma, a.beta, a.lr_bias, Q, f.Lb, f.Eb, f.Cr, f.Cf,
                                          f.Qh);
  mlp_init_kernel<<<BH, 256, 0, s>>>(h, NC, a.w0_mod, W1_0, W2_0, f.W1Tm, f.W2m, f.W1Tc, f.W2c,
                                      f.W2Tc, W1c, W2c_out);
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

// ============================================================================== backward
// Reverse over chunks for J = <dO, O> + <dW1_T, W1_final> + <dW2_T, W2_final>, with Wh1, Wh2
// the adjoints of a chunk's end weights (D = dS * w with dS the score gradients):
//   dS2 = -dO G2^T, dZq = (Gamma dO W2^T + D2 A1) * act'(Zq), dA1 = D2^T Aq - u (G2 Wh2^T),
//   dS1 = -dZq G1^T, dQ = Gamma (dZq W1^T) + D1 K,     dG1 = -S1^T dZq - u (K Wh1),
//   dB = dG1 * act'(Z1),  dG2 = -S2^T dO - u (A1 Wh2) + dB W2,   dV = -dG2,
//   dZ1 = dG1 * Bm * act''(Z1) + (dA1 + [MSE] dG2 W2^T) * act'(Z1),
//   dK = D1^T Q - u (G1 Wh1^T) + dZ1 W1^T,
//   deta_r = sum_s (dS1 S1 + dS2 S2)_sr / eta_r - exp(L_C - L_r) (Yk_r . G1_r + Ya_r . G2_r),
//   Wh1 <- Gamma_C Wh1 + Qhat^T dZq + K^T dZ1,
//   Wh2 <- Gamma_C Wh2 + (Gamma Aq)^T dO + dB^T G2 + [MSE] A1^T dG2.
// Everything that does not involve Wh1, Wh2 runs once over every chunk; the rest is eight
// launches per chunk, batched over the heads.

// token row of accumulator row r of batch b: b * bs + r0 + r
struct Tok {
  size_t bs, r0;
  __device__ size_t operator()(int b, int r) const { return (size_t)b * bs + r0 + r; }
};

// row-major store of the accumulator, bf16 or float32
template <typename TO>
struct EpiStore {
  Tok tk;
  TO* out;
  int ld;
  __device__ size_t begin(int b, int r) const { return tk(b, r); }
  __device__ void chunk(size_t& t, int col0, float (&v)[32]) const {
    if constexpr (sizeof(TO) == 4) st_f32x32(reinterpret_cast<float*>(out) + t * ld + col0, v);
    else st_global_bf16x32(reinterpret_cast<__nv_bfloat16*>(out) + t * ld + col0, v);
  }
  __device__ void end(size_t&) const {}
};

// recompute, chunk-parallel: Z1 (float32), A1 and A1^T
template <int ACT>
struct EpiZ1b {
  MCtx x;
  float* Z1;             // [BH, T, h]
  __nv_bfloat16* A1;     // [BH, T, h]
  __nv_bfloat16* A1T;    // [NB, h, C]
  __device__ Row begin(int b, int r) const { return {b, r}; }
  __device__ void chunk(Row& s, int col0, float (&v)[32]) const {
    const size_t t = (size_t)s.b * x.C + s.r;
    st_f32x32(Z1 + t * x.h + col0, v);
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] = act_f<ACT>(v[j]);
    st_global_bf16x32(A1 + t * x.h + col0, v);
    st_bf16_cols(A1T + ((size_t)s.b * x.h + col0) * x.C + s.r, x.C, v);
  }
  __device__ void end(Row&) const {}
};
// G2 and -u G2
struct EpiG2b {
  MCtx x;
  const __nv_bfloat16* V;
  __nv_bfloat16 *G2, *uG2n;  // [BH, T, 64]
  struct St {
    size_t t;
    float u;
  };
  __device__ St begin(int b, int r) const {
    const size_t tok0 = (size_t)b * x.C;
    return {tok0 + r, u_at(x, tok0, tok0 + r)};
  }
  __device__ void chunk(St& s, int col0, float (&v)[32]) const {
    float vv[32];
    ld_bf16x32(V + s.t * D + col0, vv);
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] = x.loss == 0 ? v[j] - vv[j] : -vv[j];
    st_global_bf16x32(G2 + s.t * D + col0, v);
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] *= -s.u;
    st_global_bf16x32(uG2n + s.t * D + col0, v);
  }
  __device__ void end(St&) const {}
};
// Bm, G1 = Bm * act'(Z1), G1^T and -u G1
template <int ACT>
struct EpiG1b {
  MCtx x;
  const float* Z1;
  __nv_bfloat16 *Bm, *G1, *G1T, *uG1n;
  struct St {
    int b, r;
    size_t t;
    float u;
  };
  __device__ St begin(int b, int r) const {
    const size_t tok0 = (size_t)b * x.C;
    return {b, r, tok0 + r, u_at(x, tok0, tok0 + r)};
  }
  __device__ void chunk(St& s, int col0, float (&v)[32]) const {
    float z[32];
    ld_f32x32(Z1 + s.t * x.h + col0, z);
    st_global_bf16x32(Bm + s.t * x.h + col0, v);
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      float f, d1;
      act_both<ACT>(z[j], f, d1);
      v[j] *= d1;
    }
    st_global_bf16x32(G1 + s.t * x.h + col0, v);
    st_bf16_cols(G1T + ((size_t)s.b * x.h + col0) * x.C + s.r, x.C, v);
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] *= -s.u;
    st_global_bf16x32(uG1n + s.t * x.h + col0, v);
  }
  __device__ void end(St&) const {}
};
// transposed scores: -S^T_rs = -eta_r exp(L_s - L_r) P_rs for s >= r (rows = keys r)
struct EpiScoreT {
  MCtx x;
  __nv_bfloat16* S;      // [NB, C, C]
  struct St {
    size_t tok0;
    int r;
    float ne, Lr;
  };
  __device__ St begin(int b, int r) const {
    const size_t tok0 = (size_t)b * x.C;
    return {tok0, r, -eta_at(x, tok0 + r), __ldg(x.Lb + tok0 + r)};
  }
  __device__ void chunk(St& st, int col0, float (&v)[32]) const {
    if (col0 + 31 >= st.r) {  // else every query of the group precedes the key: zeros
      float c[32];
      ld_f32x32(x.Cf + st.tok0 + col0, c);
      const float rho = st.ne * __expf(__ldg(x.Lb + st.tok0 + col0) - st.Lr);
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] = col0 + j >= st.r ? rho * c[j] * v[j] : 0.f;
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] = 0.f;
    }
    st_global_bf16x32(S + (st.tok0 + st.r) * x.C + col0, v);
  }
  __device__ void end(St&) const {}
};
// Aq (and Aq^T), (Gamma Aq)^T and act'(Zq)
template <int ACT>
struct EpiAqb {
  MCtx x;
  __nv_bfloat16 *Aq, *AqT, *AhqT, *dAct;
  struct St {
    int b, s;
    size_t t;
    float g;
  };
  __device__ St begin(int b, int s) const {
    const size_t t = (size_t)b * x.C + s;
    return {b, s, t, __expf(__ldg(x.Lb + t))};
  }
  __device__ void chunk(St& st, int col0, float (&v)[32]) const {
    float d[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) act_both<ACT>(v[j], v[j], d[j]);
    st_global_bf16x32(Aq + st.t * x.h + col0, v);
    st_global_bf16x32(dAct + st.t * x.h + col0, d);
    const size_t tc = ((size_t)st.b * x.h + col0) * x.C + st.s;
    st_bf16_cols(AqT + tc, x.C, v);
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] *= st.g;
    st_bf16_cols(AhqT + tc, x.C, v);
  }
  __device__ void end(St&) const {}
};
// transposed score gradient (rows = keys r): dS^T = -acc for s >= r; D^T = w * dS^T; and
// deta_r (+)= sum_s dS^T_rs S_sr / eta_r, with -S^T read from St
struct EpiDST {
  MCtx x;
  const __nv_bfloat16* StN;  // -S^T [NB, C, C]
  __nv_bfloat16* DT;         // [NB, C, C]
  float* deta;               // [BH, T]
  int accumulate;
  struct St {
    size_t tok0;
    int r;
    float eta, Lr, acc;
  };
  __device__ St begin(int b, int r) const {
    const size_t tok0 = (size_t)b * x.C;
    return {tok0, r, eta_at(x, tok0 + r), __ldg(x.Lb + tok0 + r), 0.f};
  }
  __device__ void chunk(St& st, int col0, float (&v)[32]) const {
    if (col0 + 31 >= st.r) {
      float sn[32], c[32];
      ld_bf16x32(StN + (st.tok0 + st.r) * x.C + col0, sn);
      ld_f32x32(x.Cf + st.tok0 + col0, c);
      const float rho = st.eta * __expf(__ldg(x.Lb + st.tok0 + col0) - st.Lr);
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const float ds = col0 + j >= st.r ? -v[j] : 0.f;
        st.acc -= ds * sn[j];
        v[j] = rho * c[j] * ds;
      }
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] = 0.f;
    }
    st_global_bf16x32(DT + (st.tok0 + st.r) * x.C + col0, v);
  }
  __device__ void end(St& st) const {
    float* d = deta + st.tok0 + st.r;
    *d = (accumulate ? *d : 0.f) + st.acc / st.eta;
  }
};
// dZq = acc * act'(Zq), Gamma dZq, dZq^T
struct EpiDZq {
  MCtx x;
  const __nv_bfloat16* dAct;
  __nv_bfloat16 *dZq, *dZqh, *dZqT;
  struct St {
    int b, s;
    size_t t;
    float g;
  };
  __device__ St begin(int b, int s) const {
    const size_t t = (size_t)b * x.C + s;
    return {b, s, t, __expf(__ldg(x.Lb + t))};
  }
  __device__ void chunk(St& st, int col0, float (&v)[32]) const {
    float d[32];
    ld_bf16x32(dAct + st.t * x.h + col0, d);
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] *= d[j];
    st_global_bf16x32(dZq + st.t * x.h + col0, v);
    st_bf16_cols(dZqT + ((size_t)st.b * x.h + col0) * x.C + st.s, x.C, v);
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] *= st.g;
    st_global_bf16x32(dZqh + st.t * x.h + col0, v);
  }
  __device__ void end(St&) const {}
};

// ---- serial steps (batch = head b, chunk c; token rows b T + c C + r)
struct SerCtx {
  MCtx x;
  int c;
  __device__ size_t tok(int b, int r) const { return (size_t)b * x.T + (size_t)c * x.C + r; }
  __device__ size_t tok0(int b) const { return (size_t)b * x.T + (size_t)c * x.C; }
};
// Yk = K Wh1: dG1 = dG1s - u Yk, Yk . G1, dB = dG1 act'(Z1) (and dB^T), dZ1a = dG1 Bm act''(Z1)
template <int ACT>
struct EpiYk {
  SerCtx sc;
  const __nv_bfloat16 *dG1s, *G1, *Bm;
  const float* Z1;
  __nv_bfloat16 *dB, *dBT;   // [BH, C, h], [BH, h, C]
  float* dZ1a;               // [BH, C, h]
  float* ykg;                // [BH, C]
  struct St {
    int b, r;
    size_t t;
    float u, acc;
  };
  __device__ St begin(int b, int r) const {
    return {b, r, sc.tok(b, r), u_at(sc.x, sc.tok0(b), sc.tok(b, r)), 0.f};
  }
  __device__ void chunk(St& st, int col0, float (&v)[32]) const {
    const int h = sc.x.h, C = sc.x.C;
    float a[32], z[32];
    ld_bf16x32(G1 + st.t * h + col0, a);
#pragma unroll
    for (int j = 0; j < 32; ++j) st.acc += v[j] * a[j];
    ld_bf16x32(dG1s + st.t * h + col0, a);
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] = a[j] - st.u * v[j];  // dG1
    ld_f32x32(Z1 + st.t * h + col0, z);
    ld_bf16x32(Bm + st.t * h + col0, a);
    float db[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      float d1 = 1.f, d2 = 0.f;
      if constexpr (ACT == 1) {
        const float s = sigm(z[j]);
        d1 = s * (1.f + z[j] * (1.f - s));
        d2 = s * (1.f - s) * (2.f + z[j] * (1.f - 2.f * s));
      }
      db[j] = v[j] * d1;
      a[j] = v[j] * a[j] * d2;
    }
    const size_t rr = (size_t)st.b * C + st.r;
    st_global_bf16x32(dB + rr * h + col0, db);
    st_bf16_cols(dBT + ((size_t)st.b * h + col0) * C + st.r, C, db);
    st_f32x32(dZ1a + rr * h + col0, a);
  }
  __device__ void end(St& st) const { ykg[(size_t)st.b * sc.x.C + st.r] = st.acc; }
};
// dA1 = dA1s + (-u G2) Wh2^T
struct EpiDA1 {
  SerCtx sc;
  const __nv_bfloat16* dA1s;
  float* dA1;                // [BH, C, h]
  __device__ Row begin(int b, int r) const { return {b, r}; }
  __device__ void chunk(Row& s, int col0, float (&v)[32]) const {
    float a[32];
    ld_bf16x32(dA1s + sc.tok(s.b, s.r) * sc.x.h + col0, a);
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] += a[j];
    st_f32x32(dA1 + ((size_t)s.b * sc.x.C + s.r) * sc.x.h + col0, v);
  }
  __device__ void end(Row&) const {}
};
// Ya = A1 Wh2 and Ya . G2
struct EpiYa {
  SerCtx sc;
  const __nv_bfloat16* G2;
  float *Ya, *yag;           // [BH, C, 64], [BH, C]
  struct St {
    int b, r;
    float acc;
  };
  __device__ St begin(int b, int r) const { return {b, r, 0.f}; }
  __device__ void chunk(St& st, int col0, float (&v)[32]) const {
    float g[32];
    ld_bf16x32(G2 + sc.tok(st.b, st.r) * D + col0, g);
#pragma unroll
    for (int j = 0; j < 32; ++j) st.acc += v[j] * g[j];
    st_f32x32(Ya + ((size_t)st.b * sc.x.C + st.r) * D + col0, v);
  }
  __device__ void end(St& st) const { yag[(size_t)st.b * sc.x.C + st.r] = st.acc; }
};
// dG2 = dG2s - u Ya + dB W2; dV = -dG2; dbeta from deta
struct EpiDG2 {
  SerCtx sc;
  const float *dG2s, *Ya, *ykg, *yag, *deta_s;
  __nv_bfloat16* dG2;        // [BH, C, 64]
  __nv_bfloat16* dV;
  float* dbeta;
  struct St {
    int b, r;
    size_t t;
    float u;
  };
  __device__ St begin(int b, int r) const {
    return {b, r, sc.tok(b, r), u_at(sc.x, sc.tok0(b), sc.tok(b, r))};
  }
  __device__ void chunk(St& st, int col0, float (&v)[32]) const {
    float a[32], y[32];
    ld_f32x32(dG2s + st.t * D + col0, a);
    const size_t rr = (size_t)st.b * sc.x.C + st.r;
    ld_f32x32(Ya + rr * D + col0, y);
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] += a[j] - st.u * y[j];
    st_global_bf16x32(dG2 + rr * D + col0, v);
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] = -v[j];
    st_global_bf16x32(dV + st.t * D + col0, v);
  }
  __device__ void end(St& st) const {
    const size_t rr = (size_t)st.b * sc.x.C + st.r;
    const float eta = eta_at(sc.x, st.t);
    const float e = __expf(__ldg(sc.x.Lb + sc.tok0(st.b) + sc.x.C - 1) - __ldg(sc.x.Lb + st.t));
    const float deta = deta_s[st.t] - e * (ykg[rr] + yag[rr]);
    dbeta[st.t] = deta * eta * (1.f - 0.5f * eta);
  }
};
// dZ1 = dZ1a + (dA1 + [MSE] dG2 W2^T) act'(Z1), and dZ1^T
template <int ACT>
struct EpiDZ1 {
  SerCtx sc;
  const float *dZ1a, *dA1, *Z1;
  __nv_bfloat16 *dZ1, *dZ1T;
  __device__ Row begin(int b, int r) const { return {b, r}; }
  __device__ void chunk(Row& s, int col0, float (&v)[32]) const {
    const int h = sc.x.h, C = sc.x.C;
    const size_t rr = (size_t)s.b * C + s.r;
    float a[32], z[32], d[32];
    ld_f32x32(dZ1a + rr * h + col0, a);
    ld_f32x32(dA1 + rr * h + col0, d);
    ld_f32x32(Z1 + sc.tok(s.b, s.r) * h + col0, z);
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      float f, d1;
      act_both<ACT>(z[j], f, d1);
      v[j] = a[j] + (d[j] + v[j]) * d1;
    }
    st_global_bf16x32(dZ1 + rr * h + col0, v);
    st_bf16_cols(dZ1T + ((size_t)s.b * h + col0) * C + s.r, C, v);
  }
  __device__ void end(Row&) const {}
};
// dK = dKs + acc
struct EpiDK {
  SerCtx sc;
  const float* dKs;
  __nv_bfloat16* dK;
  __device__ size_t begin(int b, int r) const { return sc.tok(b, r); }
  __device__ void chunk(size_t& t, int col0, float (&v)[32]) const {
    float a[32];
    ld_f32x32(dKs + t * D + col0, a);
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] += a[j];
    st_global_bf16x32(dK + t * D + col0, v);
  }
  __device__ void end(size_t&) const {}
};
// adjoint update of a weight held as [h, 64] rows: m <- Gamma_C m + acc; bf16 copies as
// [h, 64] and [64, h]; the chunk-0 result to out (transposed to [64, h] when out_t)
struct EpiAdj {
  SerCtx sc;
  float* m;                  // [BH, h, 64]
  __nv_bfloat16 *cp, *cpT;   // [BH, h, 64], [BH, 64, h]
  float* out;                // written at chunk 0
  int out_t;
  struct St {
    int b, i;
    float g;
  };
  __device__ St begin(int b, int i) const {
    return {b, i, __expf(__ldg(sc.x.Lb + sc.tok0(b) + sc.x.C - 1))};
  }
  __device__ void chunk(St& s, int col0, float (&v)[32]) const {
    const int h = sc.x.h;
    float w[32];
    float* p = m + ((size_t)s.b * h + s.i) * D + col0;
    ld_f32x32(p, w);
#pragma unroll
    for (int j = 0; j < 32; ++j) w[j] = s.g * w[j] + v[j];
    st_f32x32(p, w);
    st_global_bf16x32(cp + ((size_t)s.b * h + s.i) * D + col0, w);
    st_bf16_cols(cpT + ((size_t)s.b * D + col0) * h + s.i, h, w);
    if (sc.c == 0) {
      if (out_t) {
        float* dst = out + ((size_t)s.b * D + col0) * h + s.i;
#pragma unroll
        for (int j = 0; j < 32; ++j) dst[(size_t)j * h] = w[j];
      } else {
        st_f32x32(out + ((size_t)s.b * h + s.i) * D + col0, w);
      }
    }
  }
  __device__ void end(St&) const {}
};

// Per-chunk bf16 operand copies of the saved float32 chunk weights W1c [64, h], W2c [h, 64]:
// W1^T, W1, W2, W2^T; and the adjoint masters from dW1_final, dW2_final (or zero).
__global__ void __launch_bounds__(256)
    mlp_bwd_init_kernel(int h, int NC, const float* W1c, const float* W2c, const float* dW1f,
                        const float* dW2f, __nv_bfloat16* W1T, __nv_bfloat16* W1,
                        __nv_bfloat16* W2, __nv_bfloat16* W2T, float* Wh1m, float* Wh2m,
                        __nv_bfloat16* Wh1T_b, __nv_bfloat16* Wh1_b, __nv_bfloat16* Wh2_b,
                        __nv_bfloat16* Wh2T_b) {
  __shared__ float tile[32][33];
  const size_t bc = blockIdx.x, n = (size_t)h * D;
  transpose_to(W1c + bc * n, D, h, W1T + bc * n, (float*)nullptr, tile);
  transpose_to(W2c + bc * n, h, D, W2T + bc * n, (float*)nullptr, tile);
  copy_to(W1c + bc * n, n, W1 + bc * n, (float*)nullptr);
  copy_to(W2c + bc * n, n, W2 + bc * n, (float*)nullptr);
  if (bc % NC == 0) {
    const size_t b = bc / NC;
    transpose_to(dW1f ? dW1f + b * n : nullptr, D, h, Wh1m + b * n, Wh1T_b + b * n, tile);
    transpose_to(dW2f ? dW2f + b * n : nullptr, h, D, Wh2T_b + b * n, (float*)nullptr, tile);
    copy_to(dW1f ? dW1f + b * n : nullptr, n, Wh1_b + b * n, (float*)nullptr);
    copy_to(dW2f ? dW2f + b * n : nullptr, n, Wh2m + b * n, Wh2_b + b * n);
  }
}

struct BwdBufs {
  float *Lb, *Eb, *Cr, *Cf, *Z1, *dG2s, *dKs, *deta, *dZ1a, *dA1, *Ya, *ykg, *yag, *Wh1m, *Wh2m;
  __nv_bfloat16 *Qh, *dOh, *W1T, *W1, *W2, *W2T, *A1, *Bm, *G1, *uG1n, *Aq, *dAct, *dZq, *dZqh,
      *dA1s, *dG1s, *A1T, *G1T, *AqT, *AhqT, *dZqT, *G2, *uG2n, *S1n, *S1nT, *S2nT, *D2T, *D2,
      *D1T, *D1, *dB, *dBT, *dG2, *dZ1, *dZ1T, *Wh1T_b, *Wh1_b, *Wh2_b, *Wh2T_b;
};

size_t carve_bwd(const LayerArgs& a, int h, void* base, BwdBufs* f) {
  const size_t BH = (size_t)a.B * a.H, T = a.T, C = a.C, rows = BH * T;
  uint8_t* p = static_cast<uint8_t*>(base);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    void* r = p ? p + off : nullptr;
    off += up(bytes);
    return r;
  };
  auto bf = [&](size_t n) { return (__nv_bfloat16*)take(n * 2); };
  auto f32 = [&](size_t n) { return (float*)take(n * 4); };
  BwdBufs b{};
  b.Lb = f32(rows);
  b.Eb = f32(rows);
  b.Cr = f32(rows);
  b.Cf = f32(rows);
  b.deta = f32(rows);
  b.Qh = bf(rows * D);
  b.dOh = bf(rows * D);
  b.W1T = bf(rows / C * h * D);
  b.W1 = bf(rows / C * h * D);
  b.W2 = bf(rows / C * h * D);
  b.W2T = bf(rows / C * h * D);
  b.Z1 = f32(rows * h);
  __nv_bfloat16** hb[] = {&b.A1, &b.Bm, &b.G1, &b.uG1n, &b.Aq, &b.dAct, &b.dZq, &b.dZqh,
                          &b.dA1s, &b.dG1s, &b.A1T, &b.G1T, &b.AqT, &b.AhqT, &b.dZqT};
  for (auto q : hb) *q = bf(rows * h);
  b.G2 = bf(rows * D);
  b.uG2n = bf(rows * D);
  b.dG2s = f32(rows * D);
  b.dKs = f32(rows * D);
  __nv_bfloat16** cb[] = {&b.S1n, &b.S1nT, &b.S2nT, &b.D2T, &b.D2, &b.D1T, &b.D1};
  for (auto q : cb) *q = bf(rows * C);
  b.dB = bf(BH * C * h);
  b.dBT = bf(BH * C * h);
  b.dZ1a = f32(BH * C * h);
  b.dA1 = f32(BH * C * h);
  b.Ya = f32(BH * C * D);
  b.ykg = f32(BH * C);
  b.yag = f32(BH * C);
  b.dG2 = bf(BH * C * D);
  b.dZ1 = bf(BH * C * h);
  b.dZ1T = bf(BH * C * h);
  b.Wh1m = f32(BH * h * D);
  b.Wh2m = f32(BH * h * D);
  b.Wh1T_b = bf(BH * h * D);
  b.Wh1_b = bf(BH * h * D);
  b.Wh2_b = bf(BH * h * D);
  b.Wh2T_b = bf(BH * h * D);
  if (f) *f = b;
  return off;
}

template <int MN0, int MN1, int MN2, typename Epi>
cudaError_t gemm_h(int h, dim3 grid, const CUtensorMap* m, const bg::Prob& pr, const Epi& e,
                   unsigned* err, cudaStream_t s) {
  return h == 256 ? gemm<256, MN0, MN1, MN2>(grid, m, pr, e, err, s)
                  : gemm<128, MN0, MN1, MN2>(grid, m, pr, e, err, s);
}

template <int ACT>
cudaError_t mlp_tc_bwd_impl(const LayerArgs& a, int h, const float* W1c, const float* W2c,
                            const float* dW1f, const float* dW2f, float* dW1_0, float* dW2_0,
                            cudaStream_t s) {
  const int BH = a.B * a.H, T = a.T, C = a.C, NC = T / C, NB = BH * NC;
  BwdBufs f;
  carve_bwd(a, h, a.ws, &f);
  const auto* Q = static_cast<const __nv_bfloat16*>(a.Q);
  const auto* K = static_cast<const __nv_bfloat16*>(a.K);
  const auto* V = static_cast<const __nv_bfloat16*>(a.V);
  const auto* dO = static_cast<const __nv_bfloat16*>(a.dO);
  const MCtx x{T, C, NC, h, a.loss, f.Eb, f.Lb, f.Cr, f.Cf};
  cudaError_t e;
  mlp_scan_kernel<<<NB, 256, 0, s>>>(C, a.gamma, a.beta, a.lr_bias, Q, f.Lb, f.Eb, f.Cr, f.Cf,
                                     f.Qh, dO, f.dOh);
  mlp_bwd_init_kernel<<<NB, 256, 0, s>>>(h, NC, W1c, W2c, dW1f, dW2f, f.W1T, f.W1, f.W2, f.W2T,
                                          f.Wh1m, f.Wh2m, f.Wh1T_b, f.Wh1_b, f.Wh2_b, f.Wh2T_b);
  count_launches(2);
  if ((e = cudaGetLastError())) return e;
  // ------------------------------------------------ chunk-parallel phase (batch b h NC + c)
  auto tmr = [&](CUtensorMap* m, const void* p, int X, int box) {  // [NB, C, X] rows = tokens
    return tm3(m, p, X, C, NB, X, (uint64_t)C * X, box);
  };
  auto tmt = [&](CUtensorMap* m, const void* p, int X, int box) {  // [NB, X, C]
    return tm3(m, p, C, X, NB, C, (uint64_t)X * C, box);
  };
  CUtensorMap mK, mKb, mKmn, mQ, mQb, mQmn, mQh, mdO, mdOb, mdOmn, mdOh, mW1T, mW1, mW2, mW2T,
      mA1, mA1b, mA1T, mG2, mG2b, mG1, mG1b, mG1T, mS1n, mS1nT, mS2nT, mAq, mAqb, mAqT,
      mD2, mD2T, mD1, mD1T, mdZq, mdZqb, mdZqh, mdZqT;
  bool ok = tmr(&mK, K, D, 128) && tmr(&mKb, K, D, C) && tmr(&mKmn, K, D, 64) &&
            tmr(&mQ, Q, D, 128) && tmr(&mQb, Q, D, C) && tmr(&mQmn, Q, D, 64) &&
            tmr(&mQh, f.Qh, D, 128) && tmr(&mdO, dO, D, 128) && tmr(&mdOb, dO, D, C) &&
            tmr(&mdOmn, dO, D, 64) && tmr(&mdOh, f.dOh, D, 128) &&
            tm3(&mW1T, f.W1T, D, h, NB, D, (uint64_t)h * D, h) &&
            tm3(&mW1, f.W1, h, D, NB, h, (uint64_t)h * D, D) &&
            tm3(&mW2, f.W2, D, h, NB, D, (uint64_t)h * D, h) &&
            tm3(&mW2T, f.W2T, h, D, NB, h, (uint64_t)h * D, D) && tmr(&mA1, f.A1, h, 128) &&
            tmr(&mA1b, f.A1, h, C) && tmt(&mA1T, f.A1T, h, h) && tmr(&mG2, f.G2, D, 128) &&
            tmr(&mG2b, f.G2, D, C) && tmr(&mG1, f.G1, h, 128) && tmr(&mG1b, f.G1, h, C) &&
            tmt(&mG1T, f.G1T, h, h) && tmr(&mS1n, f.S1n, C, 128) &&
            tmr(&mS1nT, f.S1nT, C, 128) && tmr(&mS2nT, f.S2nT, C, 128) &&
            tmr(&mAq, f.Aq, h, 128) && tmr(&mAqb, f.Aq, h, C) && tmt(&mAqT, f.AqT, h, h) &&
            tmr(&mD2, f.D2, C, 128) && tmr(&mD2T, f.D2T, C, 128) && tmr(&mD1, f.D1, C, 128) &&
            tmr(&mD1T, f.D1T, C, 128) && tmr(&mdZq, f.dZq, h, 128) &&
            tmr(&mdZqb, f.dZq, h, C) && tmr(&mdZqh, f.dZqh, h, 128) &&
            tmt(&mdZqT, f.dZqT, h, h);
  if (!ok) return cudaErrorInvalidValue;
  const dim3 gP(C / 128, NB);
  const Tok tp{(size_t)C, 0};
  auto two = [](int K0, int K1) {
    bg::Prob p{};
    p.nterm = 2;
    p.t[0] = bg::Term{K0, 0, 0, 0, 0};
    p.t[1] = bg::Term{K1, 0, 0, 0, 0};
    return p;
  };
  auto gC = [&](auto ep, const CUtensorMap* m, const bg::Prob& pr) {  // N = C
    return C == 256 ? gemm<256, 0, 0, 0>(gP, m, pr, ep, a.err, s)
                    : gemm<128, 0, 0, 0>(gP, m, pr, ep, a.err, s);
  };
#define TRY(...) \
  if ((e = (__VA_ARGS__))) return e
  {
    const CUtensorMap m[6] = {mK, mW1T, mK, mK, mK, mK};
    TRY(gemm_h<0, 0, 0>(h, gP, m, prob1(D, 0, 0, 0, 0), EpiZ1b<ACT>{x, f.Z1, f.A1, f.A1T},
                           a.err, s));
  }
  {
    const CUtensorMap m[6] = {mA1, mW2T, mK, mK, mK, mK};
    TRY((gemm<64, 0, 0, 0>(gP, m, prob1(h, 0, 0, 0, 0), EpiG2b{x, V, f.G2, f.uG2n}, a.err, s)));
  }
  {
    const CUtensorMap m[6] = {mG2, mW2, mK, mK, mK, mK};
    TRY(gemm_h<0, 0, 0>(h, gP, m, prob1(D, 0, 0, 0, 0),
                           EpiG1b<ACT>{x, f.Z1, f.Bm, f.G1, f.G1T, f.uG1n}, a.err, s));
  }
  {
    const CUtensorMap m[6] = {mQ, mKb, mK, mK, mK, mK};
    TRY(gC(EpiScore{x, f.S1n}, m, prob1(D, 0, 0, 0, 0)));
    const CUtensorMap mt[6] = {mK, mQb, mK, mK, mK, mK};
    TRY(gC(EpiScoreT{x, f.S1nT}, mt, prob1(D, 0, 0, 0, 0)));
  }
  {
    const CUtensorMap m[6] = {mQh, mW1T, mS1n, mG1T, mK, mK};
    TRY(gemm_h<0, 0, 0>(h, gP, m, two(D, C), EpiAqb<ACT>{x, f.Aq, f.AqT, f.AhqT, f.dAct},
                           a.err, s));
  }
  {
    const CUtensorMap m[6] = {mA1, mAqb, mK, mK, mK, mK};
    TRY(gC(EpiScoreT{x, f.S2nT}, m, prob1(h, 0, 0, 0, 0)));
  }
  {
    const CUtensorMap m[6] = {mG2, mdOb, mK, mK, mK, mK};
    TRY(gC(EpiDST{x, f.S2nT, f.D2T, f.deta, 0}, m, prob1(D, 0, 0, 0, 0)));
    const CUtensorMap mb[6] = {mdO, mG2b, mK, mK, mK, mK};
    TRY(gC(EpiScore{x, f.D2}, mb, prob1(D, 0, 0, 0, 0)));
  }
  {
    const CUtensorMap m[6] = {mdOh, mW2, mD2, mA1T, mK, mK};
    TRY(gemm_h<0, 0, 0>(h, gP, m, two(D, C), EpiDZq{x, f.dAct, f.dZq, f.dZqh, f.dZqT}, a.err,
                           s));
  }
  {
    const CUtensorMap m[6] = {mD2T, mAqT, mK, mK, mK, mK};
    TRY(gemm_h<0, 0, 0>(h, gP, m, prob1(C, 0, 0, 0, 0),
                           EpiStore<__nv_bfloat16>{tp, f.dA1s, h}, a.err, s));
  }
  {
    const CUtensorMap m[6] = {mG1, mdZqb, mK, mK, mK, mK};
    TRY(gC(EpiDST{x, f.S1nT, f.D1T, f.deta, 1}, m, prob1(h, 0, 0, 0, 0)));
    const CUtensorMap mb[6] = {mdZq, mG1b, mK, mK, mK, mK};
    TRY(gC(EpiScore{x, f.D1}, mb, prob1(h, 0, 0, 0, 0)));
  }
  {
    const CUtensorMap m[6] = {mdZqh, mW1, mD1, mKmn, mK, mK};
    TRY((gemm<64, 0, 1, 0>(gP, m, two(h, C),
                           EpiStore<__nv_bfloat16>{tp, static_cast<__nv_bfloat16*>(a.dQ), D},
                           a.err, s)));
  }
  {
    const CUtensorMap m[6] = {mS1nT, mdZqT, mK, mK, mK, mK};
    TRY(gemm_h<0, 0, 0>(h, gP, m, prob1(C, 0, 0, 0, 0),
                           EpiStore<__nv_bfloat16>{tp, f.dG1s, h}, a.err, s));
  }
  {
    const CUtensorMap m[6] = {mS2nT, mdOmn, mK, mK, mK, mK};
    TRY((gemm<64, 1, 0, 0>(gP, m, prob1(C, 0, 0, 0, 0), EpiStore<float>{tp, f.dG2s, D}, a.err,
                           s)));
    const CUtensorMap mk[6] = {mD1T, mQmn, mK, mK, mK, mK};
    TRY((gemm<64, 1, 0, 0>(gP, mk, prob1(C, 0, 0, 0, 0),
                           EpiStore<float>{tp, f.dKs, D}, a.err, s)));
  }
  // ------------------------------------------------------ serial phase (batch = head)
  auto tms = [&](CUtensorMap* m, const void* p, int X, int rows, int box) {  // [BH, rows, X]
    return tm3(m, p, X, rows, BH, X, (uint64_t)rows * X, box);
  };
  CUtensorMap sK, sKmn, sQhmn, sdOmn, sA1, sG2mn, suG2n, suG1n, sWh1T, sWh1, sWh2, sWh2T, sdB,
      sdBT, sdG2, sdG2mn, sdZ1, sdZ1T;
  ok = tms(&sK, K, D, T, 128) && tms(&sKmn, K, D, T, 64) && tms(&sQhmn, f.Qh, D, T, 64) &&
       tms(&sdOmn, dO, D, T, 64) && tms(&sA1, f.A1, h, T, 128) && tms(&sG2mn, f.G2, D, T, 64) &&
       tms(&suG2n, f.uG2n, D, T, 128) && tms(&suG1n, f.uG1n, h, T, 128) &&
       tms(&sWh1T, f.Wh1T_b, D, h, h) && tms(&sWh1, f.Wh1_b, h, D, D) &&
       tms(&sWh2, f.Wh2_b, D, h, h) && tms(&sWh2T, f.Wh2T_b, h, D, D) &&
       tms(&sdB, f.dB, h, C, 128) && tms(&sdBT, f.dBT, C, h, 128) &&
       tms(&sdG2, f.dG2, D, C, 128) && tms(&sdG2mn, f.dG2, D, C, 64) &&
       tms(&sdZ1, f.dZ1, h, C, 128) && tms(&sdZ1T, f.dZ1T, C, h, 128);
  if (!ok) return cudaErrorInvalidValue;
  const dim3 gS(C / 128, BH), gW(h / 128, BH);
  const uint64_t wst = (uint64_t)NC * h * D, tst = (uint64_t)NC * h * C;
  for (int c = NC - 1; c >= 0; --c) {
    const SerCtx sc{x, c};
    CUtensorMap cW2T, cW2, cW1, cdZqT, cAhqT, cA1T;
    ok = tm3(&cW2T, f.W2T + (size_t)c * h * D, h, D, BH, h, wst, D) &&
         tm3(&cW2, f.W2 + (size_t)c * h * D, D, h, BH, D, wst, h) &&
         tm3(&cW1, f.W1 + (size_t)c * h * D, h, D, BH, h, wst, D) &&
         tm3(&cdZqT, f.dZqT + (size_t)c * h * C, C, h, BH, C, tst, 128) &&
         tm3(&cAhqT, f.AhqT + (size_t)c * h * C, C, h, BH, C, tst, 128) &&
         tm3(&cA1T, f.A1T + (size_t)c * h * C, C, h, BH, C, tst, 128);
    if (!ok) return cudaErrorInvalidValue;
    {  // Yk = K Wh1
      const CUtensorMap m[6] = {sK, sWh1T, sK, sK, sK, sK};
      TRY(gemm_h<0, 0, 0>(h, gS, m, prob1(D, 0, c * C, 0, 0),
                             EpiYk<ACT>{sc, f.dG1s, f.G1, f.Bm, f.Z1, f.dB, f.dBT, f.dZ1a, f.ykg},
                             a.err, s));
    }
    {  // dA1 = dA1s + (-u G2) Wh2^T
      const CUtensorMap m[6] = {suG2n, sWh2, sK, sK, sK, sK};
      TRY(gemm_h<0, 0, 0>(h, gS, m, prob1(D, 0, c * C, 0, 0), EpiDA1{sc, f.dA1s, f.dA1},
                             a.err, s));
    }
    {  // Ya = A1 Wh2
      const CUtensorMap m[6] = {sA1, sWh2T, sK, sK, sK, sK};
      TRY((gemm<64, 0, 0, 0>(gS, m, prob1(h, 0, c * C, 0, 0), EpiYa{sc, f.G2, f.Ya, f.yag},
                             a.err, s)));
    }
    {  // dG2 = dG2s - u Ya + dB W2
      const CUtensorMap m[6] = {sdB, cW2T, sK, sK, sK, sK};
      TRY((gemm<64, 0, 0, 0>(gS, m, prob1(h, 0, 0, 0, 0),
                             EpiDG2{sc, f.dG2s, f.Ya, f.ykg, f.yag, f.deta, f.dG2,
                                    static_cast<__nv_bfloat16*>(a.dV), a.dbeta},
                             a.err, s)));
    }
    {  // dZ1 = dZ1a + (dA1 + [MSE] dG2 W2^T) act'(Z1)
      const CUtensorMap m[6] = {sdG2, cW2, sK, sK, sK, sK};
      bg::Prob pr = prob1(D, 0, 0, 0, 0);
      if (a.loss != 0) pr.nterm = 0;
      TRY(gemm_h<0, 0, 0>(h, gS, m, pr, EpiDZ1<ACT>{sc, f.dZ1a, f.dA1, f.Z1, f.dZ1, f.dZ1T},
                             a.err, s));
    }
    {  // dK = dKs + (-u G1) Wh1^T + dZ1 W1^T
      const CUtensorMap m[6] = {suG1n, sWh1, sdZ1, cW1, sK, sK};
      bg::Prob pr{};
      pr.nterm = 2;
      pr.t[0] = bg::Term{h, 0, c * C, 0, 0};
      pr.t[1] = bg::Term{h, 0, 0, 0, 0};
      TRY((gemm<64, 0, 0, 0>(gS, m, pr,
                             EpiDK{sc, f.dKs, static_cast<__nv_bfloat16*>(a.dK)}, a.err, s)));
    }
    {  // Wh1^T <- Gamma_C Wh1^T + dZq^T Qhat + dZ1^T K
      const CUtensorMap m[6] = {cdZqT, sQhmn, sdZ1T, sKmn, sK, sK};
      bg::Prob pr{};
      pr.nterm = 2;
      pr.t[0] = bg::Term{C, 0, 0, 0, c * C};
      pr.t[1] = bg::Term{C, 0, 0, 0, c * C};
      TRY((gemm<64, 1, 1, 0>(gW, m, pr, EpiAdj{sc, f.Wh1m, f.Wh1T_b, f.Wh1_b, dW1_0, 1}, a.err,
                             s)));
    }
    {  // Wh2 <- Gamma_C Wh2 + (Gamma Aq)^T dO + dB^T G2 + [MSE] A1^T dG2
      const CUtensorMap m[6] = {cAhqT, sdOmn, sdBT, sG2mn, cA1T, sdG2mn};
      bg::Prob pr{};
      pr.nterm = a.loss == 0 ? 3 : 2;
      pr.t[0] = bg::Term{C, 0, 0, 0, c * C};
      pr.t[1] = bg::Term{C, 0, 0, 0, c * C};
      pr.t[2] = bg::Term{C, 0, 0, 0, 0};
      TRY((gemm<64, 1, 1, 1>(gW, m, pr, EpiAdj{sc, f.Wh2m, f.Wh2_b, f.Wh2T_b, dW2_0, 0}, a.err,
                             s)));
    }
  }
#undef TRY
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

size_t mlp_tc_bwd_workspace(const LayerArgs& a, int hidden) {
  return carve_bwd(a, hidden, nullptr, nullptr);
}

cudaError_t mlp_tc_bwd(const LayerArgs& a, int hidden, const float* W1c, const float* W2c,
                       const float* dW1f, const float* dW2f, float* dW1_0, float* dW2_0,
                       cudaStream_t s) {
  return a.act == 1 ? mlp_tc_bwd_impl<1>(a, hidden, W1c, W2c, dW1f, dW2f, dW1_0, dW2_0, s)
                    : mlp_tc_bwd_impl<0>(a, hidden, W1c, W2c, dW1f, dW2f, dW1_0, dW2_0, s);
}

}  // namespace tttk
