// TTT-MLP on CUDA cores (float32 arithmetic): the fast weight is the two-layer network
// vhat = act(k W1) W2 of page "Modular TTT: Rethinking Test-Time Training as Composable
// Modules" (TTT-MLP, the two-layer learner of its ablations and throughput table), evaluated in
// the chunk dual form that Algorithm 1 ("方法步骤详情") composes from the per-primitive rules.
// Per chunk, with W1_0, W2_0 the chunk-start weights and w_sr = eta_r exp(L_s - L_r), r <= s:
//   Z1 = K W1_0, A1 = act(Z1), G2 = A1 W2_0 - V (MSE) or -V (IP), G1 = (G2 W2_0^T) * act'(Z1)
//   Zq_s = Gamma_s q_s W1_0 - sum_r w_sr (q_s . k_r) g1_r,      Aq = act(Zq)
//   o_s  = Gamma_s Aq_s W2_0 - sum_r w_sr (Aq_s . a1_r) g2_r
//   W1_end = Gamma_C W1_0 - K^T diag(u) G1,  W2_end = Gamma_C W2_0 - A1^T diag(u) G2,
// u_r = eta_r exp(L_C - L_r). The backward walks the chunks in reverse with the adjoints of
// both weights. One block per (batch, head); every intermediate lives in the head's float32
// scratch in the workspace.
#include <cuda_bf16.h>
#include <math.h>

#include "kernels.h"
#include "simt_util.cuh"

namespace tttk {
namespace {

struct MlpDims {
  int T, dk, dv, h, C, loss, act, has_gamma;
  float lr_bias;
  int w0_mod;
};

// Per-head scratch, in floats.
struct MlpScratch {
  float *W1, *W2, *Wh1, *Wh2, *Wn1, *Wn2;                                     // weights
  float *W1T, *W2T, *Wh1T;  // transposes of W1, W2, Wh1 (reads with lanes over the other index)
  float *Z1, *A1, *Bm, *G1, *Zq, *Aq, *dZq, *dA1, *dG1, *dB, *dZ1, *Yk;       // C x h
  float *G2, *dG2, *Ya;                                                       // C x dv
  float *S1, *S2, *dS1, *dS2;                                                 // C x C
  float *eta, *L, *deta;                                                      // C
};

__host__ __device__ inline size_t mlp_head_floats(int C, int dk, int dv, int h) {
  const size_t nW = (size_t)dk * h + (size_t)h * dv;
  return 4 * nW + (size_t)dk * h + 12 * (size_t)C * h + 3 * (size_t)C * dv + 4 * (size_t)C * C + 3 * (size_t)C;
}

__device__ MlpScratch carve(float* base, const MlpDims& d) {
  MlpScratch s;
  const size_t w1 = (size_t)d.dk * d.h, w2 = (size_t)d.h * d.dv, ch = (size_t)d.C * d.h,
               cv = (size_t)d.C * d.dv, cc = (size_t)d.C * d.C;
  float* p = base;
  s.W1 = p; p += w1; s.W2 = p; p += w2;
  s.Wh1 = p; p += w1; s.Wh2 = p; p += w2;
  s.Wn1 = p; p += w1; s.Wn2 = p; p += w2;
  s.W1T = p; p += w1; s.W2T = p; p += w2; s.Wh1T = p; p += w1;
  float** chs[] = {&s.Z1, &s.A1, &s.Bm, &s.G1, &s.Zq, &s.Aq, &s.dZq, &s.dA1, &s.dG1, &s.dB, &s.dZ1, &s.Yk};
  for (float** q : chs) { *q = p; p += ch; }
  s.G2 = p; p += cv; s.dG2 = p; p += cv; s.Ya = p; p += cv;
  s.S1 = p; p += cc; s.S2 = p; p += cc; s.dS1 = p; p += cc; s.dS2 = p; p += cc;
  s.eta = p; p += d.C; s.L = p; p += d.C; s.deta = p;
  return s;
}

// eta_s = 2 sigmoid(beta_s + b) and the chunk-local prefix L_s = sum_{t<=s} log gamma_t.
__device__ void mlp_scans(const MlpDims& d, const float* beta, const float* gamma, int bh, int c,
                          float* eta, float* L) {
  const size_t t0 = (size_t)bh * d.T + (size_t)c * d.C;
  for (int s = threadIdx.x; s < d.C; s += blockDim.x) {
    eta[s] = 2.f * sigm(beta[t0 + s] + d.lr_bias);
    L[s] = d.has_gamma ? logf(gamma[t0 + s]) : 0.f;
  }
  __syncthreads();
  if (threadIdx.x == 0)
    for (int s = 1; s < d.C; ++s) L[s] += L[s - 1];
  __syncthreads();
}

// The forward quantities of one chunk from its start weights (in S.W1, S.W2): Z1, A1, G2, Bm =
// G2 W2^T, G1, the two score matrices S1, S2 (decay and eta folded in), Zq and Aq.
template <typename TI>
__device__ void mlp_chunk_forward(const MlpDims& d, const MlpScratch& S, const TI* Qh,
                                  const TI* Kh, const TI* Vh) {
  const int C = d.C, dk = d.dk, dv = d.dv, h = d.h;
  for (int e = threadIdx.x; e < C * h; e += blockDim.x) {
    const int s = e / h, i = e % h;
    float z = 0.f;
    for (int k = 0; k < dk; ++k) z += ldf(Kh + (size_t)s * dk + k) * S.W1[k * h + i];
    S.Z1[e] = z;
    S.A1[e] = actf(d.act, z);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < C * dv; e += blockDim.x) {
    const int s = e / dv, j = e % dv;
    float vh = 0.f;
    for (int i = 0; i < h; ++i) vh += S.A1[s * h + i] * S.W2[i * dv + j];
    const float v = ldf(Vh + (size_t)s * dv + j);
    S.G2[e] = d.loss == 0 ? vh - v : -v;
  }
  // S1: a warp per query row, its lanes over the key features (dk <= 128)
  for (int s = threadIdx.x >> 5; s < C; s += blockDim.x >> 5) {
    const int lane = threadIdx.x & 31;
    warp_row_dots<0>(
        (dk + 31) / 32, s + 1,
        [&](int m) {
          const int k = lane + 32 * m;
          return k < dk ? ldf(Qh + (size_t)s * dk + k) : 0.f;
        },
        [&](int r, int m) {
          const int k = lane + 32 * m;
          return k < dk ? ldf(Kh + (size_t)r * dk + k) : 0.f;
        },
        [&](int r, float p) { S.S1[s * C + r] = S.eta[r] * expf(S.L[s] - S.L[r]) * p; });
    for (int r = s + 1 + lane; r < C; r += 32) S.S1[s * C + r] = 0.f;
  }
  __syncthreads();
  for (int e = threadIdx.x; e < C * h; e += blockDim.x) {
    const int s = e / h, i = e % h;
    float b = 0.f;
    for (int j = 0; j < dv; ++j) b += S.G2[s * dv + j] * S.W2T[j * h + i];
    S.Bm[e] = b;
    S.G1[e] = b * act1(d.act, S.Z1[e]);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < C * h; e += blockDim.x) {
    const int s = e / h, i = e % h;
    float y = 0.f;
    for (int k = 0; k < dk; ++k) y += ldf(Qh + (size_t)s * dk + k) * S.W1[k * h + i];
    float zq = expf(S.L[s]) * y;
    for (int r = 0; r <= s; ++r) zq -= S.S1[s * C + r] * S.G1[r * h + i];
    S.Zq[e] = zq;
    S.Aq[e] = actf(d.act, zq);
  }
  __syncthreads();
  // S2: a warp per query row, its lanes over the hidden features (h <= 512)
  for (int s = threadIdx.x >> 5; s < C; s += blockDim.x >> 5) {
    const int lane = threadIdx.x & 31;
    warp_row_dots<0>(
        (h + 31) / 32, s + 1,
        [&](int m) {
          const int i = lane + 32 * m;
          return i < h ? S.Aq[s * h + i] : 0.f;
        },
        [&](int r, int m) {
          const int i = lane + 32 * m;
          return i < h ? S.A1[r * h + i] : 0.f;
        },
        [&](int r, float p) { S.S2[s * C + r] = S.eta[r] * expf(S.L[s] - S.L[r]) * p; });
    for (int r = s + 1 + lane; r < C; r += 32) S.S2[s * C + r] = 0.f;
  }
  __syncthreads();
}

template <typename TI>
__global__ void __launch_bounds__(512)
    mlp_fwd_kernel(MlpDims d, const TI* Q, const TI* K, const TI* V, const float* beta,
                   const float* gamma, const float* W1_0, const float* W2_0, TI* O, float* W1f,
                   float* W2f, float* W1c, float* W2c, float* ws) {
  const int bh = blockIdx.x;
  const int C = d.C, dk = d.dk, dv = d.dv, h = d.h, NC = d.T / d.C;
  const MlpScratch S = carve(ws + (size_t)bh * mlp_head_floats(C, dk, dv, h), d);
  const size_t n1 = (size_t)dk * h, n2 = (size_t)h * dv;
  const size_t b0 = (size_t)(bh % d.w0_mod);
  for (size_t e = threadIdx.x; e < n1; e += blockDim.x) S.W1[e] = W1_0[b0 * n1 + e];
  for (size_t e = threadIdx.x; e < n2; e += blockDim.x) {
    S.W2[e] = W2_0[b0 * n2 + e];
    S.W2T[(e % dv) * h + e / dv] = S.W2[e];
  }
  __syncthreads();
  for (int c = 0; c < NC; ++c) {
    const size_t tok = (size_t)bh * d.T + (size_t)c * C;
    if (W1c)
      for (size_t e = threadIdx.x; e < n1; e += blockDim.x)
        W1c[((size_t)bh * NC + c) * n1 + e] = S.W1[e];
    if (W2c)
      for (size_t e = threadIdx.x; e < n2; e += blockDim.x)
        W2c[((size_t)bh * NC + c) * n2 + e] = S.W2[e];
    mlp_scans(d, beta, gamma, bh, c, S.eta, S.L);
    mlp_chunk_forward(d, S, Q + tok * dk, K + tok * dk, V + tok * dv);
    for (int e = threadIdx.x; e < C * dv; e += blockDim.x) {
      const int s = e / dv, j = e % dv;
      float y = 0.f;
      for (int i = 0; i < h; ++i) y += S.Aq[s * h + i] * S.W2[i * dv + j];
      float o = expf(S.L[s]) * y;
      for (int r = 0; r <= s; ++r) o -= S.S2[s * C + r] * S.G2[r * dv + j];
      stf(O + (tok + s) * dv + j, o);
    }
    // state transition of both layers
    const float LC = S.L[C - 1];
    for (size_t e = threadIdx.x; e < n1; e += blockDim.x) {
      const int k = (int)(e / h), i = (int)(e % h);
      float w = expf(LC) * S.W1[e];
      for (int r = 0; r < C; ++r)
        w -= S.eta[r] * expf(LC - S.L[r]) * ldf(K + (tok + r) * dk + k) * S.G1[r * h + i];
      S.Wn1[e] = w;
    }
    for (size_t e = threadIdx.x; e < n2; e += blockDim.x) {
      const int i = (int)(e / dv), j = (int)(e % dv);
      float w = expf(LC) * S.W2[e];
      for (int r = 0; r < C; ++r)
        w -= S.eta[r] * expf(LC - S.L[r]) * S.A1[r * h + i] * S.G2[r * dv + j];
      S.Wn2[e] = w;
    }
    __syncthreads();
    for (size_t e = threadIdx.x; e < n1; e += blockDim.x) S.W1[e] = S.Wn1[e];
    for (size_t e = threadIdx.x; e < n2; e += blockDim.x) {
      S.W2[e] = S.Wn2[e];
      S.W2T[(e % dv) * h + e / dv] = S.Wn2[e];
    }
    __syncthreads();
  }
  if (W1f)
    for (size_t e = threadIdx.x; e < n1; e += blockDim.x) W1f[bh * n1 + e] = S.W1[e];
  if (W2f)
    for (size_t e = threadIdx.x; e < n2; e += blockDim.x) W2f[bh * n2 + e] = S.W2[e];
}

// Reverse over chunks for J = <dO, O> + <dW1_T, W1_final> + <dW2_T, W2_final>.
template <typename TI>
__global__ void __launch_bounds__(512)
    mlp_bwd_kernel(MlpDims d, const TI* Q, const TI* K, const TI* V, const float* beta,
                   const float* gamma, const float* W1c, const float* W2c, const TI* dO,
                   const float* dW1f, const float* dW2f, TI* dQ, TI* dK, TI* dV, float* dbeta,
                   float* dW1_0, float* dW2_0, float* ws) {
  const int bh = blockIdx.x;
  const int C = d.C, dk = d.dk, dv = d.dv, h = d.h, NC = d.T / d.C;
  const bool mse = d.loss == 0;
  const MlpScratch S = carve(ws + (size_t)bh * mlp_head_floats(C, dk, dv, h), d);
  const size_t n1 = (size_t)dk * h, n2 = (size_t)h * dv;
  for (size_t e = threadIdx.x; e < n1; e += blockDim.x) {
    S.Wh1[e] = dW1f ? dW1f[bh * n1 + e] : 0.f;
    S.Wh1T[(e % h) * dk + e / h] = S.Wh1[e];
  }
  for (size_t e = threadIdx.x; e < n2; e += blockDim.x) S.Wh2[e] = dW2f ? dW2f[bh * n2 + e] : 0.f;
  for (int c = NC - 1; c >= 0; --c) {
    const size_t tok = (size_t)bh * d.T + (size_t)c * C;
    const TI *Qh = Q + tok * dk, *Kh = K + tok * dk, *dOh = dO + tok * dv;
    for (size_t e = threadIdx.x; e < n1; e += blockDim.x) {
      S.W1[e] = W1c[((size_t)bh * NC + c) * n1 + e];
      S.W1T[(e % h) * dk + e / h] = S.W1[e];
    }
    for (size_t e = threadIdx.x; e < n2; e += blockDim.x) {
      S.W2[e] = W2c[((size_t)bh * NC + c) * n2 + e];
      S.W2T[(e % dv) * h + e / dv] = S.W2[e];
    }
    mlp_scans(d, beta, gamma, bh, c, S.eta, S.L);  // ends with a barrier
    mlp_chunk_forward(d, S, Qh, Kh, V + tok * dv);
    const float LC = S.L[C - 1];
    // routes of the keys and hidden activations into the chunk-end weights
    for (int e = threadIdx.x; e < C * h; e += blockDim.x) {
      const int r = e / h, i = e % h;
      float y = 0.f;
      for (int k = 0; k < dk; ++k) y += ldf(Kh + (size_t)r * dk + k) * S.Wh1[k * h + i];
      S.Yk[e] = y;
    }
    for (int e = threadIdx.x; e < C * dv; e += blockDim.x) {
      const int r = e / dv, j = e % dv;
      float y = 0.f;
      for (int i = 0; i < h; ++i) y += S.A1[r * h + i] * S.Wh2[i * dv + j];
      S.Ya[e] = y;
    }
    // output layer: dS2 = -dO G2^T (causal), a warp per row, its lanes over the value features
    for (int s = threadIdx.x >> 5; s < C; s += blockDim.x >> 5) {
      const int lane = threadIdx.x & 31;
      warp_row_dots<0>(
          (dv + 31) / 32, s + 1,
          [&](int m) {
            const int j = lane + 32 * m;
            return j < dv ? ldf(dOh + (size_t)s * dv + j) : 0.f;
          },
          [&](int r, int m) {
            const int j = lane + 32 * m;
            return j < dv ? S.G2[r * dv + j] : 0.f;
          },
          [&](int r, float p) { S.dS2[s * C + r] = -p; });
      for (int r = s + 1 + lane; r < C; r += 32) S.dS2[s * C + r] = 0.f;
    }
    __syncthreads();
    // dG2 (readout and transition parts), dAq -> dZq, dA1 (score and transition parts)
    for (int e = threadIdx.x; e < C * dv; e += blockDim.x) {
      const int r = e / dv, j = e % dv;
      float g = 0.f;
      for (int s = r; s < C; ++s) g -= S.S2[s * C + r] * ldf(dOh + (size_t)s * dv + j);
      S.dG2[e] = g - S.eta[r] * expf(LC - S.L[r]) * S.Ya[e];
    }
    for (int e = threadIdx.x; e < C * h; e += blockDim.x) {
      const int s = e / h, i = e % h;
      float a = 0.f;
      for (int j = 0; j < dv; ++j) a += ldf(dOh + (size_t)s * dv + j) * S.W2T[j * h + i];
      a *= expf(S.L[s]);
      for (int r = 0; r <= s; ++r)
        a += S.dS2[s * C + r] * S.eta[r] * expf(S.L[s] - S.L[r]) * S.A1[r * h + i];
      S.dZq[e] = a * act1(d.act, S.Zq[e]);
    }
    for (int e = threadIdx.x; e < C * h; e += blockDim.x) {
      const int r = e / h, i = e % h;
      float a = 0.f;
      for (int s = r; s < C; ++s)
        a += S.dS2[s * C + r] * S.eta[r] * expf(S.L[s] - S.L[r]) * S.Aq[s * h + i];
      float gw = 0.f;
      for (int j = 0; j < dv; ++j) gw += S.G2[r * dv + j] * S.Wh2[i * dv + j];
      S.dA1[e] = a - S.eta[r] * expf(LC - S.L[r]) * gw;
    }
    __syncthreads();
    // first layer: dS1 = -dZq G1^T (causal), a warp per row, its lanes over the hidden features
    for (int s = threadIdx.x >> 5; s < C; s += blockDim.x >> 5) {
      const int lane = threadIdx.x & 31;
      warp_row_dots<0>(
          (h + 31) / 32, s + 1,
          [&](int m) {
            const int i = lane + 32 * m;
            return i < h ? S.dZq[s * h + i] : 0.f;
          },
          [&](int r, int m) {
            const int i = lane + 32 * m;
            return i < h ? S.G1[r * h + i] : 0.f;
          },
          [&](int r, float p) { S.dS1[s * C + r] = -p; });
      for (int r = s + 1 + lane; r < C; r += 32) S.dS1[s * C + r] = 0.f;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < C * h; e += blockDim.x) {
      const int r = e / h, i = e % h;
      float g = 0.f;
      for (int s = r; s < C; ++s) g -= S.S1[s * C + r] * S.dZq[s * h + i];
      S.dG1[e] = g - S.eta[r] * expf(LC - S.L[r]) * S.Yk[e];
    }
    for (int e = threadIdx.x; e < C * dk; e += blockDim.x) {
      const int s = e / dk, k = e % dk;
      float a = 0.f;
      for (int i = 0; i < h; ++i) a += S.dZq[s * h + i] * S.W1T[i * dk + k];
      a *= expf(S.L[s]);
      for (int r = 0; r <= s; ++r)
        a += S.dS1[s * C + r] * S.eta[r] * expf(S.L[s] - S.L[r]) * ldf(Kh + (size_t)r * dk + k);
      stf(dQ + (tok + s) * dk + k, a);
    }
    for (int r = threadIdx.x; r < C; r += blockDim.x) {
      float acc = 0.f;
      for (int s = r; s < C; ++s)
        acc += S.dS1[s * C + r] * S.S1[s * C + r] + S.dS2[s * C + r] * S.S2[s * C + r];
      acc /= S.eta[r];
      float y = 0.f;
      for (int i = 0; i < h; ++i) y += S.Yk[r * h + i] * S.G1[r * h + i];
      for (int j = 0; j < dv; ++j) y += S.Ya[r * dv + j] * S.G2[r * dv + j];
      S.deta[r] = acc - expf(LC - S.L[r]) * y;
    }
    __syncthreads();
    // train view: G1 = Bm * act'(Z1) with Bm = G2 W2^T; dZ1 collects act'' and act' terms
    for (int e = threadIdx.x; e < C * h; e += blockDim.x) {
      const float z = S.Z1[e];
      S.dB[e] = S.dG1[e] * act1(d.act, z);
      S.dZ1[e] = S.dG1[e] * S.Bm[e] * act2(d.act, z);
    }
    __syncthreads();
    // dG2 in full; dV = -dG2 and, for MSE, dVhat = dG2 (kept in dG2)
    for (int e = threadIdx.x; e < C * dv; e += blockDim.x) {
      const int r = e / dv, j = e % dv;
      float g = S.dG2[e];
      for (int i = 0; i < h; ++i) g += S.dB[r * h + i] * S.W2[i * dv + j];
      S.dG2[e] = g;
      stf(dV + (tok + r) * dv + j, -g);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < C * h; e += blockDim.x) {
      const int r = e / h, i = e % h;
      float a = S.dA1[e];
      if (mse)
        for (int j = 0; j < dv; ++j) a += S.dG2[r * dv + j] * S.W2T[j * h + i];
      S.dZ1[e] += a * act1(d.act, S.Z1[e]);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < C * dk; e += blockDim.x) {
      const int r = e / dk, k = e % dk;
      float a = 0.f;
      for (int s = r; s < C; ++s)
        a += S.dS1[s * C + r] * S.eta[r] * expf(S.L[s] - S.L[r]) * ldf(Qh + (size_t)s * dk + k);
      float gw = 0.f, zw = 0.f;
      for (int i = 0; i < h; ++i) {
        gw += S.G1[r * h + i] * S.Wh1T[i * dk + k];
        zw += S.dZ1[r * h + i] * S.W1T[i * dk + k];
      }
      stf(dK + (tok + r) * dk + k, a - S.eta[r] * expf(LC - S.L[r]) * gw + zw);
    }
    for (int r = threadIdx.x; r < C; r += blockDim.x)
      dbeta[tok + r] = S.deta[r] * S.eta[r] * (1.f - 0.5f * S.eta[r]);
    // adjoints at the chunk start
    for (size_t e = threadIdx.x; e < n1; e += blockDim.x) {
      const int k = (int)(e / h), i = (int)(e % h);
      float acc = expf(LC) * S.Wh1[e];
      for (int s = 0; s < C; ++s)
        acc += expf(S.L[s]) * ldf(Qh + (size_t)s * dk + k) * S.dZq[s * h + i] +
               ldf(Kh + (size_t)s * dk + k) * S.dZ1[s * h + i];
      S.Wn1[e] = acc;
    }
    for (size_t e = threadIdx.x; e < n2; e += blockDim.x) {
      const int i = (int)(e / dv), j = (int)(e % dv);
      float acc = expf(LC) * S.Wh2[e];
      for (int s = 0; s < C; ++s) {
        acc += expf(S.L[s]) * S.Aq[s * h + i] * ldf(dOh + (size_t)s * dv + j) +
               S.dB[s * h + i] * S.G2[s * dv + j];
        if (mse) acc += S.A1[s * h + i] * S.dG2[s * dv + j];
      }
      S.Wn2[e] = acc;
    }
    __syncthreads();
    for (size_t e = threadIdx.x; e < n1; e += blockDim.x) {
      S.Wh1[e] = S.Wn1[e];
      S.Wh1T[(e % h) * dk + e / h] = S.Wn1[e];
    }
    for (size_t e = threadIdx.x; e < n2; e += blockDim.x) S.Wh2[e] = S.Wn2[e];
    __syncthreads();
  }
  for (size_t e = threadIdx.x; e < n1; e += blockDim.x) dW1_0[bh * n1 + e] = S.Wh1[e];
  for (size_t e = threadIdx.x; e < n2; e += blockDim.x) dW2_0[bh * n2 + e] = S.Wh2[e];
}

MlpDims mlp_dims(const LayerArgs& a, int hidden) {
  return MlpDims{a.T, a.dk, a.dv, hidden, a.C, a.loss, a.act, a.gamma != nullptr, a.lr_bias,
                 a.w0_mod};
}

}  // namespace

bool mlp_supported(const LayerArgs& a, int hidden) {
  return !a.gvec && a.dk >= 1 && a.dk <= 128 && a.dv >= 1 && a.dv <= 128 && hidden >= 1 &&
         hidden <= 512 && a.C >= 1 && a.C <= 256;
}

size_t mlp_workspace(const LayerArgs& a, int hidden) {
  return sizeof(float) * mlp_head_floats(a.C, a.dk, a.dv, hidden) * a.B * a.H;
}

cudaError_t mlp_fwd(const LayerArgs& a, int hidden, const float* W1_0, const float* W2_0,
                    float* W1f, float* W2f, float* W1c, float* W2c, cudaStream_t s) {
  const MlpDims d = mlp_dims(a, hidden);
  float* ws = static_cast<float*>(a.ws);
  if (a.dtype == 0)
    mlp_fwd_kernel<float><<<a.B * a.H, 512, 0, s>>>(
        d, (const float*)a.Q, (const float*)a.K, (const float*)a.V, a.beta, a.gamma, W1_0, W2_0,
        (float*)a.O, W1f, W2f, W1c, W2c, ws);
  else
    mlp_fwd_kernel<__nv_bfloat16><<<a.B * a.H, 512, 0, s>>>(
        d, (const __nv_bfloat16*)a.Q, (const __nv_bfloat16*)a.K, (const __nv_bfloat16*)a.V,
        a.beta, a.gamma, W1_0, W2_0, (__nv_bfloat16*)a.O, W1f, W2f, W1c, W2c, ws);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t mlp_bwd(const LayerArgs& a, int hidden, const float* W1c, const float* W2c,
                    const float* dW1f, const float* dW2f, float* dW1_0, float* dW2_0,
                    cudaStream_t s) {
  const MlpDims d = mlp_dims(a, hidden);
  float* ws = static_cast<float*>(a.ws);
  if (a.dtype == 0)
    mlp_bwd_kernel<float><<<a.B * a.H, 512, 0, s>>>(
        d, (const float*)a.Q, (const float*)a.K, (const float*)a.V, a.beta, a.gamma, W1c, W2c,
        (const float*)a.dO, dW1f, dW2f, (float*)a.dQ, (float*)a.dK, (float*)a.dV, a.dbeta, dW1_0,
        dW2_0, ws);
  else
    mlp_bwd_kernel<__nv_bfloat16><<<a.B * a.H, 512, 0, s>>>(
        d, (const __nv_bfloat16*)a.Q, (const __nv_bfloat16*)a.K, (const __nv_bfloat16*)a.V,
        a.beta, a.gamma, W1c, W2c, (const __nv_bfloat16*)a.dO, dW1f, dW2f, (__nv_bfloat16*)a.dQ,
        (__nv_bfloat16*)a.dK, (__nv_bfloat16*)a.dV, a.dbeta, dW1_0, dW2_0, ws);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace tttk
