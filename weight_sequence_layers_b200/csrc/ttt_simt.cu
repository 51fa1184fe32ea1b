// SIMT (CUDA-core, float32 arithmetic) kernels of the chunkwise TTT layer.
//
// They serve the float32 configurations and bf16 shapes outside the tensor-core kernels'
// envelope. Both evaluate the chunk dual form of page "Modular TTT: Rethinking Test-Time
// Training as Composable Modules", section "方法步骤详情" (Algorithm 1): per chunk, with
// W0 the chunk-start fast weight,
//     Z  = K W0,  G = a(Z) * act'(Z)                 (train view + inner-loss gradient)
//     S_sr = eta_r exp(L_s - L_r) (q_s . k_r), r <= s (Tril of the scaled, decayed scores)
//     O  = act(diag(Gamma) Q W0 - S G)               (query view)
//     W_end = Gamma_C W0 - K^T diag(u) G,  u_r = eta_r exp(L_C - L_r)
// with eta = 2 sigmoid(beta + b) (section "内部学习规则与学习率参数化") and
// L_s = sum_{t<=s} log gamma_t (section "权重衰减"). With a per-feature (vector) decay, L_s has one
// entry per key feature i and scales row i of W, so the decay enters inside the contractions over
// the key features:
//     S_sr = eta_r sum_i q_si k_ri exp(L_si - L_ri),   Gamma Q W0 -> (Q * exp(L)) W0,
//     W_end = diag(exp(L_C)) W0 - sum_r eta_r (k_r * exp(L_C - L_r))^T g_r.
#include <cuda_bf16.h>
#include <math.h>

#include <algorithm>

#include "kernels.h"
#include "simt_util.cuh"

namespace tttk {
namespace {

constexpr int kNvs = 32;        // value columns per forward block
constexpr int kNvsNarrow = 8;   // ... when the grid would be small (few heads): 4x the blocks
constexpr int kRows = 32;       // query rows per score tile in the forward
constexpr int kMaxC = 256;
constexpr int kMaxD = 128;


struct Dims {
  int T, dk, dv, C, loss, act, has_gamma, gvec;
  float lr_bias;
  int w0_mod;
  int smem_floats;  // backward: dynamic shared memory (floats) its scratch arrays may move into
};

// Entries of the log-decay prefix per chunk position: one, or one per key feature.
__host__ __device__ inline int lwidth(const Dims& d) { return d.gvec ? d.dk : 1; }

// Prefix L at chunk position s for key feature i (the same for every i with a scalar decay).
__device__ __forceinline__ float Lat(const Dims& d, const float* L, int s, int i) {
  return d.gvec ? L[s * d.dk + i] : L[s];
}

// eta_s and the chunk-local log-decay prefix L for the C tokens of chunk c of head bh; L is
// [C] for a scalar decay and [C][dk] for a per-feature decay.
__device__ void chunk_scans(const Dims& d, const float* beta, const float* gamma, int bh, int c,
                            float* eta, float* L) {
  const size_t t0 = (size_t)bh * d.T + (size_t)c * d.C;
  const int w = lwidth(d);
  for (int s = threadIdx.x; s < d.C; s += blockDim.x) eta[s] = 2.f * sigm(beta[t0 + s] + d.lr_bias);
  for (int e = threadIdx.x; e < d.C * w; e += blockDim.x)
    L[e] = d.has_gamma ? logf(gamma[t0 * w + e]) : 0.f;
  __syncthreads();
  if (w == 1) {
    // scalar decay: one warp, each lane a run of C / 32 positions, then a shuffle scan
    if (threadIdx.x < 32) {
      const int lane = threadIdx.x, per = (d.C + 31) / 32, s0 = lane * per;
      float run = 0.f;
      for (int s = s0; s < min(s0 + per, d.C); ++s) run += L[s];
      float incl = run;
      for (int off = 1; off < 32; off <<= 1) {
        const float o = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += o;
      }
      float acc = incl - run;  // sum of the runs before this lane's
      for (int s = s0; s < min(s0 + per, d.C); ++s) {
        acc += L[s];
        L[s] = acc;
      }
    }
  } else {
    for (int i = threadIdx.x; i < w; i += blockDim.x)
      for (int s = 1; s < d.C; ++s) L[s * w + i] += L[(s - 1) * w + i];
  }
  __syncthreads();
}

// STG: the chunk's keys and queries are staged in shared memory (float32, rows padded to dk + 1
// so that the column walks of the element loops do not collide in one bank).
template <typename TI, int kNvs, bool STG>
__global__ void __launch_bounds__(256) simt_fwd_kernel(Dims d, const TI* Q, const TI* K,
                                                       const TI* V, const float* beta,
                                                       const float* gamma, const float* W0,
                                                       TI* O, float* Wf, TI* Wc, TI* Gs,
                                                       TI* Zs) {
  extern __shared__ float smem[];
  const int bh = blockIdx.y, j0 = blockIdx.x * kNvs;
  const int nv = min(kNvs, d.dv - j0);
  const int dk = d.dk, dv = d.dv, C = d.C, NC = d.T / d.C;
  float* Ws = smem;                  // [dk][kNvs] state slice
  float* G = Ws + dk * kNvs;         // [C][kNvs]
  float* S = G + C * kNvs;           // [kRows][C]
  float* eta = S + kRows * C;        // [C]
  float* L = eta + C;                // [C] or [C][dk]
  float* X = L + C * lwidth(d);      // [C + dk]: per-key factors of the transition
  const int ldk = dk + 1;
  float* Ks = X + C + dk;            // [C][dk + 1] (STG)
  float* Qs = Ks + C * ldk;          // [C][dk + 1] (STG)
  const size_t qk0 = (size_t)bh * d.T * dk, v0 = (size_t)bh * d.T * dv;
  for (int e = threadIdx.x; e < dk * nv; e += blockDim.x) {
    const int i = e / nv, j = e % nv;
    Ws[i * kNvs + j] = W0[(size_t)(bh % d.w0_mod) * dk * dv + (size_t)i * dv + j0 + j];
  }
  __syncthreads();
  for (int c = 0; c < NC; ++c) {
    if (Wc)
      for (int e = threadIdx.x; e < dk * nv; e += blockDim.x) {
        const int i = e / nv, j = e % nv;
        stf(&Wc[(((size_t)bh * NC + c) * dk + i) * dv + j0 + j], Ws[i * kNvs + j]);
      }
    const size_t tc = (size_t)c * C;
    if constexpr (STG)
      for (int e = threadIdx.x; e < C * dk; e += blockDim.x) {
        const int s = e / dk, i = e % dk;
        Ks[s * ldk + i] = ldf(K + qk0 + (tc + s) * dk + i);
        Qs[s * ldk + i] = ldf(Q + qk0 + (tc + s) * dk + i);
      }
    // key r / query s of the chunk, feature i
    auto kat = [&](int r, int i) -> float {
      if constexpr (STG) return Ks[r * ldk + i];
      else return ldf(K + qk0 + (tc + r) * dk + i);
    };
    auto qat = [&](int s, int i) -> float {
      if constexpr (STG) return Qs[s * ldk + i];
      else return ldf(Q + qk0 + (tc + s) * dk + i);
    };
    chunk_scans(d, beta, gamma, bh, c, eta, L);  // ends with a block barrier
    // train view: G = a(Z) * act'(Z), Z = K W0
    for (int e = threadIdx.x; e < C * nv; e += blockDim.x) {
      const int s = e / nv, j = e % nv;
      float z = 0.f;
      for (int i = 0; i < dk; ++i) z += kat(s, i) * Ws[i * kNvs + j];
      const float vv = ldf(V + v0 + (tc + s) * dv + j0 + j);
      const float a = d.loss == 0 ? actf(d.act, z) - vv : -vv;
      G[s * kNvs + j] = a * act1(d.act, z);
      if (Gs) stf(&Gs[v0 + (tc + s) * dv + j0 + j], G[s * kNvs + j]);
    }
    __syncthreads();
    // query view, kRows queries at a time
    for (int s0 = 0; s0 < C; s0 += kRows) {
      if (STG && !d.gvec) {
        // scalar decay with the chunk staged: the score tile as a register-tiled product, each
        // thread two query rows x four keys (keys r = kc + ncp u, so a warp's key rows fall in
        // distinct banks), then the decay, eta and the causal mask
        const int ncp = (C + 3) / 4;
        for (int pi = threadIdx.x; pi < (kRows / 2) * ncp; pi += blockDim.x) {
          const int rp = pi / ncp, kc = pi % ncp, sa = s0 + 2 * rp;
          float acc[2][4] = {};
          if (sa < C && kc <= sa + 1) {
            const float* qa = Qs + sa * ldk;
            const float* qb = Qs + min(sa + 1, C - 1) * ldk;
            const float* kr[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) kr[u] = Ks + min(kc + ncp * u, C - 1) * ldk;
#pragma unroll 4
            for (int i = 0; i < dk; ++i) {
              const float a0 = qa[i], a1 = qb[i];
#pragma unroll
              for (int u = 0; u < 4; ++u) {
                const float b = kr[u][i];
                acc[0][u] += a0 * b;
                acc[1][u] += a1 * b;
              }
            }
          }
#pragma unroll
          for (int v = 0; v < 2; ++v) {
            const int s = sa + v;
            float* Srow = S + (2 * rp + v) * C;
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const int r = kc + ncp * u;
              if (r < C) Srow[r] = s < C && r <= s ? eta[r] * expf(L[s] - L[r]) * acc[v][u] : 0.f;
            }
          }
        }
      } else
      // a warp per query row, its lanes over the key features
      for (int sr = threadIdx.x >> 5; sr < kRows; sr += blockDim.x >> 5) {
        const int s = s0 + sr, lane = threadIdx.x & 31;
        float* Srow = S + sr * C;
        if (s >= C) {
          for (int r = lane; r < C; r += 32) Srow[r] = 0.f;
          continue;
        }
        float qv[4], lv[4];
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const int i = lane + 32 * m;
          qv[m] = i < dk ? qat(s, i) : 0.f;
          lv[m] = i < dk && d.gvec ? L[s * dk + i] : 0.f;
        }
        const float Ls = d.gvec ? 0.f : L[s];
        const bool gv = d.gvec;
        warp_row_dots<4>(
            4, s + 1, [=](int m) { return qv[m]; },
            [=](int r, int m) {
              const int i = lane + 32 * m;
              if (i >= dk) return 0.f;
              const float kv = kat(r, i);
              return gv ? kv * __expf(lv[m] - L[r * dk + i]) : kv;
            },
            [=](int r, float p) {
              Srow[r] = gv ? eta[r] * p : eta[r] * expf(Ls - L[r]) * p;
            });
        for (int r = s + 1 + lane; r < C; r += 32) Srow[r] = 0.f;
      }
      __syncthreads();
      for (int e = threadIdx.x; e < kRows * nv; e += blockDim.x) {
        const int sr = e / nv, j = e % nv, s = s0 + sr;
        if (s >= C) continue;
        float acc = 0.f;
        if (d.gvec) {
          for (int i = 0; i < dk; ++i) acc += qat(s, i) * __expf(L[s * dk + i]) * Ws[i * kNvs + j];
        } else {
          for (int i = 0; i < dk; ++i) acc += qat(s, i) * Ws[i * kNvs + j];
          acc *= expf(L[s]);
        }
        for (int r = 0; r <= s; ++r) acc -= S[sr * C + r] * G[r * kNvs + j];
        if (Zs) stf(&Zs[v0 + (tc + s) * dv + j0 + j], acc);
        stf(&O[v0 + (tc + s) * dv + j0 + j], actf(d.act, acc));
      }
      __syncthreads();
    }
    // state transition; first the decayed, lr-weighted keys eta_r exp(L_C - L_r) k_r, one
    // exponential per key (and feature): into X for a scalar decay, over L (no longer needed in
    // this chunk) for a per-feature decay, with L_C kept in X
    if (d.gvec) {
      for (int i = threadIdx.x; i < dk; i += blockDim.x) X[i] = L[(C - 1) * dk + i];
      __syncthreads();
      for (int e = threadIdx.x; e < C * dk; e += blockDim.x) {
        const int r = e / dk, i = e % dk;
        L[e] = eta[r] * expf(X[i] - L[e]) * kat(r, i);
      }
    } else {
      for (int r = threadIdx.x; r < C; r += blockDim.x) X[r] = eta[r] * expf(L[C - 1] - L[r]);
      if (threadIdx.x == 0) X[C] = L[C - 1];
    }
    __syncthreads();
    for (int e = threadIdx.x; e < dk * nv; e += blockDim.x) {
      const int i = e / nv, j = e % nv;
      float w = expf(d.gvec ? X[i] : X[C]) * Ws[i * kNvs + j];
      if (d.gvec)
        for (int r = 0; r < C; ++r) w -= L[r * dk + i] * G[r * kNvs + j];
      else
        for (int r = 0; r < C; ++r) w -= X[r] * kat(r, i) * G[r * kNvs + j];
      Ws[i * kNvs + j] = w;
    }
    __syncthreads();
  }
  if (Wf)
    for (int e = threadIdx.x; e < dk * nv; e += blockDim.x) {
      const int i = e / nv, j = e % nv;
      Wf[(size_t)bh * dk * dv + (size_t)i * dv + j0 + j] = Ws[i * kNvs + j];
    }
}

// Per-head float32 scratch of the backward (in units of floats): Wh, Wn, W0 (dk x dv each) and
// the transposes of W0 and Wh (dv x dk each, for contractions over the value features with
// lanes over the key features),
// Z, G, dZq, Y, dG, dZ, Zq (C x dv each), S, dS (C x C each), eta, L, deta, dL (C each), one
// float for the chunk-end term of the decay gradient, and the decay-scaled operands
// q_s exp(L_s) and k_r exp(L_C - L_r) (C x dk each); with a per-feature decay also the prefix L
// and two parts of dJ/dL (C x dk each) and the chunk-end term per feature (dk).
__host__ __device__ inline size_t bwd_head_floats(int C, int dk, int dv, bool gvec) {
  return 5 * (size_t)dk * dv + 7 * (size_t)C * dv + 2 * (size_t)C * C + 4 * (size_t)C + 1 +
         2 * (size_t)C * dk + (gvec ? 3 * (size_t)C * dk + dk : 0);
}

// Analytic backward of the chunk dual form, reverse over chunks; one block per head.
// Wh carries dJ/dW at the chunk end; every intermediate lives in the head's scratch.
template <typename TI>
__global__ void __launch_bounds__(512) simt_bwd_kernel(
    Dims d, const TI* Q, const TI* K, const TI* V, const float* beta, const float* gamma,
    const TI* Wc, const TI* dO, const float* dWf, const float* Wfin, TI* dQ, TI* dK, TI* dV,
    float* dbeta, float* dW0, float* dgamma, float* ws) {
  const int bh = blockIdx.x;
  const int dk = d.dk, dv = d.dv, C = d.C, NC = d.T / d.C;
  float* Wh = ws + (size_t)bh * bwd_head_floats(C, dk, dv, d.gvec);
  float* Wn = Wh + dk * dv;
  float* W0 = Wn + dk * dv;  // float copy of the chunk-start state
  float* W0T = W0 + dk * dv; // W0 transposed [dv][dk]
  float* WhT = W0T + dk * dv; // Wh transposed [dv][dk]
  float* Z = WhT + dk * dv;
  float* G = Z + C * dv;
  float* DZQ = G + C * dv;
  float* Y = DZQ + C * dv;
  float* DG = Y + C * dv;
  float* DZ = DG + C * dv;
  float* S = DZ + C * dv;
  float* DS = S + C * C;
  float* eta = DS + C * C;
  float* L = eta + C;
  float* deta = L + C;
  float* ZQ = deta + C;
  float* dL = ZQ + C * dv;
  float* wend = dL + C;  // <W_end, dW_end> of the chunk
  float* QG = wend + 1;        // q_s exp(L_s)  [C][dk]
  float* KC = QG + C * dk;     // k_r exp(L_C - L_r)  [C][dk]
  float* dLq = KC + C * dk;    // per-feature decay: q_si dQ_si  [C][dk]
  float* dLk = dLq + C * dk;   //                    -k_si (dK_si - (dZ_s W0^T)_i)  [C][dk]
  float* wendv = dLk + C * dk; //                    row sums of W_end * dW_end  [dk]
  if (d.gvec) L = wendv + dk;  //                    log-decay prefix  [C][dk]
  {
    // The arrays the loops read most move into shared memory, as many as fit (the smallest and
    // most-read first); the rest stay in the head's global scratch. Every access goes through
    // these pointers, so either place serves.
    extern __shared__ float sm[];
    size_t used = 0;
    auto place = [&](float*& a, size_t n) {
      if (used + n <= (size_t)d.smem_floats) {
        a = sm + used;
        used += n;
      }
    };
    const size_t kv = (size_t)dk * dv, cv = (size_t)C * dv, ck = (size_t)C * dk;
    place(eta, C);
    place(L, d.gvec ? ck : C);
    place(deta, C);
    place(dL, C);
    place(wend, 1);
    place(S, (size_t)C * C);
    place(DS, (size_t)C * C);
    place(W0, kv);
    place(W0T, kv);
    place(Wh, kv);
    place(WhT, kv);
    place(G, cv);
    place(DZQ, cv);
    place(QG, ck);
    place(KC, ck);
    place(Y, cv);
    place(DG, cv);
    place(DZ, cv);
    place(Wn, kv);
    place(Z, cv);
    place(ZQ, cv);
    if (d.gvec) {
      place(dLq, ck);
      place(dLk, ck);
      place(wendv, dk);
    }
  }
  const size_t qk0 = (size_t)bh * d.T * dk, v0 = (size_t)bh * d.T * dv;
  for (int e = threadIdx.x; e < dk * dv; e += blockDim.x) {
    Wh[e] = dWf ? dWf[(size_t)bh * dk * dv + e] : 0.f;
    WhT[(e % dv) * dk + e / dv] = Wh[e];
  }
  __syncthreads();
  for (int c = NC - 1; c >= 0; --c) {
    const size_t tc = (size_t)c * C;
    for (int e = threadIdx.x; e < dk * dv; e += blockDim.x) {
      W0[e] = ldf(Wc + ((size_t)bh * NC + c) * dk * dv + e);
      W0T[(e % dv) * dk + e / dv] = W0[e];
    }
    chunk_scans(d, beta, gamma, bh, c, eta, L);  // ends with __syncthreads
    // the decay-scaled operands of the readout, the chunk-end route of the keys and the dW
    // update, one exponential per token and feature
    for (int e = threadIdx.x; e < C * dk; e += blockDim.x) {
      const int s = e / dk, i = e % dk;
      const float Ls = Lat(d, L, s, i);
      QG[e] = ldf(Q + qk0 + (tc + s) * dk + i) * expf(Ls);
      KC[e] = ldf(K + qk0 + (tc + s) * dk + i) * expf(Lat(d, L, C - 1, i) - Ls);
    }
    __syncthreads();
    // Z = K W0, G
    for (int e = threadIdx.x; e < C * dv; e += blockDim.x) {
      const int s = e / dv, j = e % dv;
      float z = 0.f;
      for (int i = 0; i < dk; ++i) z += ldf(K + qk0 + (tc + s) * dk + i) * W0[i * dv + j];
      const float vv = ldf(V + v0 + (tc + s) * dv + j);
      const float a = d.loss == 0 ? actf(d.act, z) - vv : -vv;
      Z[e] = z;
      G[e] = a * act1(d.act, z);
    }
    // S (causal, scaled): a warp per query row, its lanes over the key features
    for (int s = threadIdx.x >> 5; s < C; s += blockDim.x >> 5) {
      const int lane = threadIdx.x & 31;
      float qv[4], lv[4];
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const int i = lane + 32 * m;
        qv[m] = i < dk ? ldf(Q + qk0 + (tc + s) * dk + i) : 0.f;
        lv[m] = i < dk && d.gvec ? L[s * dk + i] : 0.f;
      }
      warp_row_dots<4>(
          4, s + 1, [&](int m) { return qv[m]; },
          [&](int r, int m) {
            const int i = lane + 32 * m;
            if (i >= dk) return 0.f;
            const float kv = ldf(K + qk0 + (tc + r) * dk + i);
            return d.gvec ? kv * __expf(lv[m] - L[r * dk + i]) : kv;
          },
          [&](int r, float p) {
            S[s * C + r] = eta[r] * p * (d.gvec ? 1.f : expf(L[s] - L[r]));
          });
      for (int r = s + 1 + lane; r < C; r += 32) S[s * C + r] = 0.f;
    }
    // Y_r = (k_r * exp(L_C - L_r)) Wh: the key's route into the chunk-end state
    for (int e = threadIdx.x; e < C * dv; e += blockDim.x) {
      const int r = e / dv, j = e % dv;
      float y = 0.f;
      for (int i = 0; i < dk; ++i) y += KC[r * dk + i] * Wh[i * dv + j];
      Y[e] = y;
    }
    __syncthreads();
    // dZq = dO * act'(Zq), Zq = Gamma Q W0 - S G
    for (int e = threadIdx.x; e < C * dv; e += blockDim.x) {
      const int s = e / dv, j = e % dv;
      float zq = 0.f;
      for (int i = 0; i < dk; ++i) zq += QG[s * dk + i] * W0[i * dv + j];
      for (int r = 0; r <= s; ++r) zq -= S[s * C + r] * G[r * dv + j];
      ZQ[e] = zq;
      DZQ[e] = ldf(dO + v0 + (tc + s) * dv + j) * act1(d.act, zq);
    }
    __syncthreads();
    // dS = -dZq G^T (causal): a warp per row, its lanes over the value features
    for (int s = threadIdx.x >> 5; s < C; s += blockDim.x >> 5) {
      const int lane = threadIdx.x & 31;
      float av[4];
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const int j = lane + 32 * m;
        av[m] = j < dv ? DZQ[s * dv + j] : 0.f;
      }
      warp_row_dots<4>(
          4, s + 1, [&](int m) { return av[m]; },
          [&](int r, int m) {
            const int j = lane + 32 * m;
            return j < dv ? G[r * dv + j] : 0.f;
          },
          [&](int r, float p) { DS[s * C + r] = -p; });
      for (int r = s + 1 + lane; r < C; r += 32) DS[s * C + r] = 0.f;
    }
    // dG = -S^T dZq - diag(u) Y
    for (int e = threadIdx.x; e < C * dv; e += blockDim.x) {
      const int r = e / dv, j = e % dv;
      float g = 0.f;
      for (int s = r; s < C; ++s) g -= S[s * C + r] * DZQ[s * dv + j];
      g -= eta[r] * Y[e];
      DG[e] = g;
    }
    __syncthreads();
    // deta_r = sum_s dS_sr P_sr exp(L_s - L_r) - exp(L_C - L_r) Y_r . G_r ;  dZ, dV
    for (int r = threadIdx.x; r < C; r += blockDim.x) {
      float acc = 0.f;
      for (int s = r; s < C; ++s) acc += DS[s * C + r] * S[s * C + r];
      acc /= eta[r];
      float yg = 0.f;
      for (int j = 0; j < dv; ++j) yg += Y[r * dv + j] * G[r * dv + j];
      deta[r] = acc - yg;
    }
    for (int e = threadIdx.x; e < C * dv; e += blockDim.x) {
      const int r = e / dv, j = e % dv;
      const float z = Z[e], d1 = act1(d.act, z);
      const float vv = ldf(V + v0 + (tc + r) * dv + j);
      const float a = d.loss == 0 ? actf(d.act, z) - vv : -vv;
      const float da = DG[e] * d1;
      DZ[e] = DG[e] * a * act2(d.act, z) + (d.loss == 0 ? da * d1 : 0.f);
      stf(&dV[v0 + (tc + r) * dv + j], -da);
    }
    __syncthreads();
    // dS * eta_r (and exp(L_s - L_r) with a scalar decay) in place: the causal weights of the
    // dQ and dK contractions; deta, the last reader of dS itself, is done
    for (int e = threadIdx.x; e < C * C; e += blockDim.x) {
      const int s = e / C, r = e % C;
      if (r <= s) DS[e] *= eta[r] * (d.gvec ? 1.f : expf(L[s] - L[r]));
    }
    __syncthreads();
    // dQ = diag(Gamma) dZq W0^T + (dS * M) K   (decay of feature i inside, per feature)
    for (int e = threadIdx.x; e < C * dk; e += blockDim.x) {
      const int s = e / dk, i = e % dk;
      const float Ls = Lat(d, L, s, i);
      float a1 = 0.f;
      for (int j = 0; j < dv; ++j) a1 += DZQ[s * dv + j] * W0T[j * dk + i];
      float acc = expf(Ls) * a1;
      if (d.gvec)
        for (int r = 0; r <= s; ++r)
          acc += DS[s * C + r] * __expf(Ls - L[r * dk + i]) * ldf(K + qk0 + (tc + r) * dk + i);
      else
        for (int r = 0; r <= s; ++r) acc += DS[s * C + r] * ldf(K + qk0 + (tc + r) * dk + i);
      stf(&dQ[qk0 + (tc + s) * dk + i], acc);
      if (d.gvec && dgamma) dLq[e] = ldf(Q + qk0 + (tc + s) * dk + i) * acc;
    }
    // dK = (dS * M)^T Q - diag(u) G Wh^T + dZ W0^T
    for (int e = threadIdx.x; e < C * dk; e += blockDim.x) {
      const int r = e / dk, i = e % dk;
      const float Lr = Lat(d, L, r, i);
      float acc = 0.f;
      if (d.gvec)
        for (int s = r; s < C; ++s)
          acc += DS[s * C + r] * __expf(L[s * dk + i] - Lr) * ldf(Q + qk0 + (tc + s) * dk + i);
      else
        for (int s = r; s < C; ++s) acc += DS[s * C + r] * ldf(Q + qk0 + (tc + s) * dk + i);
      float gw = 0.f, zw = 0.f;
      for (int j = 0; j < dv; ++j) {
        gw += G[r * dv + j] * WhT[j * dk + i];
        zw += DZ[r * dv + j] * W0T[j * dk + i];
      }
      acc += -eta[r] * expf(Lat(d, L, C - 1, i) - Lr) * gw;
      if (d.gvec && dgamma) dLk[e] = -ldf(K + qk0 + (tc + r) * dk + i) * acc;
      stf(&dK[qk0 + (tc + r) * dk + i], acc + zw);
    }
    for (int r = threadIdx.x; r < C; r += blockDim.x)
      dbeta[(size_t)bh * d.T + tc + r] = deta[r] * eta[r] * (1.f - 0.5f * eta[r]);
    if (dgamma && d.gvec) {
      // per feature: dJ/dL_si = q_si dQ_si - k_si (dK_si - (dZ_s W0^T)_i), plus the row-i part
      // of <W_end, dW_end> on the last token; dgamma_ti is the suffix sum over the chunk divided
      // by gamma_ti
      for (int i = threadIdx.x; i < dk; i += blockDim.x) {
        float acc = 0.f;
        if (c + 1 < NC || dWf)
          for (int j = 0; j < dv; ++j) {
            const float we = c + 1 < NC ? ldf(Wc + (((size_t)bh * NC + c + 1) * dk + i) * dv + j)
                                        : Wfin[((size_t)bh * dk + i) * dv + j];
            acc += we * Wh[i * dv + j];
          }
        wendv[i] = acc;
      }
      __syncthreads();
      for (int i = threadIdx.x; i < dk; i += blockDim.x) {
        float acc = wendv[i];
        for (int s2 = C - 1; s2 >= 0; --s2) {
          acc += dLq[s2 * dk + i] + dLk[s2 * dk + i];
          const size_t ti = ((size_t)bh * d.T + tc + s2) * dk + i;
          dgamma[ti] = acc / gamma[ti];
        }
      }
    } else if (dgamma) {
      // dJ/dL_s = dZq_s . Zq_s - g_s . dG_s, plus <W_end, dW_end> on the last token; dgamma_t is
      // the suffix sum over the chunk divided by gamma_t
      for (int s2 = threadIdx.x; s2 < C; s2 += blockDim.x) {
        float acc = 0.f;
        for (int j = 0; j < dv; ++j)
          acc += DZQ[s2 * dv + j] * ZQ[s2 * dv + j] - G[s2 * dv + j] * DG[s2 * dv + j];
        dL[s2] = acc;
      }
      if (threadIdx.x == 0) *wend = 0.f;
      __syncthreads();
      float part = 0.f;
      if (c + 1 < NC || dWf)
        for (int e = threadIdx.x; e < dk * dv; e += blockDim.x) {
          const float we = c + 1 < NC ? ldf(Wc + ((size_t)bh * NC + c + 1) * dk * dv + e)
                                      : Wfin[(size_t)bh * dk * dv + e];
          part += we * Wh[e];
        }
      atomicAdd(wend, part);
      __syncthreads();
      if (threadIdx.x == 0) {
        float acc = *wend;
        for (int s2 = C - 1; s2 >= 0; --s2) {
          acc += dL[s2];
          dgamma[(size_t)bh * d.T + tc + s2] = acc / gamma[(size_t)bh * d.T + tc + s2];
        }
      }
    }
    // dW at the chunk start = Gamma_C Wh + Q^T diag(Gamma) dZq + K^T dZ
    for (int e = threadIdx.x; e < dk * dv; e += blockDim.x) {
      const int i = e / dv, j = e % dv;
      float acc = expf(Lat(d, L, C - 1, i)) * Wh[e];
      for (int s = 0; s < C; ++s)
        acc += QG[s * dk + i] * DZQ[s * dv + j] + ldf(K + qk0 + (tc + s) * dk + i) * DZ[s * dv + j];
      Wn[e] = acc;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < dk * dv; e += blockDim.x) {
      Wh[e] = Wn[e];
      WhT[(e % dv) * dk + e / dv] = Wn[e];
    }
    __syncthreads();
  }
  for (int e = threadIdx.x; e < dk * dv; e += blockDim.x) dW0[(size_t)bh * dk * dv + e] = Wh[e];
}

Dims dims_of(const LayerArgs& a) {
  return Dims{a.T, a.dk, a.dv, a.C, a.loss, a.act, a.gamma != nullptr, a.gvec, a.lr_bias,
              a.w0_mod};
}

// Elements of one [B, H, T, dv] plane: with SiLU, Zq follows G in the saved buffer.
size_t zq_plane(const LayerArgs& a) { return (size_t)a.B * a.H * a.T * a.dv; }

size_t fwd_smem_bytes(const LayerArgs& a, int nvs = kNvs, bool stg = false) {
  const size_t lw = a.gvec ? a.dk : 1;
  return sizeof(float) * ((size_t)a.dk * nvs + (size_t)a.C * nvs + (size_t)kRows * a.C + a.C +
                           a.C * lw + a.C + 1 + a.dk + (stg ? 2 * (size_t)a.C * (a.dk + 1) : 0));
}
constexpr size_t kFwdStageMaxSmem = 160 * 1024;  // stage the chunk's keys and queries up to this

// Value columns per forward block: narrower slices when the wide ones would leave most SMs idle
// (each block recomputes the chunk's scores, so narrow slices trade that for parallelism).
int fwd_nvs(const LayerArgs& a) {
  const long blocks = (long)((a.dv + kNvs - 1) / kNvs) * a.B * a.H;
  return blocks < 64 ? kNvsNarrow : kNvs;
}

}  // namespace

bool simt_supported(const LayerArgs& a) {
  return a.dk >= 1 && a.dk <= kMaxD && a.dv >= 1 && a.dv <= kMaxD && a.C >= 1 && a.C <= kMaxC;
}

size_t simt_fwd_workspace(const LayerArgs&) { return 0; }

size_t simt_bwd_workspace(const LayerArgs& a) {
  return sizeof(float) * bwd_head_floats(a.C, a.dk, a.dv, a.gvec) * a.B * a.H;
}

template <int NVS, bool STG>
void simt_fwd_launch(const LayerArgs& a, const Dims& d, cudaStream_t s) {
  const size_t smem = fwd_smem_bytes(a, NVS, STG);
  dim3 grid((a.dv + NVS - 1) / NVS, a.B * a.H);
  if (a.dtype == 0) {
    auto k = simt_fwd_kernel<float, NVS, STG>;
    cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    float* gs = (float*)a.G_saved;
    k<<<grid, 256, smem, s>>>(d, (const float*)a.Q, (const float*)a.K, (const float*)a.V, a.beta,
                              a.gamma, a.W0, (float*)a.O, a.W_final, (float*)a.W_chunks, gs,
                              gs && a.act ? gs + zq_plane(a) : nullptr);
  } else {
    auto k = simt_fwd_kernel<__nv_bfloat16, NVS, STG>;
    cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    __nv_bfloat16* gs = (__nv_bfloat16*)a.G_saved;
    k<<<grid, 256, smem, s>>>(d, (const __nv_bfloat16*)a.Q, (const __nv_bfloat16*)a.K,
                              (const __nv_bfloat16*)a.V, a.beta, a.gamma, a.W0,
                              (__nv_bfloat16*)a.O, a.W_final, (__nv_bfloat16*)a.W_chunks, gs,
                              gs && a.act ? gs + zq_plane(a) : nullptr);
  }
}

cudaError_t simt_fwd(const LayerArgs& a, cudaStream_t s) {
  const Dims d = dims_of(a);
  const int nvs = fwd_nvs(a);
  const bool stg = fwd_smem_bytes(a, nvs, true) <= kFwdStageMaxSmem;
  if (nvs == kNvsNarrow)
    stg ? simt_fwd_launch<kNvsNarrow, true>(a, d, s) : simt_fwd_launch<kNvsNarrow, false>(a, d, s);
  else
    stg ? simt_fwd_launch<kNvs, true>(a, d, s) : simt_fwd_launch<kNvs, false>(a, d, s);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t simt_bwd(const LayerArgs& a, cudaStream_t s) {
  Dims d = dims_of(a);
  // as much of the head's scratch as fits in shared memory (up to 200 KB)
  const size_t hf = bwd_head_floats(a.C, a.dk, a.dv, a.gvec);
  d.smem_floats = (int)std::min<size_t>(hf, 200 * 1024 / sizeof(float));
  const size_t smem = (size_t)d.smem_floats * sizeof(float);
  if (a.dtype == 0) {
    auto k = simt_bwd_kernel<float>;
    cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    k<<<a.B * a.H, 512, smem, s>>>(
        d, (const float*)a.Q, (const float*)a.K, (const float*)a.V, a.beta, a.gamma,
        (const float*)a.W_chunks, (const float*)a.dO, a.dW_final, a.W_final_in, (float*)a.dQ,
        (float*)a.dK, (float*)a.dV, a.dbeta, a.dW0, a.dgamma, (float*)a.ws);
  } else {
    auto k = simt_bwd_kernel<__nv_bfloat16>;
    cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    k<<<a.B * a.H, 512, smem, s>>>(
        d, (const __nv_bfloat16*)a.Q, (const __nv_bfloat16*)a.K, (const __nv_bfloat16*)a.V,
        a.beta, a.gamma, (const __nv_bfloat16*)a.W_chunks, (const __nv_bfloat16*)a.dO,
        a.dW_final, a.W_final_in, (__nv_bfloat16*)a.dQ, (__nv_bfloat16*)a.dK,
        (__nv_bfloat16*)a.dV, a.dbeta, a.dW0, a.dgamma, (float*)a.ws);
  }
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace tttk
