// CPU oracle for the chunkwise test-time-training (TTT) layer.
//
// TEST INFRASTRUCTURE ONLY. Nothing on the product path may link, load or
// call this file: only tests/, __graft_entry__.smoke() and bench.py's
// cpu_baseline / reference leg use it. It shares no code, header, table or
// helper with the CUDA library.
//
// What it computes (page "Modular TTT: Rethinking Test-Time Training as
// Composable Modules"):
//   * the fast-weight view of TTT: the hidden state is the weight W of a
//     linear map, trained online by a gradient step per token on a
//     self-supervised loss and read with queries (section "前置知识",
//     "测试时训练与快速权重");
//   * learning rate eta_t = 2*sigmoid(beta_t + b) (section "内部学习规则与
//     学习率参数化");
//   * decay of past writes (section "权重衰减"): scalar (one gamma_t per token)
//     or per feature (vector decay: gamma_t has one factor per key feature and
//     scales the matching row of W, W_s = diag(gamma_s) W_{s-1} - ...);
//   * Algorithm 1, three passes per chunk: train-view forward Vhat = act(K W0),
//     train-view backward of the inner loss (MSE or inner product), query-view
//     readout, with the chunk-start weight W0 used for every gradient in the
//     chunk and the state transition W_end = W_start - Khat^T dVhat
//     (section "方法步骤详情").
//
// It does NOT use the chunk dual form. It evolves the per-token state
// literally:
//     W_s = gamma_s * W_{s-1} - eta_s * k_s^T g_s,   g_s = dLoss/dz at z_s = k_s W0
//     o_s = act(q_s W_s)                              (readout after the token's own write)
// which, expanded, equals the dual form O = act(Gamma Q W0 - Tril(...) G).
// The readings of the pages it fixes are:
//   - Tril includes the diagonal (token s reads its own write);
//   - decay then undecayed write: W_s = gamma_s W_{s-1} - eta_s k_s^T g_s;
//   - gradients in a chunk are taken at the chunk-start W0 (C is semantic);
//   - MSE is 1/2 ||vhat - v||^2 (write signal vhat - v), IP is -<vhat, v>
//     (write signal -v), no 1/C or 1/d scaling;
//   - the query view applies the same activation: O = act(Zq).
//
// The backward is reverse-mode differentiation of the same per-token loop
// for J = <dO, O> + <dW_T, W_final>, returning dQ, dK, dV, dbeta and dW0, and
// on request the decay gradient dgamma_s = <adjoint of W_s, W_{s-1}> (per feature:
// the same inner product restricted to row i of both).
//
// Pins (tests/test_oracle_pins.py): brute-force evaluation of the chunk dual
// form printed on the page, the C = 1 delta rule and decayed Hebbian closed
// forms, chunk-size invariance of the inner-product/identity case, eta = 0,
// the affine state transition (I - K^T diag(eta) K) W0 + K^T diag(eta) V,
// streaming, column independence, hand-worked golden values and central
// finite differences for every backward output.
#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>
#ifdef _OPENMP
#include <omp.h>
#endif

namespace {

enum { LOSS_MSE = 0, LOSS_IP = 1 };
enum { ACT_ID = 0, ACT_SILU = 1 };

template <typename R> inline R sigmoid_(R x) { return R(1) / (R(1) + std::exp(-x)); }

template <typename R> inline R act_f(int act, R z) {
  return act == ACT_SILU ? z * sigmoid_(z) : z;
}
// d/dz of act
template <typename R> inline R act_d1(int act, R z) {
  if (act != ACT_SILU) return R(1);
  R s = sigmoid_(z);
  return s * (R(1) + z * (R(1) - s));
}
// d2/dz2 of act
template <typename R> inline R act_d2(int act, R z) {
  if (act != ACT_SILU) return R(0);
  R s = sigmoid_(z);
  return s * (R(1) - s) * (R(2) + z * (R(1) - R(2) * s));
}

struct Shape {
  int B, H, T, dk, dv, C, loss, act;
  double lr_bias;
  int gvec;  // gamma holds one factor per key feature: [B,H,T,dk] instead of [B,H,T]
};

// Decay of row (key feature) i of W at token t.
template <typename R, typename In>
inline R decay_at(const Shape& sh, const In* gamma, size_t t, int i) {
  if (!gamma) return R(1);
  return R(sh.gvec ? gamma[t * sh.dk + i] : gamma[t]);
}

// Train view of token t at the chunk-start weight W0: z = k W0, g = a * act'(z).
template <typename R, typename In>
inline void train_view(const Shape& sh, const In* kt, const In* vt, const R* W0, R* z, R* g) {
  const int dk = sh.dk, dv = sh.dv;
  for (int j = 0; j < dv; ++j) z[j] = R(0);
  for (int i = 0; i < dk; ++i) {
    const R ki = R(kt[i]);
    const R* wrow = W0 + (size_t)i * dv;
    for (int j = 0; j < dv; ++j) z[j] += ki * wrow[j];
  }
  for (int j = 0; j < dv; ++j) {
    const R vh = act_f(sh.act, z[j]);
    const R a = sh.loss == LOSS_MSE ? vh - R(vt[j]) : -R(vt[j]);
    g[j] = a * act_d1(sh.act, z[j]);
  }
}

template <typename R, typename In>
void fwd_head(const Shape& sh, const In* q, const In* k, const In* v, const In* beta,
              const In* gamma, const In* w_init, R* o, R* w_final, R* w_chunks) {
  const int dk = sh.dk, dv = sh.dv, C = sh.C, NC = sh.T / sh.C;
  std::vector<R> W((size_t)dk * dv), W0((size_t)dk * dv), z(dv), g(dv), zq(dv);
  for (size_t e = 0; e < W.size(); ++e) W[e] = R(w_init[e]);
  for (int c = 0; c < NC; ++c) {
    W0 = W;  // chunk-start weight: every gradient in this chunk is taken here
    if (w_chunks) std::memcpy(w_chunks + (size_t)c * dk * dv, W0.data(), sizeof(R) * W0.size());
    for (int s = 0; s < C; ++s) {
      const size_t t = (size_t)c * C + s;
      const In* kt = k + t * dk;
      const In* qt = q + t * dk;
      train_view<R, In>(sh, kt, v + t * dv, W0.data(), z.data(), g.data());
      const R eta = R(2) * sigmoid_(R(beta[t]) + R(sh.lr_bias));
      for (int i = 0; i < dk; ++i) {
        const R gam = decay_at<R, In>(sh, gamma, t, i);
        const R eki = eta * R(kt[i]);
        R* wrow = W.data() + (size_t)i * dv;
        for (int j = 0; j < dv; ++j) wrow[j] = gam * wrow[j] - eki * g[j];
      }
      for (int j = 0; j < dv; ++j) zq[j] = R(0);
      for (int i = 0; i < dk; ++i) {
        const R qi = R(qt[i]);
        const R* wrow = W.data() + (size_t)i * dv;
        for (int j = 0; j < dv; ++j) zq[j] += qi * wrow[j];
      }
      R* ot = o + t * dv;
      for (int j = 0; j < dv; ++j) ot[j] = act_f(sh.act, zq[j]);
    }
  }
  if (w_final) std::memcpy(w_final, W.data(), sizeof(R) * W.size());
}

template <typename R, typename In>
void bwd_head(const Shape& sh, const In* q, const In* k, const In* v, const In* beta,
              const In* gamma, const In* w_init, const In* dO, const In* dW_T,
              R* dq, R* dk_, R* dv_, R* dbeta, R* dw0, R* dgamma) {
  const int dk = sh.dk, dv = sh.dv, C = sh.C, NC = sh.T / sh.C;
  const size_t WS = (size_t)dk * dv;
  // with dgamma, the state before every token of the chunk being swept (W_{s-1})
  std::vector<R> Wprev(dgamma ? (size_t)C * WS : 0);
  // Forward: keep only the chunk-start weights.
  std::vector<R> Wc((size_t)NC * WS), W(WS), z(dv), g(dv);
  for (size_t e = 0; e < WS; ++e) W[e] = R(w_init[e]);
  for (int c = 0; c < NC; ++c) {
    std::memcpy(Wc.data() + (size_t)c * WS, W.data(), sizeof(R) * WS);
    const R* W0 = Wc.data() + (size_t)c * WS;
    for (int s = 0; s < C; ++s) {
      const size_t t = (size_t)c * C + s;
      train_view<R, In>(sh, k + t * dk, v + t * dv, W0, z.data(), g.data());
      const R eta = R(2) * sigmoid_(R(beta[t]) + R(sh.lr_bias));
      for (int i = 0; i < dk; ++i) {
        const R gam = decay_at<R, In>(sh, gamma, t, i);
        const R eki = eta * R(k[t * dk + i]);
        R* wrow = W.data() + (size_t)i * dv;
        for (int j = 0; j < dv; ++j) wrow[j] = gam * wrow[j] - eki * g[j];
      }
    }
  }
  // Reverse over chunks. Wh is the adjoint of the running state.
  std::vector<R> Wh(WS, R(0)), Wh0(WS), Ws(WS), Z((size_t)C * dv), G((size_t)C * dv),
      DZQ((size_t)C * dv), kW(dv), dz(dv), zq(dv);
  if (dW_T)
    for (size_t e = 0; e < WS; ++e) Wh[e] = R(dW_T[e]);
  for (int c = NC - 1; c >= 0; --c) {
    const R* W0 = Wc.data() + (size_t)c * WS;
    // Re-sweep the chunk forward: z, g, dzq and the readout part of dq.
    std::memcpy(Ws.data(), W0, sizeof(R) * WS);
    for (int s = 0; s < C; ++s) {
      const size_t t = (size_t)c * C + s;
      R* zs = Z.data() + (size_t)s * dv;
      R* gs = G.data() + (size_t)s * dv;
      train_view<R, In>(sh, k + t * dk, v + t * dv, W0, zs, gs);
      const R eta = R(2) * sigmoid_(R(beta[t]) + R(sh.lr_bias));
      if (dgamma) std::memcpy(Wprev.data() + (size_t)s * WS, Ws.data(), sizeof(R) * WS);
      for (int i = 0; i < dk; ++i) {
        const R gam = decay_at<R, In>(sh, gamma, t, i);
        const R eki = eta * R(k[t * dk + i]);
        R* wrow = Ws.data() + (size_t)i * dv;
        for (int j = 0; j < dv; ++j) wrow[j] = gam * wrow[j] - eki * gs[j];
      }
      for (int j = 0; j < dv; ++j) zq[j] = R(0);
      for (int i = 0; i < dk; ++i) {
        const R qi = R(q[t * dk + i]);
        const R* wrow = Ws.data() + (size_t)i * dv;
        for (int j = 0; j < dv; ++j) zq[j] += qi * wrow[j];
      }
      R* dzq = DZQ.data() + (size_t)s * dv;
      for (int j = 0; j < dv; ++j) dzq[j] = R(dO[t * dv + j]) * act_d1(sh.act, zq[j]);
      for (int i = 0; i < dk; ++i) {
        const R* wrow = Ws.data() + (size_t)i * dv;
        R acc = R(0);
        for (int j = 0; j < dv; ++j) acc += dzq[j] * wrow[j];
        dq[t * dk + i] = acc;
      }
    }
    // Reverse sweep over the tokens of the chunk.
    std::fill(Wh0.begin(), Wh0.end(), R(0));
    for (int s = C - 1; s >= 0; --s) {
      const size_t t = (size_t)c * C + s;
      const R* zs = Z.data() + (size_t)s * dv;
      const R* gs = G.data() + (size_t)s * dv;
      const R* dzq = DZQ.data() + (size_t)s * dv;
      const R eta = R(2) * sigmoid_(R(beta[t]) + R(sh.lr_bias));
      // readout o_s = act(q_s W_s) adds to the adjoint of W_s
      for (int i = 0; i < dk; ++i) {
        const R qi = R(q[t * dk + i]);
        R* whrow = Wh.data() + (size_t)i * dv;
        for (int j = 0; j < dv; ++j) whrow[j] += qi * dzq[j];
      }
      // W_s = gam W_{s-1} - eta k_s^T g_s
      for (int j = 0; j < dv; ++j) kW[j] = R(0);
      for (int i = 0; i < dk; ++i) {
        const R ki = R(k[t * dk + i]);
        const R* whrow = Wh.data() + (size_t)i * dv;
        R acc = R(0);
        for (int j = 0; j < dv; ++j) {
          kW[j] += ki * whrow[j];
          acc += gs[j] * whrow[j];
        }
        dk_[t * dk + i] = -eta * acc;
      }
      R deta = R(0);
      for (int j = 0; j < dv; ++j) deta -= kW[j] * gs[j];
      // W_s = diag(gam) W_{s-1} - ...: dJ/dgam_i = <row i of the adjoint of W_s, row i of
      // W_{s-1}>, summed over the rows for a scalar decay
      if (dgamma) {
        const R* wp = Wprev.data() + (size_t)s * WS;
        R tot = R(0);
        for (int i = 0; i < dk; ++i) {
          R acc = R(0);
          for (int j = 0; j < dv; ++j) acc += Wh[(size_t)i * dv + j] * wp[(size_t)i * dv + j];
          if (sh.gvec) dgamma[t * dk + i] = acc;
          tot += acc;
        }
        if (!sh.gvec) dgamma[t] = tot;
      }
      for (int i = 0; i < dk; ++i) {
        const R gam = decay_at<R, In>(sh, gamma, t, i);
        for (int j = 0; j < dv; ++j) Wh[(size_t)i * dv + j] *= gam;
      }
      // g = a * act'(z),  a = act(z) - v (MSE) or -v (IP),  z = k W0
      for (int j = 0; j < dv; ++j) {
        const R dg = -eta * kW[j];
        const R d1 = act_d1(sh.act, zs[j]);
        const R a = sh.loss == LOSS_MSE ? act_f(sh.act, zs[j]) - R(v[t * dv + j]) : -R(v[t * dv + j]);
        const R da = dg * d1;
        dz[j] = dg * a * act_d2(sh.act, zs[j]) + (sh.loss == LOSS_MSE ? da * d1 : R(0));
        dv_[t * dv + j] = -da;
      }
      for (int i = 0; i < dk; ++i) {
        const R* w0row = W0 + (size_t)i * dv;
        const R ki = R(k[t * dk + i]);
        R* wh0row = Wh0.data() + (size_t)i * dv;
        R acc = R(0);
        for (int j = 0; j < dv; ++j) {
          acc += dz[j] * w0row[j];
          wh0row[j] += ki * dz[j];
        }
        dk_[t * dk + i] += acc;
      }
      dbeta[t] = deta * eta * (R(1) - eta / R(2));
    }
    for (size_t e = 0; e < WS; ++e) Wh[e] += Wh0[e];
  }
  std::memcpy(dw0, Wh.data(), sizeof(R) * WS);
}

int set_threads(int nthreads) {
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
  return omp_get_max_threads();
#else
  (void)nthreads;
  return 1;
#endif
}

template <typename R, typename In>
int fwd_all(const Shape& sh, const In* Q, const In* K, const In* V, const In* beta, const In* gamma,
            const In* W0, R* O, R* Wf, R* Wc, int nthreads) {
  const int used = set_threads(nthreads);
  const int BH = sh.B * sh.H, NC = sh.T / sh.C;
  const size_t tk = (size_t)sh.T * sh.dk, tv = (size_t)sh.T * sh.dv, ws = (size_t)sh.dk * sh.dv;
#pragma omp parallel for schedule(dynamic, 1)
  for (int bh = 0; bh < BH; ++bh) {
    fwd_head<R, In>(sh, Q + bh * tk, K + bh * tk, V + bh * tv, beta + (size_t)bh * sh.T,
                    gamma ? gamma + (size_t)bh * sh.T * (sh.gvec ? sh.dk : 1) : nullptr,
                    W0 + bh * ws, O + bh * tv,
                    Wf ? Wf + bh * ws : nullptr, Wc ? Wc + (size_t)bh * NC * ws : nullptr);
  }
  return used;
}

}  // namespace

extern "C" {

// Forward, fp64 state and arithmetic. Q,K [B,H,T,dk]; V,O [B,H,T,dv]; beta [B,H,T]; gamma
// [B,H,T], or [B,H,T,dk] with gamma_per_feature set (gamma may be NULL: no decay); W0, W_final
// [B,H,dk,dv]; W_chunks [B,H,T/C,dk,dv] or NULL.
// Returns the number of threads used, or -1 on a bad shape.
int ttt_oracle_fwd_f64(int B, int H, int T, int dk, int dv, int C, int loss, int act, double lr_bias,
                       int gamma_per_feature, const double* Q, const double* K, const double* V, const double* beta,
                       const double* gamma, const double* W0, double* O, double* W_final,
                       double* W_chunks, int nthreads) {
  if (B <= 0 || H <= 0 || T <= 0 || dk <= 0 || dv <= 0 || C <= 0 || T % C) return -1;
  Shape sh{B, H, T, dk, dv, C, loss, act, lr_bias, gamma_per_feature != 0};
  return fwd_all<double, double>(sh, Q, K, V, beta, gamma, W0, O, W_final, W_chunks, nthreads);
}

// Forward with an fp32 state and fp32 arithmetic (the per-token fp32 state evolver; used as the
// timed CPU baseline). Same layouts as above with float buffers.
int ttt_oracle_fwd_f32(int B, int H, int T, int dk, int dv, int C, int loss, int act, double lr_bias,
                       int gamma_per_feature, const float* Q, const float* K, const float* V, const float* beta,
                       const float* gamma, const float* W0, float* O, float* W_final,
                       float* W_chunks, int nthreads) {
  if (B <= 0 || H <= 0 || T <= 0 || dk <= 0 || dv <= 0 || C <= 0 || T % C) return -1;
  Shape sh{B, H, T, dk, dv, C, loss, act, lr_bias, gamma_per_feature != 0};
  return fwd_all<float, float>(sh, Q, K, V, beta, gamma, W0, O, W_final, W_chunks, nthreads);
}

// Backward, fp64: reverse-mode of the per-token loop for J = <dO, O> + <dW_T, W_final>.
// dW_T may be NULL (zero). Outputs dQ,dK [B,H,T,dk], dV [B,H,T,dv], dbeta [B,H,T], dW0 [B,H,dk,dv],
// and dgamma (the shape of gamma) when both gamma and dgamma are non-NULL.
int ttt_oracle_bwd_f64(int B, int H, int T, int dk, int dv, int C, int loss, int act, double lr_bias,
                       int gamma_per_feature, const double* Q, const double* K, const double* V, const double* beta,
                       const double* gamma, const double* W0, const double* dO, const double* dW_T,
                       double* dQ, double* dK, double* dV, double* dbeta, double* dW0,
                       double* dgamma, int nthreads) {
  if (B <= 0 || H <= 0 || T <= 0 || dk <= 0 || dv <= 0 || C <= 0 || T % C) return -1;
  Shape sh{B, H, T, dk, dv, C, loss, act, lr_bias, gamma_per_feature != 0};
  const int used = set_threads(nthreads);
  const int BH = B * H;
  const size_t tk = (size_t)T * dk, tv = (size_t)T * dv, ws = (size_t)dk * dv;
  const size_t tg = (size_t)T * (gamma_per_feature ? dk : 1);
#pragma omp parallel for schedule(dynamic, 1)
  for (int bh = 0; bh < BH; ++bh) {
    bwd_head<double, double>(sh, Q + bh * tk, K + bh * tk, V + bh * tv, beta + (size_t)bh * T,
                             gamma ? gamma + bh * tg : nullptr, W0 + bh * ws, dO + bh * tv,
                             dW_T ? dW_T + bh * ws : nullptr, dQ + bh * tk, dK + bh * tk,
                             dV + bh * tv, dbeta + (size_t)bh * T, dW0 + bh * ws,
                             gamma && dgamma ? dgamma + bh * tg : nullptr);
  }
  return used;
}

}  // extern "C"
