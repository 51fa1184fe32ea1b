// tcgen05 forward of the chunkwise TTT layer (bf16 operands, fp32 state and accumulators).
//
// Page "Modular TTT: Rethinking Test-Time Training as Composable Modules", section
// "方法步骤详情" (Algorithm 1) with the lr of section "内部学习规则与学习率参数化" and the
// scalar decay of section "权重衰减". Per chunk of C tokens, with W0 the chunk-start state:
//   Z   = K W0                          (train view, one MMA per 128-token block)
//   G   = a(Z) * act'(Z)                (inner-loss gradient; MSE a = act(Z) - V, IP a = -V)
//   Zq  = diag(Gamma) Q W0 - S G,  S_sr = eta_r exp(L_s - L_r) (q_s . k_r) for r <= s
//   O   = act(Zq)
//   W   = Gamma_C W0 - K^T diag(u) G,  u_r = eta_r exp(L_C - L_r)
//
// One CTA owns one (batch, head, 64-wide slice of d_v): the columns of W, V, G, Z, Zq and O
// evolve independently, so d_v = 128 runs as two CTAs per head. The fp32 state lives in TMEM
// for the whole sequence; a bf16 copy in shared memory is the MMA operand of the next chunk.
//
// Warp roles: warp 0 TMA producer; warp 1 issues the state-chain MMAs (Z = K W0 and the
// transition) and owns TMEM; warp 11 issues the query-side MMAs (Y = Q W0, the score blocks and
// S G), so the next chunk's Z never waits behind this chunk's score work; warps 2-9 epilogue
// (two warpgroups; warpgroup g handles value columns [32g, 32g+32) of each 128-row block and
// score columns [64g, 64g+64) of each 128x128 score block); warp 10 computes the lr and decay
// scans of the next chunk into the other of two buffers. Every wait is bounded.
//
// TMEM columns: [0,64) W (lanes = key features; held pre-multiplied by the chunk's Gamma_C),
// [64, 64+64NB) Z blocks, [64+64NB, 64+128NB) Y / Zq blocks, [64+128NB, +128) score buffer A.
// With two 128-token blocks per chunk the Z columns double as score buffer B once G has been
// formed, so the next score block's MMA runs while the epilogue masks the current one. The
// epilogue writes S (bf16) in place over the fp32 scores it read; the S G MMA takes S straight
// from TMEM.
// Shared memory: K as two 128-row halves with their own full/free barriers, V double-buffered,
// so the next chunk's loads start as soon as each buffer's last reader has finished.
#include <cuda_bf16.h>
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "tc_util.cuh"

namespace tttk {
namespace {

constexpr int NV = 64;             // value columns per CTA
constexpr int kThreads = 384;      // 12 warps
constexpr int kEpiWarps = 8;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t PANEL128 = 128 * 128;  // 128 rows x 128 bytes

struct FwdParams {
  int BH, T, NC, nslice;
  float lr_bias;
  const float* beta;
  const float* gamma;     // nullable
  const float* W0;        // [BH, D, D] fp32 (or [H, D, D]: block bh % w0_mod)
  int w0_mod;
  __nv_bfloat16* O;       // [BH, T, D]
  float* W_final;         // nullable
  __nv_bfloat16* W_chunks;  // nullable, [BH, NC, D, D]
  int save_g;               // store G of every token (bulk stores through tmG)
  __nv_bfloat16* Zq;        // nullable, [BH, T, D]: the SiLU readout before the activation
  unsigned* err;
};

template <int D, int NB>
struct Layout {
  static constexpr int C = 128 * NB;
  static constexpr int KP = D / 64;                      // 64-wide key-feature panels
  static constexpr uint32_t KH = KP * PANEL128;          // one 128-row half of K (or of Q)
  static constexpr uint32_t OFF_K = 0;                   // K half b, panel p at OFF_K + (b KP + p) PANEL128
  static constexpr uint32_t OFF_Q = OFF_K + NB * KH;     // Q half h at OFF_Q + h KH
  // two rotating buffers: chunk c's V (then G, in place) in buffer c & 1 and its -u G in the
  // other one, which then receives V of chunk c + 1 once the transition MMA has read -u G
  static constexpr uint32_t OFF_VG = OFF_Q + NB * KH;
  static constexpr uint32_t OFF_W0 = OFF_VG + 2 * C * 128;  // bf16 state, MN-major [D][64]
  static constexpr uint32_t OFF_F = OFF_W0 + D * 128;       // scan arrays, 2 buffers x 6 x 256
  static constexpr uint32_t OFF_BG = OFF_F + 2 * 6 * 256 * 4;  // beta, gamma of 2 chunks
  static constexpr uint32_t OFF_BAR = OFF_BG + 4 * C * 4;
  static constexpr uint32_t BYTES = OFF_BAR + 512;
  static constexpr uint32_t V_TX = C * 128;
  // TMEM columns
  static constexpr uint32_t T_W = 0, T_Z = 64, T_Y = 64 + 64 * NB, T_PA = 64 + 128 * NB;
  // score buffer x: A (x = 0) its own 128 columns, B (x = 1) the Z columns once G is formed
  __host__ __device__ static constexpr uint32_t tbuf(int x) { return x ? T_Z : T_PA; }
};

struct __align__(8) FwdBars {
  uint64_t k_full[2], k_free[2], q_full[2], q_free[2], v_full[2], z_full, g_ready, y_full[2],
      y_scaled[2], p_full[2], s_ready[2], s_done[2], zq_full[2], y_free[2], w_full, w0_ready,
      g_done, scan_full[2], scan_free[2], bg_full[2], st_free, g_read[2], z_issued, t_issued;
  uint32_t tmem_base;
  int abort_flag;
};

template <int D, int NB, int ACT, int LOSS>
__global__ void __launch_bounds__(kThreads, 1)
    ttt_fwd_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmQ,
                      const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmWc,
                      const __grid_constant__ CUtensorMap tmG, const FwdParams p) {
  using L = Layout<D, NB>;
  constexpr int C = L::C;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sK = sbase + L::OFF_K, sQ = sbase + L::OFF_Q, sVG = sbase + L::OFF_VG,
                 sW0 = sbase + L::OFF_W0;
  // scan arrays of buffer i: eta, L (chunk-local log decay), Gamma = exp(L), exp(L_C - L),
  // cF16 = eta exp(L_{r16} - L), cT16 = exp(L - L_{r16})
  float* f_scan = reinterpret_cast<float*>(smem + L::OFF_F);
  float* f_bg = reinterpret_cast<float*>(smem + L::OFF_BG);   // [parity][beta, gamma][C]
  FwdBars* bars = reinterpret_cast<FwdBars*>(smem + L::OFF_BAR);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int bh = blockIdx.x / p.nslice, slice = blockIdx.x % p.nslice;
  Abort ab{&bars->abort_flag, p.err};
#define BAR(x) smem_u32(&bars->x)

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(BAR(k_full[i]), 1);
      mbar_init(BAR(k_free[i]), 2);  // both MMA issuers read K
      mbar_init(BAR(q_full[i]), 1);
      mbar_init(BAR(q_free[i]), 1);
      mbar_init(BAR(v_full[i]), 1);
      mbar_init(BAR(y_full[i]), 1);
      mbar_init(BAR(y_scaled[i]), kEpiWarps);
      mbar_init(BAR(p_full[i]), 1);
      mbar_init(BAR(s_ready[i]), kEpiWarps);
      mbar_init(BAR(s_done[i]), 1);
      mbar_init(BAR(zq_full[i]), 1);
      mbar_init(BAR(y_free[i]), kEpiWarps);
      mbar_init(BAR(scan_full[i]), 1);
      mbar_init(BAR(scan_free[i]), kEpiWarps);
      mbar_init(BAR(bg_full[i]), 1);
      mbar_init(BAR(g_read[i]), 1);
    }
    mbar_init(BAR(z_full), 1);
    mbar_init(BAR(g_ready), kEpiWarps);
    mbar_init(BAR(w_full), 1);
    mbar_init(BAR(w0_ready), kEpiWarps);
    mbar_init(BAR(g_done), 1);
    mbar_init(BAR(st_free), 1);
    mbar_init(BAR(z_issued), 1);
    mbar_init(BAR(t_issued), 1);
    bars->abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmV);
  }
  if (warp == 1) {
    tmem_alloc(BAR(tmem_base), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  const int NC = p.NC;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      // beta, gamma of chunk c go to buffer c & 1 on bg_full[c & 1] (phase (c >> 1) & 1),
      // one chunk ahead of the scan that reads them
      auto load_bg = [&](int cc) {
        const uint32_t bg = smem_u32(f_bg + (cc & 1) * 2 * C);
        const uint32_t bar = BAR(bg_full[cc & 1]);
        const size_t r0 = (size_t)bh * p.T + (size_t)cc * C;
        mbar_arrive_expect_tx(bar, (p.gamma ? 2 : 1) * C * 4);
        bulk_g2s(bg, p.beta + r0, C * 4, bar);
        if (p.gamma) bulk_g2s(bg + C * 4, p.gamma + r0, C * 4, bar);
      };
      load_bg(0);
      mbar_arrive_expect_tx(BAR(v_full[0]), L::V_TX);
      tma_load_2d(sVG, &tmV, BAR(v_full[0]), NV * slice, bh * p.T);
      for (int c = 0; c < NC; ++c) {
        const int row0 = bh * p.T + c * C;
        // K halves of chunk c, each free once its last reader of chunk c-1 is done
        for (int h = 0; h < NB; ++h) {
          if (c > 0 && !mbar_wait(BAR(k_free[h]), (c - 1) & 1, ab)) goto done_prod;
          mbar_arrive_expect_tx(BAR(k_full[h]), L::KH);
#pragma unroll
          for (int kp = 0; kp < L::KP; ++kp)
            tma_load_2d(sK + (h * L::KP + kp) * PANEL128, &tmK, BAR(k_full[h]), 64 * kp,
                        row0 + 128 * h);
        }
        // both Q halves of chunk c
        for (int h = 0; h < NB; ++h) {
          if (c > 0 && !mbar_wait(BAR(q_free[h]), (c - 1) & 1, ab)) goto done_prod;
          mbar_arrive_expect_tx(BAR(q_full[h]), L::KH);
#pragma unroll
          for (int kp = 0; kp < L::KP; ++kp)
            tma_load_2d(sQ + (h * L::KP + kp) * PANEL128, &tmQ, BAR(q_full[h]), 64 * kp,
                        row0 + 128 * h);
        }
        if (c + 1 < NC) {
          // buffer (c+1)&1 of beta/gamma was last read by the scan of chunk c-1
          if (c > 0 && !mbar_wait(BAR(scan_full[(c - 1) & 1]), ((c - 1) >> 1) & 1, ab))
            goto done_prod;
          load_bg(c + 1);
          // V of chunk c+1 into the buffer holding chunk c's -u G, once the transition MMA has
          // read it (and, with G saved, once the bulk store of chunk c-1's G there has read it)
          const int vb = (c + 1) & 1;
          if (!mbar_wait(BAR(w_full), c & 1, ab)) goto done_prod;
          if (c >= 1 && p.save_g && !mbar_wait(BAR(g_read[vb]), ((c - 1) >> 1) & 1, ab))
            goto done_prod;
          mbar_arrive_expect_tx(BAR(v_full[vb]), L::V_TX);
          tma_load_2d(sVG + vb * C * 128, &tmV, BAR(v_full[vb]), NV * slice, row0 + C);
        }
      }
    done_prod:;
    }
  } else if (warp == 1) {
    // ------------------------------------------------------ state-chain MMAs: Z, transition
    if (lane == 0) {
      const uint32_t idZ = idesc_bf16(128, NV, 0, 1);   // K-major A, MN-major B
      const uint32_t idW = idesc_bf16(128, NV, 1, 1);   // MN-major A and B
      const uint32_t lboKt = D == 128 ? PANEL128 : 0;  // second 64-row block of K^T
      for (int c = 0; c < NC; ++c) {
        const uint32_t sUG = sVG + ((c + 1) & 1) * C * 128;
        bool ok = mbar_wait(BAR(w0_ready), c & 1, ab);
        for (int b = 0; b < NB && ok; ++b) ok = mbar_wait(BAR(k_full[b]), c & 1, ab);
        // with two blocks the Z columns are score buffer B, read last by S_00 G_0 of chunk c-1
        if (ok && NB == 2 && c > 0) ok = mbar_wait(BAR(s_done[1]), (c - 1) & 1, ab);
        if (!ok) break;
        tc_fence_after();
        // Z_b = K_b W0
        for (int b = 0; b < NB; ++b) {
#pragma unroll
          for (int j = 0; j < D / 16; ++j)
            mma_bf16_ss(tmem + L::T_Z + NV * b,
                        sdesc_sw128(sK + (b * L::KP + j / 4) * PANEL128 + (j % 4) * 32, 16, 1024),
                        sdesc_sw128(sW0 + j * 2048, 0, 1024), idZ, j > 0);
        }
        mma_commit(BAR(z_full));
        // the query side issues this chunk's Y only now, so Z is first in the tensor pipe
        mbar_arrive(BAR(z_issued));
        if (!mbar_wait(BAR(g_ready), c & 1, ab)) break;
        tc_fence_after();
        // W += K^T (u * -G), W already scaled by Gamma_C
        for (int j = 0; j < C / 16; ++j)
          mma_bf16_ss(tmem + L::T_W, sdesc_sw128(sK + (j / 8) * L::KH + (j % 8) * 2048, lboKt, 1024),
                      sdesc_sw128(sUG + j * 2048, 0, 1024), idW, 1);
        mma_commit(BAR(w_full));
        for (int b = 0; b < NB; ++b) mma_commit(BAR(k_free[b]));
        mbar_arrive(BAR(t_issued));
      }
    }
  } else if (warp == 11) {
    // ------------------------------------------------- query-side MMAs: Y, scores, S G
    // Score blocks of a chunk: with two query halves (1,0) goes to buffer A first, (0,0) to B
    // (the Z columns) once G is formed, (1,1) to A once S_10 G_0 has read it; so the Z columns
    // are free for the next chunk as soon as S_00 G_0 is done. With one half, (0,0) uses A.
    if (lane == 0) {
      const uint32_t idZ = idesc_bf16(128, NV, 0, 1);   // K-major A, MN-major B
      const uint32_t idP = idesc_bf16(128, 128, 0, 0);  // K-major A and B
      int sdA = 0, srA = 0;                             // buffer A: S G commits, s_ready phases
      auto issue_y = [&](int h) {
#pragma unroll
        for (int j = 0; j < D / 16; ++j)
          mma_bf16_ss(tmem + L::T_Y + NV * h,
                      sdesc_sw128(sQ + (h * L::KP + j / 4) * PANEL128 + (j % 4) * 32, 16, 1024),
                      sdesc_sw128(sW0 + j * 2048, 0, 1024), idZ, j > 0);
        mma_commit(BAR(y_full[h]));
      };
      auto issue_p = [&](int h, int b, int x) {
#pragma unroll
        for (int j = 0; j < D / 16; ++j)
          mma_bf16_ss(tmem + L::tbuf(x),
                      sdesc_sw128(sQ + (h * L::KP + j / 4) * PANEL128 + (j % 4) * 32, 16, 1024),
                      sdesc_sw128(sK + (b * L::KP + j / 4) * PANEL128 + (j % 4) * 32, 16, 1024),
                      idP, j > 0);
        mma_commit(BAR(p_full[x]));
      };
      auto wait_a_free = [&]() -> bool {
        return sdA == 0 || mbar_wait(BAR(s_done[0]), (sdA - 1) & 1, ab);
      };
      // Zq_h += (-S_hb) G_b; S (bf16) in TMEM, 32 packed columns per warpgroup
      auto issue_sg = [&](int h, int b, int x, uint32_t sG, int ready_phase) -> bool {
        if (!mbar_wait(BAR(s_ready[x]), ready_phase & 1, ab)) return false;
        tc_fence_after();
#pragma unroll
        for (int j = 0; j < 8; ++j)
          mma_bf16_ts(tmem + L::T_Y + NV * h, tmem + L::tbuf(x) + packed_col<64>(j),
                      sdesc_sw128(sG + b * PANEL128 + j * 2048, 0, 1024), idZ, 1);
        mma_commit(BAR(s_done[x]));
        if (x == 0) ++sdA;
        return true;
      };
      for (int c = 0; c < NC; ++c) {
        const uint32_t sG = sVG + (c & 1) * C * 128;
        // Y_h = Q_h W0 with this chunk's bf16 state copy, behind Z in the tensor pipe
        bool ok = mbar_wait(BAR(w0_ready), c & 1, ab) && mbar_wait(BAR(z_issued), c & 1, ab);
        for (int h = 0; h < NB && ok; ++h) {
          ok = mbar_wait(BAR(q_full[h]), c & 1, ab) &&
               (c == 0 || mbar_wait(BAR(y_free[h]), (c - 1) & 1, ab));
          if (ok) {
            tc_fence_after();
            issue_y(h);
          }
        }
        for (int b = 0; b < NB && ok; ++b) ok = mbar_wait(BAR(k_full[b]), c & 1, ab);
        if (!ok || !wait_a_free()) break;
        tc_fence_after();
        if constexpr (NB == 1) {
          issue_p(0, 0, 0);
          mma_commit(BAR(q_free[0]));
          mma_commit(BAR(k_free[0]));
          if (!mbar_wait(BAR(y_scaled[0]), c & 1, ab) || !issue_sg(0, 0, 0, sG, srA++)) break;
          mma_commit(BAR(zq_full[0]));
        } else {
          issue_p(1, 0, 0);                                    // (1,0) -> A
          // the Z columns are free once G is formed; waiting for the transition's issue as
          // well keeps the state chain ahead of this block in the tensor pipe
          if (!mbar_wait(BAR(t_issued), c & 1, ab)) break;
          tc_fence_after();
          issue_p(0, 0, 1);                                    // (0,0) -> B
          mma_commit(BAR(q_free[0]));
          mma_commit(BAR(k_free[0]));
          if (!mbar_wait(BAR(y_scaled[1]), c & 1, ab) || !issue_sg(1, 0, 0, sG, srA++)) break;
          if (!wait_a_free()) break;
          tc_fence_after();
          issue_p(1, 1, 0);                                    // (1,1) -> A
          mma_commit(BAR(q_free[1]));
          mma_commit(BAR(k_free[1]));
          if (!mbar_wait(BAR(y_scaled[0]), c & 1, ab) || !issue_sg(0, 0, 1, sG, c)) break;
          mma_commit(BAR(zq_full[0]));
          if (!issue_sg(1, 1, 0, sG, srA++)) break;
          mma_commit(BAR(zq_full[1]));
        }
        mma_commit(BAR(g_done));  // G of chunk c (in its V buffer) fully read
      }
    }
  } else if (warp == 10) {
    // ------------------------------------------------------------------ scans, one chunk ahead
    for (int c = 0; c < NC; ++c) {
      const int sb = c & 1;
      if (c >= 2 && !mbar_wait(BAR(scan_free[sb]), ((c - 2) >> 1) & 1, ab)) break;
      if (!mbar_wait(BAR(bg_full[sb]), (c >> 1) & 1, ab)) break;
      const float* bg = f_bg + sb * 2 * C;
      float* fs = f_scan + sb * 6 * 256;
      chunk_scan_warp<C>(bg, p.gamma ? bg + C : nullptr, p.lr_bias, fs, fs + 256, fs + 512,
                         fs + 768, fs + 1024, fs + 1280);
      if (lane == 0) mbar_arrive(BAR(scan_full[sb]));
    }
  } else {
    // ------------------------------------------------------------------ epilogue
    const int ew = warp - 2;          // 0..7
    const int g = ew / 4;             // warpgroup: value columns [32g, 32g+32)
    const int q = warp & 3;           // TMEM lane quadrant
    const int lrow = q * 32 + lane;   // TMEM lane = row inside a 128-row block
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    const bool w_rows = q * 32 < D;   // this warp holds state rows
    // this thread's 32 state entries: in W_final (per sequence) and in W0 (maybe shared)
    const size_t wofs = (size_t)bh * D * D + (size_t)lrow * D + NV * slice + 32 * g;
    const size_t w0ofs = (size_t)(bh % p.w0_mod) * D * D + (size_t)lrow * D + NV * slice + 32 * g;
    bool ok = true;
    // initial state: Gamma_C(0) W0 into TMEM, bf16 operand copy, chunk-0 checkpoint
    if (!mbar_wait(BAR(scan_full[0]), 0, ab)) ok = false;
    if (ok && w_rows) {
      float w[32];
      const float4* src = reinterpret_cast<const float4*>(p.W0 + w0ofs);
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const float4 v = src[k];
        w[4 * k] = v.x; w[4 * k + 1] = v.y; w[4 * k + 2] = v.z; w[4 * k + 3] = v.w;
      }
      st_row32(sW0, lrow, 4 * g, w);
      if (p.W_chunks)
        st_global_bf16x32(p.W_chunks + (size_t)bh * NC * D * D + (size_t)lrow * D + NV * slice + 32 * g, w);
      const float gam0 = f_scan[512 + C - 1];
#pragma unroll
      for (int j = 0; j < 32; ++j) w[j] *= gam0;
      tmem_st32(tmem + lane_off + L::T_W + 32 * g, w);
      tmem_wait_st();
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(BAR(w0_ready));

    int puse0 = 0, puse1 = 0;  // score blocks consumed per buffer
    for (int c = 0; c < NC && ok; ++c) {
      const size_t tok0 = (size_t)bh * p.T + (size_t)c * C;
      const uint32_t sG = sVG + (c & 1) * C * 128, sUG = sVG + ((c + 1) & 1) * C * 128;
      // -------- this chunk's scan arrays (computed by warp 10)
      if (!mbar_wait(BAR(scan_full[c & 1]), (c >> 1) & 1, ab)) { ok = false; break; }
      const float* f_eta = f_scan + (c & 1) * 6 * 256;
      const float* f_L = f_eta + 256;
      const float* f_gam = f_eta + 512;
      const float* f_eLC = f_eta + 768;
      const float* f_cF16 = f_eta + 1024;

      // -------- train view: G = a(Z) act'(Z) in place over V, -u G into the other buffer
      if (ew == 0 && c > 0) {
        // the previous chunk's bulk stores (the state checkpoint from the bf16 state copy, G)
        // must have read their sources before those are rewritten
        if (lane == 0) {
          bulk_wait_read0();
          mbar_arrive(BAR(st_free));
          mbar_arrive(BAR(g_read[(c - 1) & 1]));
        }
        __syncwarp();
      }
      if (c > 0 && !mbar_wait(BAR(st_free), (c - 1) & 1, ab)) { ok = false; break; }
      // -u G goes over chunk c-1's G, which its last S G MMA must have read
      if (c > 0 && !mbar_wait(BAR(g_done), (c - 1) & 1, ab)) { ok = false; break; }
      if (!mbar_wait(BAR(v_full[c & 1]), (c >> 1) & 1, ab)) { ok = false; break; }
      if (!mbar_wait(BAR(z_full), c & 1, ab)) { ok = false; break; }
      __syncwarp();
      tc_fence_after();
      {
        // both Z blocks in flight at once
        constexpr int ZB = NB;
        float z[ZB][32];
#pragma unroll
        for (int b0 = 0; b0 < NB; b0 += ZB) {
#pragma unroll
          for (int i = 0; i < ZB; ++i)
            tmem_ld32(tmem + lane_off + L::T_Z + NV * (b0 + i) + 32 * g, z[i]);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < ZB; ++i) {
            float v[32];
            const int row = 128 * (b0 + i) + lrow;
            ld_row32(sG, row, 4 * g, v);
            const float un = -f_eta[row] * f_eLC[row];
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              float fz, d1;
              act_both<ACT>(z[i][j], fz, d1);
              const float a = LOSS == 0 ? fz - v[j] : -v[j];
              const float gg = a * d1;
              v[j] = gg;
              z[i][j] = un * gg;
            }
            st_row32(sG, row, 4 * g, v);
            st_row32(sUG, row, 4 * g, z[i]);
          }
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(g_ready));
      if (ew == 0 && p.save_g) {
        // G of the chunk's tokens, one bulk store per 128-row block of this value slice
        if (lane == 0) {
          ok = mbar_wait(BAR(g_ready), c & 1, ab);
          if (ok) {
            for (int b = 0; b < NB; ++b)
              tma_store_2d(&tmG, sG + b * PANEL128, NV * slice, (int)tok0 + 128 * b);
            bulk_commit();
          }
        }
        if (!__shfl_sync(0xffffffffu, (int)ok, 0)) { ok = false; break; }
      }

      // -------- Y_h *= Gamma_s for both query halves (while the transition MMA runs)
      for (int h = 0; h < NB; ++h) {
        if (!mbar_wait(BAR(y_full[h]), c & 1, ab)) { ok = false; break; }
        __syncwarp();
        tc_fence_after();
        float y[32];
        tmem_ld32(tmem + lane_off + L::T_Y + NV * h + 32 * g, y);
        tmem_wait_ld();
        const float gs = f_gam[128 * h + lrow];
#pragma unroll
        for (int j = 0; j < 32; ++j) y[j] *= gs;
        tmem_st32(tmem + lane_off + L::T_Y + NV * h + 32 * g, y);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(BAR(y_scaled[h]));
      }
      if (!ok) break;
      // -------- state copy for the next chunk: after the transition MMA and after the last MMA
      // that reads the current bf16 copy (Y of the last query half). The fp32 state goes back
      // into TMEM already decayed by the next chunk's Gamma_C.
      {
        const bool more = c + 1 < NC;
        if (!mbar_wait(BAR(w_full), c & 1, ab) || !mbar_wait(BAR(y_full[NB - 1]), c & 1, ab) ||
            (more && !mbar_wait(BAR(scan_full[(c + 1) & 1]), ((c + 1) >> 1) & 1, ab))) {
          ok = false;
          break;
        }
        __syncwarp();
        tc_fence_after();
        if (w_rows) {
          float w[32];
          tmem_ld32(tmem + lane_off + L::T_W + 32 * g, w);
          tmem_wait_ld();
          if (more) {
            st_row32(sW0, lrow, 4 * g, w);
            const float gnext = f_scan[((c + 1) & 1) * 6 * 256 + 512 + C - 1];
#pragma unroll
            for (int j = 0; j < 32; ++j) w[j] *= gnext;
            tmem_st32(tmem + lane_off + L::T_W + 32 * g, w);
            tmem_wait_st();
          } else if (p.W_final) {
            float4* dst = reinterpret_cast<float4*>(p.W_final + wofs);
#pragma unroll
            for (int k = 0; k < 8; ++k)
              dst[k] = make_float4(w[4 * k], w[4 * k + 1], w[4 * k + 2], w[4 * k + 3]);
          }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(BAR(w0_ready));
        if (ew == 0 && more && p.W_chunks) {
          // checkpoint of the next chunk's start state, one bulk store of the bf16 copy
          if (lane == 0) {
            ok = mbar_wait(BAR(w0_ready), (c + 1) & 1, ab);
            if (ok) {
              tma_store_2d(&tmWc, sW0, NV * slice, (bh * NC + c + 1) * D);
              bulk_commit();
            }
          }
          if (!__shfl_sync(0xffffffffu, (int)ok, 0)) { ok = false; break; }
        }
      }

      // -------- score blocks S = -(Q K^T) * weights, bf16 in place, in the order the query-side
      // issuer produces them: (1,0) in A, (0,0) in B, (1,1) in A; or (0,0) in A
      for (int k = 0; k < (NB == 2 ? 3 : 1); ++k) {
        const int h = NB == 2 ? (k == 1 ? 0 : 1) : 0, b = NB == 2 ? (k == 2 ? 1 : 0) : 0;
        const int x = (NB == 2 && k == 1) ? 1 : 0;
        const int pu = x ? puse1++ : puse0++;
        if (!mbar_wait(BAR(p_full[x]), pu & 1, ab)) { ok = false; break; }
        __syncwarp();
        tc_fence_after();
        const int srow = 128 * h + lrow;
        const QWeights w{f_L, f_cF16, srow, 128 * b, f_L[srow]};
        pack_in_place<64>(tmem + lane_off + L::tbuf(x), g, g + 1, q, b == h, w);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(BAR(s_ready[x]));
      }
      if (!ok) break;
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(scan_free[c & 1]));
      // -------- O_h = act(Zq_h), straight from registers to global memory
      for (int h = 0; h < NB; ++h) {
        if (!mbar_wait(BAR(zq_full[h]), c & 1, ab)) { ok = false; break; }
        __syncwarp();
        tc_fence_after();
        float o[32];
        tmem_ld32(tmem + lane_off + L::T_Y + NV * h + 32 * g, o);
        tmem_wait_ld();
        if (ACT == 1 && p.Zq)
          st_global_bf16x32(p.Zq + (tok0 + 128 * h + lrow) * D + NV * slice + 32 * g, o);
#pragma unroll
        for (int j = 0; j < 32; ++j) o[j] = act_f<ACT>(o[j]);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(BAR(y_free[h]));
        st_global_bf16x32(p.O + (tok0 + 128 * h + lrow) * D + NV * slice + 32 * g, o);
      }
    }
    if (ew == 0 && lane == 0) bulk_wait0();
  }
#undef BAR
  tc_fence_before();
  __syncthreads();
  if (bars->abort_flag) __nanosleep(100000);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int D, int NB, int ACT, int LOSS>
cudaError_t launch(const LayerArgs& a, cudaStream_t s) {
  using L = Layout<D, NB>;
  const uint64_t rows = (uint64_t)a.B * a.H * a.T;
  CUtensorMap tk, tq, tv, twc, tg;
  const uint64_t wrows = (uint64_t)a.B * a.H * (a.T / a.C) * D;
  if (!make_tmap_bf16(&tk, a.K, D, rows, D, 64, 128) ||
      !make_tmap_bf16(&tq, a.Q, D, rows, D, 64, 128) ||
      !make_tmap_bf16(&tv, a.V, D, rows, D, 64, L::C) ||
      (a.W_chunks && !make_tmap_bf16(&twc, a.W_chunks, D, wrows, D, 64, D)) ||
      (a.G_saved && !make_tmap_bf16(&tg, a.G_saved, D, rows, D, 64, 128)))
    return cudaErrorInvalidValue;
  if (!a.W_chunks) twc = tk;  // never used
  if (!a.G_saved) tg = tk;    // never used
  FwdParams p{};
  p.BH = a.B * a.H;
  p.T = a.T;
  p.NC = a.T / a.C;
  p.nslice = D / NV;
  p.lr_bias = a.lr_bias;
  p.beta = a.beta;
  p.gamma = a.gamma;
  p.W0 = a.W0;
  p.w0_mod = a.w0_mod;
  p.O = static_cast<__nv_bfloat16*>(a.O);
  p.W_final = a.W_final;
  p.W_chunks = static_cast<__nv_bfloat16*>(a.W_chunks);
  p.save_g = a.G_saved != nullptr;
  // with SiLU the saved buffer has a second plane for Zq, which the backward needs for dZq
  p.Zq = ACT == 1 && a.G_saved ? static_cast<__nv_bfloat16*>(a.G_saved) + rows * D : nullptr;
  p.err = a.err;
  const size_t smem = L::BYTES + 1024;
  auto k = ttt_fwd_tc_kernel<D, NB, ACT, LOSS>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  k<<<p.BH * p.nslice, kThreads, smem, s>>>(tk, tq, tv, twc, tg, p);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace

bool tc_fwd_supported(const LayerArgs& a) {
  return a.dtype == 1 && !a.gvec && a.dk == a.dv && (a.dk == 64 || a.dk == 128) &&
         (a.C == 128 || a.C == 256) && a.T % a.C == 0;
}

size_t tc_fwd_workspace(const LayerArgs&) { return 0; }

template <int D, int NB>
cudaError_t launch_variant(const LayerArgs& a, cudaStream_t s) {
  if (a.act == 0) return a.loss == 0 ? launch<D, NB, 0, 0>(a, s) : launch<D, NB, 0, 1>(a, s);
  return a.loss == 0 ? launch<D, NB, 1, 0>(a, s) : launch<D, NB, 1, 1>(a, s);
}

cudaError_t tc_fwd(const LayerArgs& a, cudaStream_t s) {
  if (a.dk == 64) return a.C == 128 ? launch_variant<64, 1>(a, s) : launch_variant<64, 2>(a, s);
  return a.C == 128 ? launch_variant<128, 1>(a, s) : launch_variant<128, 2>(a, s);
}

}  // namespace tttk
