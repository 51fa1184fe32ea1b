// Host-side interface between the C ABI (api.cu) and the kernel translation units.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>

#include <mutex>

namespace tttk {

struct LayerArgs {
  int B, H, T, dk, dv, C, dtype, loss, act;
  float lr_bias;
  int gvec;  // gamma is [B, H, T, dk]: one decay per key feature
  int w0_mod;  // the initial state of (batch, head) bh is block bh % w0_mod of W0 (H: shared)
  const void *Q, *K, *V;
  const float *beta, *gamma, *W0;
  void* O;
  float* W_final;
  void* W_chunks;
  void* G_saved;  // nullable: G of every token [B, H, T, dv]
  const void* dO;
  const float* dW_final;
  const void* O_in;        // forward output, read for dgamma
  const float* W_final_in; // forward output, read for dgamma when dW_final is set
  float* dgamma;           // nullable
  void *dQ, *dK, *dV;
  float *dbeta, *dW0;
  void* ws;
  size_t ws_bytes;
  unsigned* err;  // per-device error word
};

// SIMT kernels (float32 or bf16 storage, float32 arithmetic).
size_t simt_fwd_workspace(const LayerArgs& a);
size_t simt_bwd_workspace(const LayerArgs& a);
bool simt_supported(const LayerArgs& a);
cudaError_t simt_fwd(const LayerArgs& a, cudaStream_t s);
cudaError_t simt_bwd(const LayerArgs& a, cudaStream_t s);

// tcgen05 kernels (bf16 storage).
bool tc_fwd_supported(const LayerArgs& a);
size_t tc_fwd_workspace(const LayerArgs& a);
cudaError_t tc_fwd(const LayerArgs& a, cudaStream_t s);
// Vector (per-feature) decay, identity activation, d_k = d_v = 64: a chunk-parallel pass that
// forms the decayed operands, a serial state pass and a chunk-parallel readout on the tensor
// cores.
bool tc_vec_fwd_supported(const LayerArgs& a);
size_t tc_vec_fwd_workspace(const LayerArgs& a);
cudaError_t tc_vec_fwd(const LayerArgs& a, cudaStream_t s);
// Its backward (same shapes; reads the forward's W_chunks and, when given, its saved buffer:
// G, the decayed operands with L, and R).
size_t tc_vec_bwd_workspace(const LayerArgs& a, bool g_saved);
size_t tc_vec_saved_bytes(const LayerArgs& a);
cudaError_t tc_vec_bwd(const LayerArgs& a, cudaStream_t s);

// The decayed operands of the vector decay, one chunk-parallel pass (chunk-local L, chunk
// length C = 128 NB, query block qb with reference token m(qb) = 128 qb + 63).
struct VecPrep {
  void* Qt;   // bf16 [B H T, 64]: q_s exp(L_s - L_m(qb(s)))
  void* Kh;   // bf16 [B H T, 64]: k_r exp(L_C - L_r)
  void* Kt;   // bf16 [B H NC NV 128, 64]: k_r exp(L_m(qb) - L_r) for every qb >= kb(r),
              // version v = qb (qb + 1) / 2 + kb(r), NV = NB (NB + 1) / 2
  float* GC;  // float32 [B H NC, 64]: exp(L_C)
  float* Em;  // float32 [B H NC NB, 64]: exp(L_m(qb))
  float* Lf;  // nullable: float32 [B H T, 64], L itself
  void* Qt2;  // nullable (C = 256, with L): bf16 [B H NC 128, 64], the second query block's
              // q_s exp(L_s - L_m(0)) (the backward's key side refers both blocks to m(0))
};
size_t vec_prep_bytes(const LayerArgs& a, bool with_L);
VecPrep vec_prep_carve(const LayerArgs& a, void* base, bool with_L);
cudaError_t vec_prep(const LayerArgs& a, const VecPrep& o, cudaStream_t s);
bool tc_bwd_supported(const LayerArgs& a);
size_t tc_bwd_workspace(const LayerArgs& a, bool g_saved, bool dgamma);
cudaError_t tc_bwd(const LayerArgs& a, cudaStream_t s);

// TTT-MLP on the tensor cores (bf16, d = 64, hidden 128 or 256, C = 128 or 256): a program of
// batched tcgen05 GEMMs with fused epilogues.
bool mlp_tc_supported(const LayerArgs& a, int hidden);
size_t mlp_tc_fwd_workspace(const LayerArgs& a, int hidden);
cudaError_t mlp_tc_fwd(const LayerArgs& a, int hidden, const float* W1_0, const float* W2_0,
                       float* W1f, float* W2f, float* W1c, float* W2c, cudaStream_t s);
size_t mlp_tc_bwd_workspace(const LayerArgs& a, int hidden);
cudaError_t mlp_tc_bwd(const LayerArgs& a, int hidden, const float* W1c, const float* W2c,
                       const float* dW1f, const float* dW2f, float* dW1_0, float* dW2_0,
                       cudaStream_t s);

// TTT-MLP (SIMT).
bool mlp_supported(const LayerArgs& a, int hidden);
size_t mlp_workspace(const LayerArgs& a, int hidden);
cudaError_t mlp_fwd(const LayerArgs& a, int hidden, const float* W1_0, const float* W2_0,
                    float* W1f, float* W2f, float* W1c, float* W2c, cudaStream_t s);
cudaError_t mlp_bwd(const LayerArgs& a, int hidden, const float* W1c, const float* W2c,
                    const float* dW1f, const float* dW2f, float* dW1_0, float* dW2_0,
                    cudaStream_t s);

// In-Place TTT.
// `reset` (nullable, host, NC entries): chunks that start a new document.
size_t inplace_workspace(int T, int d_ff, int d_model, int C, bool docs);
cudaError_t inplace_run(int T, int d_ff, int d_model, int C, float lr, const void* Z,
                        const void* Vhat, float* W, void* O, void* W_chunks, const bool* reset,
                        void* ws, unsigned* err, cudaStream_t s);
size_t inplace_target_workspace(int T, int d);
cudaError_t inplace_target_run(int T, int d, int k, const void* X0, const float* conv_w,
                               const void* W_target, void* Vhat, void* ws, unsigned* err,
                               cudaStream_t s);
size_t inplace_target_bwd_workspace(int T, int d, int k);
cudaError_t inplace_target_bwd_run(int T, int d, int k, const void* X0, const float* conv_w,
                                   const void* W_target, const void* dVhat, void* dX0,
                                   float* dconv_w, float* dW_target, void* ws, unsigned* err,
                                   cudaStream_t s);
cudaError_t inplace_delta_run(int T, int d_ff, int d_model, float lr, const void* Z,
                              const void* Vhat, float* dW, void* ws, unsigned* err,
                              cudaStream_t s);
cudaError_t add_f32_run(float* dst, const float* src, size_t n, cudaStream_t s);
cudaError_t inplace_bwd_run(int T, int d_ff, int d_model, int C, float lr, const void* Z,
                            const void* Vhat, const void* W_chunks, const void* dO,
                            const float* dW_final, void* dZ, void* dVhat, float* dW,
                            const bool* reset, void* ws, unsigned* err, cudaStream_t s);

// Address of the current device's error word (looked up once per device); NULL on failure.
unsigned* current_error_word();

// Adds n to the process-wide count of kernel launches (reported by ttt_kernel_launches).
void count_launches(int n);

// 2-D bf16 tensor map with 128-byte swizzle: `rows` rows of `inner` elements, rows
// `row_stride_elems` apart; box = {box_inner (64), box_rows}. Returns false on failure.
bool make_tmap_bf16(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows,
                    uint64_t row_stride_elems, uint32_t box_inner, uint32_t box_rows);
// 2-D float32 tensor map without swizzle (row-major boxes of box_rows x box_inner floats).
bool make_tmap_f32(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows,
                   uint64_t row_stride_elems, uint32_t box_inner, uint32_t box_rows);
// 3-D bf16 tensor map (inner, rows, batch) with 128-byte swizzle; box = {box_inner, box_rows, 1}.
bool make_tmap3_bf16(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows,
                     uint64_t batch, uint64_t row_stride_elems, uint64_t batch_stride_elems,
                     uint32_t box_inner, uint32_t box_rows);

// The tensor-core backward's per-device pair of internal streams (the serial chain at the
// higher priority, the chunk-parallel work that does not depend on it at the lower) and the
// events that fork the caller's stream into them and join it again, created on first use. A
// backward enqueues its whole sequence while holding fork_mutex(), so calls from several host
// threads keep their dependencies.
struct ForkSet {
  cudaStream_t hi = nullptr, lo = nullptr;
  cudaEvent_t e0 = nullptr, eg = nullptr, ehi = nullptr, elo = nullptr;
};
ForkSet* fork_set();      // nullptr if the streams or events cannot be created
std::mutex& fork_mutex();

}  // namespace tttk
