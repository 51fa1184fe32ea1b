// ttt_chunk_bwd_noalloc: the tensor-core backward with its scratch in a fixed device array,
// for callers that cannot allocate device memory at call time (see include/ttt.h).
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include <mutex>

#include "../../include/ttt.h"
#include "kernels.h"

namespace tttk {

ttt_status check_config(const ttt_config* c);  // api.cu

namespace {

// The scratch of every ttt_chunk_bwd_noalloc call on this device. In host code this name is
// only a stand-in: its device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[TTT_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
void* g_scratch_ptr[kMaxDevices];
std::mutex g_scratch_mu;

// Device address of the array on the current device, looked up on first use per device.
void* scratch_address() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
    g_scratch_ptr[dev] = p;
  }
  return g_scratch_ptr[dev];
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace tttk

using namespace tttk;

extern "C" ttt_status ttt_chunk_bwd_noalloc(const ttt_config* cfg, const void* Q, const void* K,
                                            const void* V, const float* beta, const float* gamma,
                                            const float* W0, const void* W_chunks,
                                            const void* G_saved, const void* dO,
                                            const float* dW_final, const void* O,
                                            const float* W_final, void* dQ, void* dK, void* dV,
                                            float* dbeta, float* dW0, float* dgamma,
                                            void* stream) {
  const ttt_status cs = check_config(cfg);
  if (cs != TTT_OK) return cs;
  if (!Q || !K || !V || !beta || !W0 || !W_chunks || !dO || !dQ || !dK || !dV || !dbeta || !dW0)
    return TTT_ERR_INVALID_ARG;
  if (dgamma && (!gamma || !O || (dW_final && !W_final))) return TTT_ERR_INVALID_ARG;
  const void* ptrs[] = {Q, K, V, beta, gamma, W0, W_chunks, G_saved, dO, dW_final,
                        O, W_final, dQ, dK, dV, dbeta, dW0, dgamma};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return TTT_ERR_ALIGNMENT;
  LayerArgs a{};
  a.B = cfg->B; a.H = cfg->H; a.T = cfg->T; a.dk = cfg->dk; a.dv = cfg->dv; a.C = cfg->C;
  a.dtype = cfg->dtype; a.loss = cfg->loss; a.act = cfg->act; a.lr_bias = cfg->lr_bias;
  a.gvec = cfg->decay == TTT_DECAY_VECTOR;
  // SiLU on the tensor cores also needs the forward's saved G and Zq
  if (!tc_bwd_supported(a) || (a.act == TTT_ACT_SILU && !G_saved)) return TTT_ERR_UNSUPPORTED;
  const size_t need = tc_bwd_workspace(a, G_saved != nullptr, dgamma != nullptr);
  if (need > TTT_NOALLOC_SCRATCH_BYTES) return TTT_ERR_WORKSPACE;
  void* scratch = scratch_address();
  unsigned* err = current_error_word();
  if (!scratch || !err) return TTT_ERR_CUDA;
  a.Q = Q; a.K = K; a.V = V; a.beta = beta; a.gamma = gamma; a.W0 = W0;
  a.W_chunks = const_cast<void*>(W_chunks);
  a.G_saved = const_cast<void*>(G_saved);
  a.dO = dO; a.dW_final = dW_final; a.dQ = dQ; a.dK = dK; a.dV = dV; a.dbeta = dbeta;
  a.dW0 = dW0; a.ws = scratch; a.ws_bytes = TTT_NOALLOC_SCRATCH_BYTES; a.err = err;
  a.O_in = O; a.W_final_in = W_final; a.dgamma = dgamma;
  return tc_bwd(a, static_cast<cudaStream_t>(stream)) == cudaSuccess ? TTT_OK : TTT_ERR_CUDA;
}
