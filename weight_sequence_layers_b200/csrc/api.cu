// C ABI of the library: argument checks on the host, dispatch to the kernels, the per-device
// error word that bounded in-kernel waits report into, and the tensor-map encoder.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include <atomic>
#include <memory>
#include <new>
#include <mutex>
#include <vector>

#include "../../include/ttt.h"
#include "common.cuh"
#include "kernels.h"

namespace tttk {

// One error word per device: kernels OR error codes into it, ttt_get_device_error reads and
// clears it.
__device__ unsigned g_error_word;

namespace {

constexpr int kMaxDevices = 64;
unsigned* g_err_ptr[kMaxDevices];
std::mutex g_err_mu;

unsigned* error_word(cudaError_t* e) {
  int dev = 0;
  *e = cudaGetDevice(&dev);
  if (*e != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    if (*e == cudaSuccess) *e = cudaErrorInvalidDevice;
    return nullptr;
  }
  std::lock_guard<std::mutex> lk(g_err_mu);
  if (!g_err_ptr[dev]) {
    void* p = nullptr;
    *e = cudaGetSymbolAddress(&p, g_error_word);
    if (*e != cudaSuccess) return nullptr;
    g_err_ptr[dev] = static_cast<unsigned*>(p);
  }
  return g_err_ptr[dev];
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

// Checks the config; returns TTT_OK or the first failure.
ttt_status check_config(const ttt_config* c) {
  if (!c) return TTT_ERR_INVALID_ARG;
  if (c->B < 1 || c->H < 1 || c->T < 1 || c->dk < 1 || c->dv < 1 || c->C < 1)
    return TTT_ERR_INVALID_ARG;
  if (c->T % c->C) return TTT_ERR_INVALID_ARG;
  if (c->dtype != TTT_F32 && c->dtype != TTT_BF16) return TTT_ERR_INVALID_ARG;
  if (c->loss != TTT_LOSS_MSE && c->loss != TTT_LOSS_IP) return TTT_ERR_INVALID_ARG;
  if (c->act != TTT_ACT_ID && c->act != TTT_ACT_SILU) return TTT_ERR_INVALID_ARG;
  if (!isfinite(c->lr_bias)) return TTT_ERR_INVALID_ARG;
  if (c->decay != TTT_DECAY_SCALAR && c->decay != TTT_DECAY_VECTOR) return TTT_ERR_INVALID_ARG;
  if (c->w0_shared != 0 && c->w0_shared != 1) return TTT_ERR_INVALID_ARG;
  if ((long long)c->B * c->H * c->T * (c->dk > c->dv ? c->dk : c->dv) > (1ll << 40))
    return TTT_ERR_INVALID_ARG;
  // token rows are addressed with 32-bit indices (and TMA coordinates) inside the kernels
  if ((long long)c->B * c->H * c->T >= (1ll << 31)) return TTT_ERR_INVALID_ARG;
  return TTT_OK;
}

namespace {

LayerArgs args_of(const ttt_config* c) {
  LayerArgs a{};
  a.B = c->B;
  a.H = c->H;
  a.T = c->T;
  a.dk = c->dk;
  a.dv = c->dv;
  a.C = c->C;
  a.dtype = c->dtype;
  a.loss = c->loss;
  a.act = c->act;
  a.lr_bias = c->lr_bias;
  a.gvec = c->decay == TTT_DECAY_VECTOR;
  a.w0_mod = c->w0_shared ? c->H : c->B * c->H;
  return a;
}

enum Path { PATH_NONE, PATH_SIMT, PATH_TC, PATH_TC_VEC };

// The vector decay's forward on the tensor cores needs the decay itself (gamma non-NULL), which
// the workspace query does not see: it sizes for that case.
Path fwd_path(const LayerArgs& a) {
  if (a.dtype == TTT_BF16 && tc_fwd_supported(a)) return PATH_TC;
  if (a.dtype == TTT_BF16 && tc_vec_fwd_supported(a)) return PATH_TC_VEC;
  if (simt_supported(a)) return PATH_SIMT;
  return PATH_NONE;
}
// The tensor-core backward with SiLU reads the forward's Zq, saved beside G. A SiLU call on a
// tensor-core shape without it is refused rather than sent to the SIMT kernels, which would
// take several hundred times longer for the same result.
Path bwd_path(const LayerArgs& a, bool g_saved) {
  if (a.dtype == TTT_BF16 && tc_bwd_supported(a))
    return a.act == TTT_ACT_ID || g_saved ? PATH_TC : PATH_NONE;
  if (a.dtype == TTT_BF16 && tc_vec_fwd_supported(a)) return PATH_TC_VEC;
  if (simt_supported(a)) return PATH_SIMT;
  return PATH_NONE;
}

ttt_status launch_status(cudaError_t e) { return e == cudaSuccess ? TTT_OK : TTT_ERR_CUDA; }

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

__global__ void selftest_wait_kernel(unsigned spin_limit, unsigned* err) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // Nothing ever arrives on `bar`: the wait must give up after spin_limit polls.
    bool done = false;
    for (unsigned it = 0; it < spin_limit && !done; ++it) done = mbar_try_wait(smem_u32(&bar), 0);
    if (!done) atomicOr(err, ERR_WAIT_TIMEOUT);
  }
}

}  // namespace

unsigned* current_error_word() {
  cudaError_t e;
  return error_word(&e);
}

std::atomic<unsigned long long> g_launches{0};
void count_launches(int n) { g_launches.fetch_add((unsigned long long)n, std::memory_order_relaxed); }

bool make_tmap_bf16(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows,
                    uint64_t row_stride_elems, uint32_t box_inner, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {row_stride_elems * 2};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool make_tmap_f32(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows,
                   uint64_t row_stride_elems, uint32_t box_inner, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {row_stride_elems * 4};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool make_tmap3_bf16(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows,
                     uint64_t batch, uint64_t row_stride_elems, uint64_t batch_stride_elems,
                     uint32_t box_inner, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {inner, rows, batch};
  cuuint64_t strides[2] = {row_stride_elems * 2, batch_stride_elems * 2};
  cuuint32_t box[3] = {box_inner, box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace tttk

using namespace tttk;

extern "C" {

const char* ttt_status_string(ttt_status s) {
  switch (s) {
    case TTT_OK: return "ok";
    case TTT_ERR_INVALID_ARG: return "invalid argument";
    case TTT_ERR_UNSUPPORTED: return "unsupported configuration";
    case TTT_ERR_ALIGNMENT: return "pointer not 16-byte aligned";
    case TTT_ERR_WORKSPACE: return "workspace missing or too small";
    case TTT_ERR_CUDA: return "CUDA error";
    case TTT_ERR_TIMEOUT: return "bounded in-kernel wait timed out";
    case TTT_ERR_RANGE: return "input outside the range the kernel supports";
  }
  return "unknown status";
}

size_t ttt_workspace_bytes(const ttt_config* cfg, int for_bwd) {
  if (check_config(cfg) != TTT_OK) return (size_t)-1;
  LayerArgs a = args_of(cfg);
  if (!for_bwd) {
    a.gamma = reinterpret_cast<const float*>(16);  // a decay is given (never dereferenced)
    switch (fwd_path(a)) {
      case PATH_TC: return tc_fwd_workspace(a);
      case PATH_TC_VEC: return tc_vec_fwd_workspace(a);
      case PATH_SIMT: return simt_fwd_workspace(a);
      default: return (size_t)-1;
    }
  }
  if (for_bwd != 1 && for_bwd != 2) return (size_t)-1;
  a.gamma = reinterpret_cast<const float*>(16);  // as above
  switch (bwd_path(a, for_bwd == 2)) {
    case PATH_TC: return tc_bwd_workspace(a, for_bwd == 2, true);
    case PATH_TC_VEC: return tc_vec_bwd_workspace(a, for_bwd == 2);
    case PATH_SIMT: return simt_bwd_workspace(a);
    default: return (size_t)-1;
  }
}

ttt_status ttt_chunk_fwd(const ttt_config* cfg, const void* Q, const void* K, const void* V,
                         const float* beta, const float* gamma, const float* W0, void* O,
                         float* W_final, void* W_chunks, void* G_saved, void* workspace,
                         size_t workspace_bytes, void* stream) {
  ttt_status st = check_config(cfg);
  if (st != TTT_OK) return st;
  if (!Q || !K || !V || !beta || !W0 || !O) return TTT_ERR_INVALID_ARG;
  const void* ptrs[] = {Q, K, V, beta, gamma, W0, O, W_final, W_chunks, G_saved, workspace};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return TTT_ERR_ALIGNMENT;
  LayerArgs a = args_of(cfg);
  a.gamma = gamma;
  const Path path = fwd_path(a);
  if (path == PATH_NONE) return TTT_ERR_UNSUPPORTED;
  const size_t need = path == PATH_TC       ? tc_fwd_workspace(a)
                      : path == PATH_TC_VEC ? tc_vec_fwd_workspace(a)
                                            : simt_fwd_workspace(a);
  if (need && (!workspace || workspace_bytes < need)) return TTT_ERR_WORKSPACE;
  cudaError_t e;
  unsigned* err = error_word(&e);
  if (!err) return TTT_ERR_CUDA;
  a.Q = Q; a.K = K; a.V = V; a.beta = beta; a.gamma = gamma; a.W0 = W0; a.O = O;
  a.W_final = W_final; a.W_chunks = W_chunks; a.G_saved = G_saved; a.ws = workspace;
  a.ws_bytes = workspace_bytes;
  a.err = err;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return launch_status(path == PATH_TC       ? tc_fwd(a, s)
                       : path == PATH_TC_VEC ? tc_vec_fwd(a, s)
                                             : simt_fwd(a, s));
}

ttt_status ttt_chunk_bwd(const ttt_config* cfg, const void* Q, const void* K, const void* V,
                         const float* beta, const float* gamma, const float* W0,
                         const void* W_chunks, const void* G_saved, const void* dO,
                         const float* dW_final, const void* O, const float* W_final, void* dQ,
                         void* dK, void* dV, float* dbeta, float* dW0, float* dgamma,
                         void* workspace, size_t workspace_bytes, void* stream) {
  ttt_status st = check_config(cfg);
  if (st != TTT_OK) return st;
  if (!Q || !K || !V || !beta || !W0 || !W_chunks || !dO || !dQ || !dK || !dV || !dbeta || !dW0)
    return TTT_ERR_INVALID_ARG;
  // the decay gradient needs the decay, the forward's O, and W_final when dW_final is set
  if (dgamma && (!gamma || !O || (dW_final && !W_final))) return TTT_ERR_INVALID_ARG;
  const void* ptrs[] = {Q, K, V, beta, gamma, W0, W_chunks, G_saved, dO, dW_final,
                        O, W_final, dQ, dK, dV, dbeta, dW0, dgamma, workspace};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return TTT_ERR_ALIGNMENT;
  LayerArgs a = args_of(cfg);
  a.gamma = gamma;
  const Path path = bwd_path(a, G_saved != nullptr);
  if (path == PATH_NONE) return TTT_ERR_UNSUPPORTED;
  const size_t need =
      path == PATH_TC       ? tc_bwd_workspace(a, G_saved != nullptr, dgamma != nullptr)
      : path == PATH_TC_VEC ? tc_vec_bwd_workspace(a, G_saved != nullptr)
                            : simt_bwd_workspace(a);
  if (need && (!workspace || workspace_bytes < need)) return TTT_ERR_WORKSPACE;
  cudaError_t e;
  unsigned* err = error_word(&e);
  if (!err) return TTT_ERR_CUDA;
  a.Q = Q; a.K = K; a.V = V; a.beta = beta; a.gamma = gamma; a.W0 = W0; a.W_chunks =
      const_cast<void*>(W_chunks);
  a.G_saved = const_cast<void*>(G_saved);
  a.dO = dO; a.dW_final = dW_final; a.dQ = dQ; a.dK = dK; a.dV = dV; a.dbeta = dbeta;
  a.dW0 = dW0; a.ws = workspace; a.ws_bytes = workspace_bytes; a.err = err;
  a.O_in = O; a.W_final_in = W_final; a.dgamma = dgamma;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return launch_status(path == PATH_TC       ? tc_bwd(a, s)
                       : path == PATH_TC_VEC ? tc_vec_bwd(a, s)
                                             : simt_bwd(a, s));
}

size_t ttt_mlp_workspace_bytes(const ttt_config* cfg, int hidden) {
  if (check_config(cfg) != TTT_OK) return (size_t)-1;
  const LayerArgs a = args_of(cfg);
  if (!mlp_supported(a, hidden)) return (size_t)-1;
  const size_t simt = mlp_workspace(a, hidden);
  if (!mlp_tc_supported(a, hidden)) return simt;
  const size_t f = mlp_tc_fwd_workspace(a, hidden), b = mlp_tc_bwd_workspace(a, hidden);
  const size_t tc = f > b ? f : b;
  return tc > simt ? tc : simt;
}

ttt_status ttt_mlp_fwd(const ttt_config* cfg, int hidden, const void* Q, const void* K,
                       const void* V, const float* beta, const float* gamma, const float* W1_0,
                       const float* W2_0, void* O, float* W1_final, float* W2_final,
                       float* W1_chunks, float* W2_chunks, void* workspace,
                       size_t workspace_bytes, void* stream) {
  const ttt_status st = check_config(cfg);
  if (st != TTT_OK) return st;
  LayerArgs a = args_of(cfg);
  if (!mlp_supported(a, hidden)) return TTT_ERR_UNSUPPORTED;
  if (!Q || !K || !V || !beta || !W1_0 || !W2_0 || !O) return TTT_ERR_INVALID_ARG;
  const void* ptrs[] = {Q, K, V, beta, gamma, W1_0, W2_0, O, W1_final, W2_final, W1_chunks,
                        W2_chunks, workspace};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return TTT_ERR_ALIGNMENT;
  const bool tc = mlp_tc_supported(a, hidden);
  const size_t need = tc ? mlp_tc_fwd_workspace(a, hidden) : mlp_workspace(a, hidden);
  if (!workspace || workspace_bytes < need) return TTT_ERR_WORKSPACE;
  cudaError_t e;
  unsigned* err = error_word(&e);
  if (!err) return TTT_ERR_CUDA;
  a.Q = Q; a.K = K; a.V = V; a.beta = beta; a.gamma = gamma; a.O = O; a.ws = workspace;
  a.err = err;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  return launch_status(tc ? mlp_tc_fwd(a, hidden, W1_0, W2_0, W1_final, W2_final, W1_chunks,
                                       W2_chunks, s)
                          : mlp_fwd(a, hidden, W1_0, W2_0, W1_final, W2_final, W1_chunks,
                                    W2_chunks, s));
}

ttt_status ttt_mlp_bwd(const ttt_config* cfg, int hidden, const void* Q, const void* K,
                       const void* V, const float* beta, const float* gamma,
                       const float* W1_chunks, const float* W2_chunks, const void* dO,
                       const float* dW1_final, const float* dW2_final, void* dQ, void* dK,
                       void* dV, float* dbeta, float* dW1_0, float* dW2_0, void* workspace,
                       size_t workspace_bytes, void* stream) {
  const ttt_status st = check_config(cfg);
  if (st != TTT_OK) return st;
  LayerArgs a = args_of(cfg);
  if (!mlp_supported(a, hidden)) return TTT_ERR_UNSUPPORTED;
  if (!Q || !K || !V || !beta || !W1_chunks || !W2_chunks || !dO || !dQ || !dK || !dV || !dbeta ||
      !dW1_0 || !dW2_0)
    return TTT_ERR_INVALID_ARG;
  const void* ptrs[] = {Q, K, V, beta, gamma, W1_chunks, W2_chunks, dO, dW1_final, dW2_final,
                        dQ, dK, dV, dbeta, dW1_0, dW2_0, workspace};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return TTT_ERR_ALIGNMENT;
  const bool tc = mlp_tc_supported(a, hidden);
  const size_t need = tc ? mlp_tc_bwd_workspace(a, hidden) : mlp_workspace(a, hidden);
  if (!workspace || workspace_bytes < need) return TTT_ERR_WORKSPACE;
  cudaError_t e;
  unsigned* err = error_word(&e);
  if (!err) return TTT_ERR_CUDA;
  a.Q = Q; a.K = K; a.V = V; a.beta = beta; a.gamma = gamma; a.dO = dO; a.dQ = dQ; a.dK = dK;
  a.dV = dV; a.dbeta = dbeta; a.ws = workspace; a.err = err;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  return launch_status(tc ? mlp_tc_bwd(a, hidden, W1_chunks, W2_chunks, dW1_final, dW2_final,
                                       dW1_0, dW2_0, s)
                          : mlp_bwd(a, hidden, W1_chunks, W2_chunks, dW1_final, dW2_final,
                                    dW1_0, dW2_0, s));
}

size_t inplace_ttt_workspace_bytes(int T, int d_ff, int d_model, int C) {
  if (T < 1 || d_ff < 1 || d_model < 1 || C < 1 || T % C || C % 128 || d_ff % 64 ||
      d_model % 128)
    return (size_t)-1;
  return inplace_workspace(T, d_ff, d_model, C, false);
}

size_t inplace_ttt_docs_workspace_bytes(int T, int d_ff, int d_model, int C) {
  if (inplace_ttt_workspace_bytes(T, d_ff, d_model, C) == (size_t)-1) return (size_t)-1;
  return inplace_workspace(T, d_ff, d_model, C, true);
}

namespace {
ttt_status inplace_sizes(int T, int d_ff, int d_model, int C, float lr) {
  if (T < 1 || d_ff < 1 || d_model < 1 || C < 1 || T % C || !isfinite(lr))
    return TTT_ERR_INVALID_ARG;
  if (C % 128 || d_ff % 64 || d_model % 128) return TTT_ERR_UNSUPPORTED;
  if ((long long)T * d_ff > (1ll << 40) || (long long)(T / C) * d_model * d_ff > (1ll << 40))
    return TTT_ERR_INVALID_ARG;
  return TTT_OK;
}

// Chunk flags from a host list of document-start chunks (strictly increasing, each in
// [1, NC - 1]); false if the list is malformed.
bool doc_flags(const int* starts, int n, int NC, std::vector<bool>& flags) {
  try {
    flags.assign(NC, false);
  } catch (...) {
    return false;
  }
  if (n < 0 || (n > 0 && !starts)) return false;
  for (int k = 0; k < n; ++k) {
    if (starts[k] < 1 || starts[k] >= NC || (k > 0 && starts[k] <= starts[k - 1])) return false;
    flags[starts[k]] = true;
  }
  return true;
}

ttt_status inplace_fwd_impl(int T, int d_ff, int d_model, int C, float lr, const void* Z,
                            const void* Vhat, float* W, void* O, void* W_chunks,
                            const int* doc_starts, int n_docs, void* workspace,
                            size_t workspace_bytes, void* stream) {
  const ttt_status st = inplace_sizes(T, d_ff, d_model, C, lr);
  if (st != TTT_OK) return st;
  if (!Z || !Vhat || !W || !O) return TTT_ERR_INVALID_ARG;
  std::vector<bool> flags;
  if (!doc_flags(doc_starts, n_docs, T / C, flags)) return TTT_ERR_INVALID_ARG;
  const void* ptrs[] = {Z, Vhat, W, O, W_chunks, workspace};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return TTT_ERR_ALIGNMENT;
  const size_t need = inplace_workspace(T, d_ff, d_model, C, n_docs > 0);
  if (need && (!workspace || workspace_bytes < need)) return TTT_ERR_WORKSPACE;
  cudaError_t e;
  unsigned* err = error_word(&e);
  if (!err) return TTT_ERR_CUDA;
  std::unique_ptr<bool[]> reset(n_docs > 0 ? new (std::nothrow) bool[T / C] : nullptr);
  if (n_docs > 0 && !reset) return TTT_ERR_INVALID_ARG;
  for (int i = 0; reset && i < T / C; ++i) reset[i] = flags[i];
  return launch_status(inplace_run(T, d_ff, d_model, C, lr, Z, Vhat, W, O, W_chunks, reset.get(),
                                   workspace, err, static_cast<cudaStream_t>(stream)));
}

ttt_status inplace_bwd_impl(int T, int d_ff, int d_model, int C, float lr, const void* Z,
                            const void* Vhat, const void* W_chunks, const void* dO,
                            const float* dW_final, void* dZ, void* dVhat, float* dW,
                            const int* doc_starts, int n_docs, void* workspace,
                            size_t workspace_bytes, void* stream) {
  const ttt_status st = inplace_sizes(T, d_ff, d_model, C, lr);
  if (st != TTT_OK) return st;
  if (!Z || !Vhat || !W_chunks || !dO || !dZ || !dVhat || !dW) return TTT_ERR_INVALID_ARG;
  std::vector<bool> flags;
  if (!doc_flags(doc_starts, n_docs, T / C, flags)) return TTT_ERR_INVALID_ARG;
  const void* ptrs[] = {Z, Vhat, W_chunks, dO, dW_final, dZ, dVhat, dW, workspace};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return TTT_ERR_ALIGNMENT;
  const size_t need = inplace_workspace(T, d_ff, d_model, C, n_docs > 0);
  if (need && (!workspace || workspace_bytes < need)) return TTT_ERR_WORKSPACE;
  cudaError_t e;
  unsigned* err = error_word(&e);
  if (!err) return TTT_ERR_CUDA;
  std::unique_ptr<bool[]> reset(n_docs > 0 ? new (std::nothrow) bool[T / C] : nullptr);
  if (n_docs > 0 && !reset) return TTT_ERR_INVALID_ARG;
  for (int i = 0; reset && i < T / C; ++i) reset[i] = flags[i];
  return launch_status(inplace_bwd_run(T, d_ff, d_model, C, lr, Z, Vhat, W_chunks, dO, dW_final,
                                       dZ, dVhat, dW, reset.get(), workspace, err,
                                       static_cast<cudaStream_t>(stream)));
}
}  // namespace

ttt_status inplace_ttt_fwd(int T, int d_ff, int d_model, int C, float lr, const void* Z,
                           const void* Vhat, float* W, void* O, void* W_chunks, void* workspace,
                           size_t workspace_bytes, void* stream) {
  return inplace_fwd_impl(T, d_ff, d_model, C, lr, Z, Vhat, W, O, W_chunks, nullptr, 0,
                          workspace, workspace_bytes, stream);
}

ttt_status inplace_ttt_fwd_docs(int T, int d_ff, int d_model, int C, float lr, const void* Z,
                                const void* Vhat, float* W, void* O, void* W_chunks,
                                const int* doc_starts, int n_docs, void* workspace,
                                size_t workspace_bytes, void* stream) {
  return inplace_fwd_impl(T, d_ff, d_model, C, lr, Z, Vhat, W, O, W_chunks, doc_starts, n_docs,
                          workspace, workspace_bytes, stream);
}

size_t ttt_saved_bytes(const ttt_config* cfg) {
  if (check_config(cfg) != TTT_OK) return (size_t)-1;
  LayerArgs a = args_of(cfg);
  a.gamma = reinterpret_cast<const float*>(16);  // a decay is given (never dereferenced)
  if (fwd_path(a) == PATH_TC_VEC) return tc_vec_saved_bytes(a);
  const size_t elem = cfg->dtype == TTT_BF16 ? 2 : 4;
  return (size_t)cfg->B * cfg->H * cfg->T * cfg->dv * elem * (cfg->act == TTT_ACT_SILU ? 2 : 1);
}

ttt_status inplace_ttt_delta(int T, int d_ff, int d_model, float lr, const void* Z,
                             const void* Vhat, float* dW, void* workspace, size_t workspace_bytes,
                             void* stream) {
  if (T < 1 || d_ff < 1 || d_model < 1 || !isfinite(lr) || (long long)T * d_ff > (1ll << 40))
    return TTT_ERR_INVALID_ARG;
  if (T % 128 || d_ff % 64 || d_model % 128) return TTT_ERR_UNSUPPORTED;
  if (!Z || !Vhat || !dW) return TTT_ERR_INVALID_ARG;
  const void* ptrs[] = {Z, Vhat, dW, workspace};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return TTT_ERR_ALIGNMENT;
  if (!workspace || workspace_bytes < 256) return TTT_ERR_WORKSPACE;
  cudaError_t e;
  unsigned* err = error_word(&e);
  if (!err) return TTT_ERR_CUDA;
  return launch_status(inplace_delta_run(T, d_ff, d_model, lr, Z, Vhat, dW, workspace, err,
                                         static_cast<cudaStream_t>(stream)));
}

ttt_status ttt_add_f32(float* dst, const float* src, size_t n, void* stream) {
  if (!dst || !src || n % 4) return TTT_ERR_INVALID_ARG;
  if (!aligned16(dst) || !aligned16(src)) return TTT_ERR_ALIGNMENT;
  return launch_status(add_f32_run(dst, src, n, static_cast<cudaStream_t>(stream)));
}

size_t inplace_ttt_target_workspace_bytes(int T, int d_model) {
  if (T < 1 || d_model < 1 || T % 128 || d_model % 128 || (long long)T * d_model > (1ll << 40))
    return (size_t)-1;
  return inplace_target_workspace(T, d_model);
}

ttt_status inplace_ttt_target(int T, int d_model, int k, const void* X0, const float* conv_w,
                              const void* W_target, void* Vhat, void* workspace,
                              size_t workspace_bytes, void* stream) {
  if (T < 1 || d_model < 1 || k < 1 || (long long)T * d_model > (1ll << 40))
    return TTT_ERR_INVALID_ARG;
  if (T % 128 || d_model % 128 || k > 8) return TTT_ERR_UNSUPPORTED;
  if (!X0 || !conv_w || !W_target || !Vhat) return TTT_ERR_INVALID_ARG;
  const void* ptrs[] = {X0, conv_w, W_target, Vhat, workspace};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return TTT_ERR_ALIGNMENT;
  const size_t need = inplace_target_workspace(T, d_model);
  if (!workspace || workspace_bytes < need) return TTT_ERR_WORKSPACE;
  cudaError_t e;
  unsigned* err = error_word(&e);
  if (!err) return TTT_ERR_CUDA;
  return launch_status(inplace_target_run(T, d_model, k, X0, conv_w, W_target, Vhat, workspace,
                                          err, static_cast<cudaStream_t>(stream)));
}

size_t inplace_ttt_target_bwd_workspace_bytes(int T, int d_model, int k) {
  if (T < 1 || d_model < 1 || k < 1 || k > 8 || T % 128 || d_model % 128 ||
      (long long)T * d_model > (1ll << 40))
    return (size_t)-1;
  return inplace_target_bwd_workspace(T, d_model, k);
}

ttt_status inplace_ttt_target_bwd(int T, int d_model, int k, const void* X0, const float* conv_w,
                                  const void* W_target, const void* dVhat, void* dX0,
                                  float* dconv_w, float* dW_target, void* workspace,
                                  size_t workspace_bytes, void* stream) {
  if (T < 1 || d_model < 1 || k < 1 || (long long)T * d_model > (1ll << 40))
    return TTT_ERR_INVALID_ARG;
  if (T % 128 || d_model % 128 || k > 8) return TTT_ERR_UNSUPPORTED;
  if (!X0 || !conv_w || !W_target || !dVhat || !dX0 || !dconv_w || !dW_target)
    return TTT_ERR_INVALID_ARG;
  const void* ptrs[] = {X0, conv_w, W_target, dVhat, dX0, dconv_w, dW_target, workspace};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return TTT_ERR_ALIGNMENT;
  if (!workspace || workspace_bytes < inplace_target_bwd_workspace(T, d_model, k))
    return TTT_ERR_WORKSPACE;
  cudaError_t e;
  unsigned* err = error_word(&e);
  if (!err) return TTT_ERR_CUDA;
  return launch_status(inplace_target_bwd_run(T, d_model, k, X0, conv_w, W_target, dVhat, dX0,
                                              dconv_w, dW_target, workspace, err,
                                              static_cast<cudaStream_t>(stream)));
}

ttt_status inplace_ttt_bwd(int T, int d_ff, int d_model, int C, float lr, const void* Z,
                           const void* Vhat, const void* W_chunks, const void* dO,
                           const float* dW_final, void* dZ, void* dVhat, float* dW,
                           void* workspace, size_t workspace_bytes, void* stream) {
  return inplace_bwd_impl(T, d_ff, d_model, C, lr, Z, Vhat, W_chunks, dO, dW_final, dZ, dVhat, dW,
                          nullptr, 0, workspace, workspace_bytes, stream);
}

ttt_status inplace_ttt_bwd_docs(int T, int d_ff, int d_model, int C, float lr, const void* Z,
                                const void* Vhat, const void* W_chunks, const void* dO,
                                const float* dW_final, void* dZ, void* dVhat, float* dW,
                                const int* doc_starts, int n_docs, void* workspace,
                                size_t workspace_bytes, void* stream) {
  return inplace_bwd_impl(T, d_ff, d_model, C, lr, Z, Vhat, W_chunks, dO, dW_final, dZ, dVhat, dW,
                          doc_starts, n_docs, workspace, workspace_bytes, stream);
}

ttt_status ttt_get_device_error(void* stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return TTT_ERR_CUDA;
  cudaError_t e;
  unsigned* err = error_word(&e);
  if (!err) return TTT_ERR_CUDA;
  unsigned h = 0;
  if (cudaMemcpy(&h, err, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess) return TTT_ERR_CUDA;
  if (h) {
    const unsigned zero = 0;
    if (cudaMemcpy(err, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess)
      return TTT_ERR_CUDA;
    return (h & ERR_WAIT_TIMEOUT) ? TTT_ERR_TIMEOUT : TTT_ERR_RANGE;
  }
  return TTT_OK;
}

unsigned long long ttt_kernel_launches(void) { return g_launches.load(); }

ttt_status ttt_selftest_bounded_wait(unsigned spin_limit, void* stream) {
  cudaError_t e;
  unsigned* err = error_word(&e);
  if (!err) return TTT_ERR_CUDA;
  selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(spin_limit, err);
  count_launches(1);
  return launch_status(cudaGetLastError());
}

}  // extern "C"
