/*
 * ttt.h -- C ABI of the B200 (sm_100a) chunkwise test-time-training library.
 *
 * The operations follow two papers, as described on the pages they are cited from:
 *
 *  - Modular TTT (page "Modular TTT: Rethinking Test-Time Training as Composable
 *    Modules"): the hidden state is a fast weight W (d_k x d_v per batch and head),
 *    trained online on keys/values and read with queries. Per chunk of C tokens,
 *    section "方法步骤详情" (Algorithm 1) runs three passes: train-view forward
 *    Z = K W0 (optionally one SiLU, section "实验结果": a single nonlinearity after
 *    Linear), train-view backward of the inner loss (MSE or inner product), and the
 *    causal query-view readout O = Q W_start - Tril(Q Khat^T) dVhat, ending with the
 *    state transition W_end = W_start - Khat^T dVhat. The learning rate is
 *    eta_t = 2 sigmoid(beta_t + b) (section "内部学习规则与学习率参数化"); a decay
 *    shrinks past writes (section "权重衰减"): scalar, or per feature (vector decay, one
 *    factor per key feature scaling that row of W).
 *  - In-Place TTT (page "In-Place Test-Time Training", section "核心方法和技术细节"):
 *    W_down of a gated MLP is the fast weight; per chunk O_i = Z_i W_i^T, then
 *    W_{i+1} = W_i + eta Vhat_i^T Z_i.
 *
 * Exact per-token semantics implemented (one head; t = token, s = position in its chunk,
 * W0 = state at the chunk start, act = identity or SiLU):
 *     z_t  = k_t W0;   g_t = a_t * act'(z_t),  a_t = act(z_t) - v_t (MSE) or -v_t (IP)
 *     eta_t = 2 sigmoid(beta_t + lr_bias)
 *     W_t  = gamma_t W_{t-1} - eta_t k_t^T g_t          (gamma_t = 1 without decay;
 *                                                       diag(gamma_t) for a vector decay)
 *     o_t  = act(q_t W_t)                              (the token reads its own write)
 * which the kernels evaluate in the chunk dual form.
 *
 * Conventions shared by every entry point
 *  - All tensor pointers are DEVICE pointers to contiguous row-major buffers owned by
 *    the caller; the library never allocates, frees or retains them. Scratch memory is
 *    passed in as `workspace` (size from the matching *_workspace_bytes query).
 *  - Work is enqueued asynchronously on `stream` (a cudaStream_t; NULL = the legacy
 *    default stream). A call returns after argument checks and launches; results are
 *    ready when the stream reaches that point.
 *  - Argument checks run on the host before anything is launched. On any error nothing
 *    is launched and no output is touched. Device pointers must be 16-byte aligned.
 *  - No exceptions cross the ABI and the library keeps no per-call state: calls on different
 *    streams may overlap provided their buffers do not alias, with one exception. The
 *    tensor-core path of ttt_chunk_bwd forks the caller's stream onto two library-owned
 *    streams of the current device (it runs its serial adjoint kernel beside a chunk-parallel
 *    one) and joins them back into the caller's stream before returning; these streams and four
 *    events are created by the first such call on each device and shared by every later call,
 *    under a process-wide lock. Backward calls from different streams or host threads therefore
 *    serialise on the GPU, and the first tensor-core backward on a device should come before
 *    any stream capture.
 *  - Kernels never trap. Every wait inside a kernel is bounded; a wait that runs out
 *    sets a per-device error word and the kernel returns early (outputs then invalid).
 *    ttt_get_device_error() reports and clears it.
 */
#ifndef TTT_H_
#define TTT_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  TTT_OK = 0,
  TTT_ERR_INVALID_ARG = 1,  /* NULL required pointer, bad sizes, T % C != 0, ...      */
  TTT_ERR_UNSUPPORTED = 2,  /* valid but outside what the kernels implement           */
  TTT_ERR_ALIGNMENT = 3,    /* a pointer is not 16-byte aligned                        */
  TTT_ERR_WORKSPACE = 4,    /* workspace NULL or smaller than the query returned       */
  TTT_ERR_CUDA = 5,         /* a CUDA runtime call or kernel launch failed             */
  TTT_ERR_TIMEOUT = 6,      /* a bounded in-kernel wait ran out (device error word)     */
  TTT_ERR_RANGE = 7         /* an input left the range a kernel supports (device error
                               word), e.g. a vector decay too strong for the tensor cores */
} ttt_status;

typedef enum { TTT_F32 = 0, TTT_BF16 = 1 } ttt_dtype;    /* type of Q,K,V,O,dO,dQ,dK,dV     */
typedef enum { TTT_LOSS_MSE = 0, TTT_LOSS_IP = 1 } ttt_loss;
typedef enum { TTT_ACT_ID = 0, TTT_ACT_SILU = 1 } ttt_act;
typedef enum { TTT_DECAY_SCALAR = 0, TTT_DECAY_VECTOR = 1 } ttt_decay;

/* Shape and variant of one TTT layer call. */
typedef struct {
  int B, H;        /* batch, heads                                                     */
  int T;           /* tokens per sequence; T % C == 0; B * H * T < 2^31                   */
  int dk, dv;      /* key/query width and value width of the fast weight (1..128)        */
  int C;           /* chunk size (semantic: gradients inside a chunk are taken at W0)    */
  int dtype;       /* ttt_dtype                                                         */
  int loss;        /* ttt_loss: MSE = 1/2||act(z)-v||^2, IP = -<act(z), v>               */
  int act;         /* ttt_act applied to both the train view and the query view         */
  float lr_bias;   /* b in eta_t = 2 sigmoid(beta_t + b)                                 */
  int decay;       /* ttt_decay: layout of gamma (zero-initialised configs: scalar)      */
  int w0_shared;   /* 0: W0 (and W1_0, W2_0 of TTT-MLP) holds one initial state per sequence
                      and head, [B, H, ...]; 1: one per head, [H, ...], shared by the B
                      sequences. W_final, W_chunks and dW0 stay per sequence either way; a
                      caller that shares W0 sums dW0 over B. Zero-initialised configs: 0.  */
} ttt_config;

/* Layouts (all contiguous):
 *   Q, K, dQ, dK        [B, H, T, dk]   dtype
 *   V, O, dO, dV        [B, H, T, dv]   dtype
 *   beta, dbeta         [B, H, T]       float32
 *   gamma, dgamma       [B, H, T] (scalar decay) or [B, H, T, dk] (vector decay)  float32;
 *                       gamma NULL = no decay (gamma == 1)
 *   W0, W_final, dW_final, dW0   [B, H, dk, dv]  float32, row index = key feature
 *   W_chunks            [B, H, T/C, dk, dv]  dtype: the state at the start of every chunk
 *   G_saved             [B, H, T, dv]   dtype: G of every token, the value the token's write
 *                       subtracts (W_t = gamma_t W_{t-1} - eta_t k_t^T g_t); with SiLU
 *                       [2, B, H, T, dv]: G, then Zq = q_t W_t, the readout before the activation
 */

/* Bytes of workspace ttt_chunk_fwd (for_bwd = 0) or ttt_chunk_bwd needs for this config; 0 if
 * none. for_bwd = 1: the backward without G_saved (it rebuilds G in the workspace); for_bwd = 2:
 * the backward given G_saved. The backward figure covers a call that asks for dgamma (on the
 * tensor-core path that adds B*H*T*4 bytes, which calls without dgamma do not touch).
 * Returns (size_t)-1 if the config (or for_bwd) is invalid. */
size_t ttt_workspace_bytes(const ttt_config* cfg, int for_bwd);

/* Bytes of the G_saved buffer of this config (B*H*T*dv elements of cfg->dtype, twice that with
 * SiLU, where Zq follows G); on the vector-decay tensor-core path (bf16, vector decay, identity,
 * dk == dv == 64, C in {128, 256}) G is followed by the decayed operands the forward forms
 * (q and k scaled per feature, the log decay L of every token) and the effective query R, so
 * that the backward need not form them again: B*H*T*64*2 bytes for G, then that library-defined
 * region. (size_t)-1 if the config is invalid. */
size_t ttt_saved_bytes(const ttt_config* cfg);

/* Forward of the chunkwise TTT layer.
 *  in : Q, K, V, beta, gamma (nullable), W0
 *  out: O; W_final (nullable) = state after the last token; W_chunks (nullable) = chunk-start
 *       states, needed by ttt_chunk_bwd; G_saved (nullable) = G of every token (and, with
 *       SiLU, Zq), which ttt_chunk_bwd then reads instead of rebuilding it.
 * bf16 configs with dk == dv in {64, 128}, C in {128, 256} and a scalar decay (or none) run on
 * the tcgen05 kernel. A vector decay with bf16, dk == dv == 64, C in {128, 256} and the
 * identity activation runs on tcgen05 kernels too: its per-feature weights enter the Q K^T
 * contraction as operands scaled against a reference token in the middle of each 128-query
 * block, so each scaled factor spans at most 64 tokens of one feature's decay; a factor beyond
 * exp(80) (a feature's decay product below e^-80 over 64 tokens) is clamped and reported as
 * TTT_ERR_RANGE by ttt_get_device_error, and such inputs take the float32 config instead. Other
 * shapes (dk, dv <= 128, C <= 256), all float32 configs and the other vector-decay configs run
 * on the SIMT kernels. */
ttt_status ttt_chunk_fwd(const ttt_config* cfg, const void* Q, const void* K, const void* V,
                         const float* beta, const float* gamma, const float* W0, void* O,
                         float* W_final, void* W_chunks, void* G_saved, void* workspace,
                         size_t workspace_bytes, void* stream);

/* Analytic backward of the layer for the objective J = <dO, O> + <dW_final, W_final>.
 *  in : Q, K, V, beta, gamma (nullable), W0, W_chunks (from ttt_chunk_fwd, required),
 *       G_saved (from ttt_chunk_fwd, nullable: rebuilt from W_chunks when NULL; kernels that
 *       rebuild G anyway may ignore it; with SiLU the tensor-core backward needs it, for Zq,
 *       and a SiLU call on a tensor-core shape without it returns TTT_ERR_UNSUPPORTED; on the
 *       vector-decay tensor-core path it supplies the forward's decayed operands and R),
 *       dO, dW_final (nullable = 0);
 *       O and W_final (the forward's outputs) are read only for dgamma (then O is required,
 *       and W_final too when dW_final is non-NULL).
 *  out: dQ, dK, dV, dbeta, dW0 (plain stores, not accumulated); dgamma (nullable; requires
 *       gamma) = dJ/dgamma. If the caller shares W0 across the batch it reduces dW0 over B.
 * The decay gradient follows from L_s = sum_{t<=s} log gamma_t (chunk-local): with Zq the
 * readout before the activation and dG the adjoint of G,
 *     dJ/dL_s = dZq_s . Zq_s - g_s . dG_s  (+ <W_end, dW_end> on the chunk's last token)
 *     dgamma_t = (1 / gamma_t) sum_{s >= t in the chunk} dJ/dL_s.
 * For a vector decay L_s has one entry per key feature i and, with dZ the adjoint of
 * Z = K W0,
 *     dJ/dL_si = q_si dQ_si - k_si (dK_si - (dZ_s W0^T)_i)  (+ row i of <W_end, dW_end>)
 *     dgamma_ti = (1 / gamma_ti) sum_{s >= t in the chunk} dJ/dL_si. */
ttt_status ttt_chunk_bwd(const ttt_config* cfg, const void* Q, const void* K, const void* V,
                         const float* beta, const float* gamma, const float* W0,
                         const void* W_chunks, const void* G_saved, const void* dO,
                         const float* dW_final, const void* O, const float* W_final, void* dQ,
                         void* dK, void* dV, float* dbeta, float* dW0, float* dgamma,
                         void* workspace, size_t workspace_bytes, void* stream);

/* Backward without caller-provided scratch (no counterpart in the papers: a deployment aid).
 * Some callers cannot allocate device memory when they call the library: a host framework
 * that owns every byte of device memory through its own pool, or a plugin that is handed only
 * its input and output buffers. For them this variant takes the same arguments as
 * ttt_chunk_bwd minus the workspace, and keeps its scratch (the per-chunk adjoint states and
 * the bf16 inner-loss gradient G of every token) in a fixed array of TTT_NOALLOC_SCRATCH_BYTES
 * that the library holds on every GPU it is loaded on, until the process exits. It allocates no
 * device memory and calls no allocating routine.
 *  - Only configs of the tensor-core backward are accepted (bf16, dk == dv in {64, 128},
 *    C in {128, 256}, scalar or no decay; SiLU only with G_saved); others return
 *    TTT_ERR_UNSUPPORTED.
 *  - Configs needing more than the fixed scratch (B*H*(T/C)*dk*dv*2 bytes, plus B*H*T*dv*2 when
 *    G_saved is NULL, plus B*H*T*4 when dgamma is non-NULL, plus 4*B*H*T*dv*2 with SiLU) return
 *    TTT_ERR_WORKSPACE with nothing launched; ttt_chunk_bwd serves those.
 *  - The first call on a device looks up the array's device address (with that device
 *    current) and, unless a ttt_chunk_bwd call on the tensor cores ran there before, creates
 *    the library's two fork streams and four events of that device (see the stream conventions
 *    at the top): make that first call before any stream capture. Later calls create nothing.
 *  - Every call shares the one array and leaves its contents behind. Calls that overlap on
 *    the GPU (different streams, or different host threads) race on it: serialise them.
 *    Nothing in the array has to start at zero. */
#define TTT_NOALLOC_SCRATCH_BYTES ((size_t)8 << 20)
ttt_status ttt_chunk_bwd_noalloc(const ttt_config* cfg, const void* Q, const void* K, const void* V,
                                 const float* beta, const float* gamma, const float* W0,
                                 const void* W_chunks, const void* G_saved, const void* dO,
                                 const float* dW_final, const void* O, const float* W_final,
                                 void* dQ, void* dK, void* dV, float* dbeta, float* dW0,
                                 float* dgamma, void* stream);

/* TTT-MLP: the fast weight is the two-layer network vhat = act(k W1) W2 (page "Modular TTT:
 * Rethinking Test-Time Training as Composable Modules", TTT-MLP; cfg->act is the hidden
 * activation, the output layer is linear). Per token t of a chunk, gradients at the chunk-start
 * weights W1_0, W2_0:
 *     z = k W1_0, a = act(z), g2 = a W2_0 - v (MSE) or -v (IP), g1 = (g2 W2_0^T) * act'(z)
 *     W1_t = gamma_t W1_{t-1} - eta_t k^T g1,  W2_t = gamma_t W2_{t-1} - eta_t a^T g2
 *     o_t  = act(q_t W1_t) W2_t
 * evaluated in the chunk dual form. bf16 configs with dk == dv == 64, hidden in {128, 256} and
 * C in {128, 256} run as a program of batched tcgen05 GEMMs with fused epilogues (fp32
 * accumulation and fp32 master weights); the others on the SIMT kernels (float32 arithmetic).
 * Layouts: Q, K, dQ, dK [B,H,T,dk] and V, O, dO, dV [B,H,T,dv] in cfg->dtype; beta, gamma, dbeta
 * [B,H,T] float32 (gamma nullable; scalar decay only); W1 [B,H,dk,hidden], W2 [B,H,hidden,dv]
 * float32, likewise W1_final, W2_final, dW1_final, dW2_final, dW1_0, dW2_0; W1_chunks
 * [B,H,T/C,dk,hidden] and W2_chunks [B,H,T/C,hidden,dv] float32 (chunk-start weights, written by
 * the forward when non-NULL, required by the backward). dk, dv <= 128, hidden <= 512, C <= 256. */
size_t ttt_mlp_workspace_bytes(const ttt_config* cfg, int hidden);
ttt_status ttt_mlp_fwd(const ttt_config* cfg, int hidden, const void* Q, const void* K,
                       const void* V, const float* beta, const float* gamma, const float* W1_0,
                       const float* W2_0, void* O, float* W1_final, float* W2_final,
                       float* W1_chunks, float* W2_chunks, void* workspace,
                       size_t workspace_bytes, void* stream);
/* Backward for J = <dO, O> + <dW1_final, W1_final> + <dW2_final, W2_final> (dW*_final nullable
 * = 0): dQ, dK, dV, dbeta and the gradients of the initial weights dW1_0, dW2_0. */
ttt_status ttt_mlp_bwd(const ttt_config* cfg, int hidden, const void* Q, const void* K,
                       const void* V, const float* beta, const float* gamma,
                       const float* W1_chunks, const float* W2_chunks, const void* dO,
                       const float* dW1_final, const float* dW2_final, void* dQ, void* dK,
                       void* dV, float* dbeta, float* dW1_0, float* dW2_0, void* workspace,
                       size_t workspace_bytes, void* stream);

/* Workspace bytes of inplace_ttt_fwd and of inplace_ttt_bwd (the same figure);
 * (size_t)-1 for invalid sizes. */
size_t inplace_ttt_workspace_bytes(int T, int d_ff, int d_model, int C);

/* In-Place TTT forward of the W_down fast weight (one sequence); page "In-Place Test-Time
 * Training", section "核心方法和技术细节".
 *  Z     [T, d_ff]      bf16   (the gated-MLP activation phi(H W_gate^T) * (H W_up^T))
 *  Vhat  [T, d_model]   bf16   (the update target)
 *  W     [d_model, d_ff] float32, in: W_down at token 0, out: W_down after the last chunk
 *  O     [T, d_model]   bf16   out: O_i = Z_i W_i^T (apply, then update: no intra-chunk term)
 *  W_chunks [T/C, d_model, d_ff] bf16, nullable; out: W_i, the weight chunk i applied (what
 *        inplace_ttt_bwd reads; 2 bytes per weight per chunk)
 * Requirements: T % C == 0, C % 128 == 0, d_ff % 64 == 0, d_model % 128 == 0. */
ttt_status inplace_ttt_fwd(int T, int d_ff, int d_model, int C, float lr, const void* Z,
                           const void* Vhat, float* W, void* O, void* W_chunks, void* workspace,
                           size_t workspace_bytes, void* stream);

/* Document resets (page "In-Place Test-Time Training", section "实践建议": the fast weight is
 * reset at document boundaries so that no information leaks across documents). Same as
 * inplace_ttt_fwd / inplace_ttt_bwd with a HOST array doc_starts of n_docs chunk indices
 * (strictly increasing, each in [1, T/C - 1]) where a new document begins: that chunk applies,
 * and its update starts from, the initial W_down (the W passed in). W_final is the last
 * document's end state; the backward's adjoint does not cross a boundary and dW sums the
 * adjoints reaching every document start. Boundaries fall on chunk starts (pack or pad
 * documents to multiples of C). Workspace from inplace_ttt_docs_workspace_bytes (one float32
 * d_model x d_ff matrix more). A malformed list returns TTT_ERR_INVALID_ARG. */
size_t inplace_ttt_docs_workspace_bytes(int T, int d_ff, int d_model, int C);
ttt_status inplace_ttt_fwd_docs(int T, int d_ff, int d_model, int C, float lr, const void* Z,
                                const void* Vhat, float* W, void* O, void* W_chunks,
                                const int* doc_starts, int n_docs, void* workspace,
                                size_t workspace_bytes, void* stream);
ttt_status inplace_ttt_bwd_docs(int T, int d_ff, int d_model, int C, float lr, const void* Z,
                                const void* Vhat, const void* W_chunks, const void* dO,
                                const float* dW_final, void* dZ, void* dVhat, float* dW,
                                const int* doc_starts, int n_docs, void* workspace,
                                size_t workspace_bytes, void* stream);

/* Context-parallel building blocks (page "In-Place Test-Time Training", section "核心方法和技术
 * 细节": the update is associative, so a sequence split across devices runs as a parallel scan):
 * with the sequence cut into shards, shard g starts from W_0 + sum_{h<g} dW_h where
 *     dW_h = lr Vhat_h^T Z_h     (inplace_ttt_delta: every chunk update of shard h, summed)
 * and then runs inplace_ttt_fwd on its own tokens. The exchange of the dW_h between devices is
 * the caller's (the Python binding's inplace_cp_fwd uses torch.distributed); ttt_add_f32 adds
 * them on the device.
 *  Z [T, d_ff], Vhat [T, d_model] bf16; dW [d_model, d_ff] float32 out (plain stores).
 *  Requirements: T % 128 == 0, d_ff % 64 == 0, d_model % 128 == 0; workspace >= 256 bytes. */
ttt_status inplace_ttt_delta(int T, int d_ff, int d_model, float lr, const void* Z,
                             const void* Vhat, float* dW, void* workspace, size_t workspace_bytes,
                             void* stream);
/* dst[i] += src[i] over n float32 (device pointers, n % 4 == 0). */
ttt_status ttt_add_f32(float* dst, const float* src, size_t n, void* stream);

/* Workspace bytes of inplace_ttt_target; (size_t)-1 for invalid sizes. */
size_t inplace_ttt_target_workspace_bytes(int T, int d_model);

/* NTP-aligned update target of In-Place TTT (page "In-Place Test-Time Training", section
 * "核心方法和技术细节": Vhat = Conv1D(X0) W_target, the convolution extracting nearby future
 * tokens of the embeddings). Reading: a depthwise convolution over the current and the next
 * k - 1 tokens, zero past the last token, then the projection with row vectors:
 *     Y_t = sum_{j<k} conv_w[j] * X0_{t+j}   (per channel),   Vhat = Y W_target.
 *  X0        [T, d_model]       bf16     token embeddings
 *  conv_w    [k, d_model]       float32  tap j weights token t + j
 *  W_target  [d_model, d_model] bf16     input rows, output columns
 *  Vhat      [T, d_model]       bf16     out (the Vhat of inplace_ttt_fwd)
 * Requirements: T % 128 == 0, d_model % 128 == 0, 1 <= k <= 8. Y is rounded to bf16 before
 * the projection. */
ttt_status inplace_ttt_target(int T, int d_model, int k, const void* X0, const float* conv_w,
                              const void* W_target, void* Vhat, void* workspace,
                              size_t workspace_bytes, void* stream);

/* Workspace bytes of inplace_ttt_target_bwd; (size_t)-1 for invalid sizes. */
size_t inplace_ttt_target_bwd_workspace_bytes(int T, int d_model, int k);

/* Backward of inplace_ttt_target for J = <dVhat, Vhat> (the page gives only the forward):
 *     dY = dVhat W_target^T,  dW_target = Y^T dVhat,
 *     dX0_t = sum_{j<k, t-j>=0} conv_w[j] * dY_{t-j},  dconv_w[j] = sum_t dY_t * X0_{t+j}.
 *  in : X0, conv_w, W_target as in the forward; dVhat [T, d_model] bf16
 *  out: dX0 [T, d_model] bf16, dconv_w [k, d_model] float32, dW_target [d_model, d_model]
 *       float32 (plain stores). Y is recomputed (in bf16); requirements as the forward. */
ttt_status inplace_ttt_target_bwd(int T, int d_model, int k, const void* X0, const float* conv_w,
                                  const void* W_target, const void* dVhat, void* dX0,
                                  float* dconv_w, float* dW_target, void* workspace,
                                  size_t workspace_bytes, void* stream);

/* Backward of inplace_ttt_fwd (no counterpart on the page, which gives only the forward): the
 * reverse-mode of the apply-then-update loop for J = sum_i <dO_i, O_i> + <dW_final, W_final>.
 * With Wh the adjoint of the fast weight (dW_final, or 0, after the last chunk), chunk i from
 * the last one down gives
 *     dVhat_i = lr Z_i Wh_{i+1}^T,  dZ_i = dO_i W_i + lr Vhat_i Wh_{i+1},  Wh_i = Wh_{i+1} + dO_i^T Z_i.
 *  in : Z, Vhat as in the forward; W_chunks from inplace_ttt_fwd (required); dO [T, d_model]
 *       bf16; dW_final [d_model, d_ff] float32 (nullable = 0)
 *  out: dZ [T, d_ff] bf16, dVhat [T, d_model] bf16, dW [d_model, d_ff] float32 = Wh_0, the
 *       gradient of the initial W_down (plain stores)
 * Requirements as inplace_ttt_fwd; workspace from inplace_ttt_workspace_bytes. */
ttt_status inplace_ttt_bwd(int T, int d_ff, int d_model, int C, float lr, const void* Z,
                           const void* Vhat, const void* W_chunks, const void* dO,
                           const float* dW_final, void* dZ, void* dVhat, float* dW,
                           void* workspace, size_t workspace_bytes, void* stream);

/* Synchronises `stream`, then returns TTT_ERR_TIMEOUT if any kernel of this library on the
 * current device recorded a bounded wait that ran out since the last call, else TTT_ERR_RANGE
 * if one recorded an input outside its range (and clears the word), TTT_ERR_CUDA if the stream
 * reports an error, else TTT_OK. */
ttt_status ttt_get_device_error(void* stream);

/* Launches a one-warp kernel whose wait on an mbarrier that nothing completes is bounded
 * by `spin_limit` polls; it must end by recording a timeout in the device error word.
 * Used to test the failure path without faulting the GPU. */
ttt_status ttt_selftest_bounded_wait(unsigned spin_limit, void* stream);

/* Number of kernels this library has launched in this process (all devices, all entry
 * points) since it was loaded. Lets a caller check what ran without a profiler. */
unsigned long long ttt_kernel_launches(void);

/* Static description of a status code. */
const char* ttt_status_string(ttt_status s);

#ifdef __cplusplus
}
#endif
#endif /* TTT_H_ */
