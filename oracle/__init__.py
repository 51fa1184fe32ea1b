"""CPU oracle for the chunkwise TTT layer and In-Place TTT.

TEST INFRASTRUCTURE ONLY: only tests/, __graft_entry__.smoke() and bench.py's
cpu_baseline / reference leg may import this package. The product library
(weight_sequence_layers_b200) never imports it and shares no code with it.

* ttt_fwd / ttt_bwd call the C++ per-token state evolver in ttt_oracle.cpp
  (fp64 state and arithmetic; ttt_fwd_f32 is the fp32-state build).
* inplace_fwd follows In-Place TTT (page "In-Place Test-Time Training",
  section "核心方法和技术细节", the chunkwise apply-then-update rule
  W^(i+1) = W^(i) + eta * Vhat_[i]^T Z_[i]) with fp64 numpy matmuls;
  inplace_bwd is the reverse-mode of that loop (the pages print no backward),
  inplace_bwd_dz_tokens evaluates sampled rows of its dZ at any size;
  inplace_target is the NTP-aligned target Vhat = Conv1D(X0) W_target of the same
  section, with its reverse-mode inplace_target_bwd.

Every function here is pinned by tests/test_oracle_pins.py; no function is
"parity unpinned" except for absolute agreement with the authors' own
implementation, which the pages neither ship nor print values of.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ttt_oracle.cpp")
_LIB = os.path.join(_HERE, "libttt_oracle.so")
_lib = None

LOSS = {"mse": 0, "ip": 1}
ACT = {"id": 0, "silu": 1}


def build(force: bool = False) -> str:
    """Compile the oracle shared library in-tree (g++ -O2 -fopenmp)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["g++", "-O2", "-std=c++17", "-fPIC", "-shared", "-fopenmp", _SRC, "-o", _LIB]
        subprocess.run(cmd, check=True)
    return _LIB


def open_library(path: str):
    """A build of ttt_oracle.cpp at `path`, with the C signatures of its entry points."""
    lib = ctypes.CDLL(path)
    d, i = ctypes.c_double, ctypes.c_int
    p = ctypes.c_void_p
    lib.ttt_oracle_fwd_f64.argtypes = [i] * 8 + [d, i] + [p] * 9 + [i]
    lib.ttt_oracle_fwd_f32.argtypes = [i] * 8 + [d, i] + [p] * 9 + [i]
    lib.ttt_oracle_bwd_f64.argtypes = [i] * 8 + [d, i] + [p] * 14 + [i]
    for fn in (lib.ttt_oracle_fwd_f64, lib.ttt_oracle_fwd_f32, lib.ttt_oracle_bwd_f64):
        fn.restype = i
    return lib


def _load():
    global _lib
    if _lib is None:
        build()
        _lib = open_library(_LIB)
    return _lib


def _np(x, dtype):
    """torch tensor or array -> C-contiguous numpy array of `dtype` (exact upcast)."""
    if x is None:
        return None
    if hasattr(x, "detach"):
        x = x.detach().to("cpu").float().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=dtype))


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _gvec(g, q):
    """1 when gamma carries one decay per key feature ([B,H,T,dk]), 0 for [B,H,T] or None."""
    if g is None:
        return 0
    if g.shape == q.shape:
        return 1
    if g.shape != q.shape[:3]:
        raise ValueError("gamma must be [B,H,T] or [B,H,T,dk]")
    return 0


def ttt_fwd(Q, K, V, beta, gamma, W0, *, C: int, loss: str = "mse", act: str = "id",
            lr_bias: float, nthreads: int = 0, state: str = "f64"):
    """Per-token fast-weight evolution of the chunkwise TTT layer (page "Modular TTT:
    Rethinking Test-Time Training as Composable Modules", section "方法步骤详情", Algorithm 1,
    with the learning rate of section "内部学习规则与学习率参数化" and the decay of section
    "权重衰减"), run by ttt_oracle.cpp. Returns (O, W_final, W_chunks, threads_used).

    Q, K: [B,H,T,dk]; V: [B,H,T,dv]; beta: [B,H,T]; gamma: [B,H,T] (scalar decay),
    [B,H,T,dk] (per-feature decay of the rows of W) or None (no decay);
    W0: [B,H,dk,dv]. state="f64" (parity) or "f32" (fp32 state, timed baseline).
    """
    lib = _load()
    dt = np.float64 if state == "f64" else np.float32
    q, k, v = _np(Q, dt), _np(K, dt), _np(V, dt)
    b_, g_, w0 = _np(beta, dt), _np(gamma, dt), _np(W0, dt)
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    if T % C:
        raise ValueError("T must be a multiple of C")
    o = np.empty((B, H, T, dv), dt)
    wf = np.empty((B, H, dk, dv), dt)
    wc = np.empty((B, H, T // C, dk, dv), dt)
    fn = lib.ttt_oracle_fwd_f64 if state == "f64" else lib.ttt_oracle_fwd_f32
    used = fn(B, H, T, dk, dv, C, LOSS[loss], ACT[act], float(lr_bias), _gvec(g_, q), _ptr(q),
              _ptr(k), _ptr(v),
              _ptr(b_), _ptr(g_), _ptr(w0), _ptr(o), _ptr(wf), _ptr(wc), int(nthreads))
    if used < 0:
        raise ValueError("oracle rejected the shape")
    return o, wf, wc, used


def ttt_bwd(Q, K, V, beta, gamma, W0, dO, dW_T=None, *, C: int, loss: str = "mse",
            act: str = "id", lr_bias: float, nthreads: int = 0):
    """Reverse-mode of ttt_fwd's per-token loop for J = <dO,O> + <dW_T,W_final> (fp64), run by
    ttt_oracle.cpp. The page (section "技术新颖性") hand-derives analytic backward operators
    without printing them; this is the plain reverse-mode of the forward it follows.
    Returns dict dQ, dK, dV, dbeta, dW0, and dgamma (shaped like gamma) when gamma is given."""
    lib = _load()
    dt = np.float64
    q, k, v = _np(Q, dt), _np(K, dt), _np(V, dt)
    b_, g_, w0 = _np(beta, dt), _np(gamma, dt), _np(W0, dt)
    do, dwt = _np(dO, dt), _np(dW_T, dt)
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    if T % C:
        raise ValueError("T must be a multiple of C")
    out = dict(dQ=np.empty((B, H, T, dk)), dK=np.empty((B, H, T, dk)),
               dV=np.empty((B, H, T, dv)), dbeta=np.empty((B, H, T)),
               dW0=np.empty((B, H, dk, dv)))
    if g_ is not None:
        out["dgamma"] = np.empty(g_.shape)
    used = lib.ttt_oracle_bwd_f64(B, H, T, dk, dv, C, LOSS[loss], ACT[act], float(lr_bias),
                                  _gvec(g_, q), _ptr(q), _ptr(k), _ptr(v), _ptr(b_), _ptr(g_), _ptr(w0),
                                  _ptr(do), _ptr(dwt), _ptr(out["dQ"]), _ptr(out["dK"]),
                                  _ptr(out["dV"]), _ptr(out["dbeta"]), _ptr(out["dW0"]),
                                  _ptr(out.get("dgamma")), int(nthreads))
    if used < 0:
        raise ValueError("oracle rejected the shape")
    return out


def inplace_fwd(Z, Vhat, W, *, C: int, lr: float, rows=None, doc_starts=()):
    """In-Place TTT W_down forward, apply-then-update per chunk (fp64).

    Z: [T, d_ff]; Vhat: [T, d_model]; W: [d_model, d_ff] (the fast weight W_down).
    For chunk i: O_i = Z_i W_i^T, then W_{i+1} = W_i + lr * Vhat_i^T Z_i.
    `rows` (optional index array into d_model) restricts the computation to
    those rows of W (and columns of O and Vhat): the rows evolve independently,
    so the restricted result is exact. `doc_starts`: chunk indices where a new
    document begins (section "实践建议": the fast weight is reset at document
    boundaries); its first chunk applies the initial W again. Returns
    (O[:, rows], W_final[rows]).
    """
    z = _np(Z, np.float64)
    vh = _np(Vhat, np.float64)
    w = _np(W, np.float64)
    if rows is not None:
        rows = np.asarray(rows)
        vh = vh[:, rows]
        w = w[rows]
    w0 = w.copy()
    w = w.copy()
    T = z.shape[0]
    if T % C:
        raise ValueError("T must be a multiple of C")
    o = np.empty((T, w.shape[0]))
    starts = set(doc_starts)
    for i in range(T // C):
        if i in starts:
            w = w0.copy()  # a new document starts from the initial fast weight
        zi = z[i * C:(i + 1) * C]
        o[i * C:(i + 1) * C] = zi @ w.T          # apply with the current fast weight
        w += lr * (vh[i * C:(i + 1) * C].T @ zi)  # then update it with this chunk
    return o, w


def inplace_bwd(Z, Vhat, W, dO, dW_final=None, *, C: int, lr: float, rows=None, doc_starts=()):
    """Reverse-mode of inplace_fwd for J = sum_i <dO_i, O_i> + <dW_final, W_final> (fp64).

    The chunks are walked backwards carrying Wh, the adjoint of the fast weight (dW_final, or
    zero, after the last chunk). With W_i the weight chunk i applied:
        O_i = Z_i W_i^T                  gives  dZ_i += dO_i W_i,           Wh += dO_i^T Z_i
        W_{i+1} = W_i + lr Vhat_i^T Z_i  gives  dZ_i += lr Vhat_i Wh_{i+1},  dVhat_i = lr Z_i Wh_{i+1}^T
    (Wh_{i+1} is the adjoint before chunk i's own O_i term is added). Returns dict dZ [T, d_ff],
    dVhat [T, d_model] and dW [d_model, d_ff], the gradient with respect to the initial W.
    With `doc_starts` (see inplace_fwd) a document's first chunk applied the initial W, so the
    adjoint reaching it joins dW and the previous document's end state gets no adjoint.
    `rows` restricts the computation to those rows of W (columns of Vhat and dO): dVhat[:, rows]
    and dW[rows] are then exact, and dZ, a sum over every row, is not returned (None).
    """
    z = _np(Z, np.float64)
    vh = _np(Vhat, np.float64)
    w = _np(W, np.float64)
    do = _np(dO, np.float64)
    dwf = np.zeros_like(w) if dW_final is None else _np(dW_final, np.float64)
    if rows is not None:
        rows = np.asarray(rows)
        vh, do, w, dwf = vh[:, rows], do[:, rows], w[rows], dwf[rows]
    T = z.shape[0]
    if T % C:
        raise ValueError("T must be a multiple of C")
    starts = set(doc_starts)
    applied = []
    cur = w.copy()
    for i in range(T // C):
        sl = slice(i * C, (i + 1) * C)
        if i in starts:
            cur = w.copy()
        applied.append(cur.copy())
        cur = cur + lr * (vh[sl].T @ z[sl])
    wh = dwf.copy()
    dw = np.zeros_like(w)
    dz = np.zeros_like(z) if rows is None else None
    dvh = np.zeros_like(vh)
    for i in reversed(range(T // C)):
        sl = slice(i * C, (i + 1) * C)
        if dz is not None:
            dz[sl] = do[sl] @ applied[i] + lr * (vh[sl] @ wh)
        dvh[sl] = lr * (z[sl] @ wh.T)
        wh = wh + do[sl].T @ z[sl]
        if i in starts or i == 0:
            dw = dw + wh              # this document's start state is the initial W
            wh = np.zeros_like(wh)    # the previous document's end state is discarded
    return dict(dZ=dz, dVhat=dvh, dW=dw)


def inplace_bwd_dz_tokens(Z, Vhat, W, dO, dW_final=None, *, C: int, lr: float, tokens):
    """Rows `tokens` of dZ from inplace_bwd, by expanding both sums (fp64): for token t of
    chunk i, W_i = W + lr Vhat_{<i}^T Z_{<i} and Wh_{i+1} = dW_final + dO_{>i}^T Z_{>i} (<i: the
    tokens of the chunks before i, >i: after it), so
        dZ_t = dO_t W + lr (dO_t Vhat_{<i}^T) Z_{<i} + lr Vhat_t dW_final + lr (Vhat_t dO_{>i}^T) Z_{>i}.
    Cheap for a few tokens at any size: no d_model x d_ff product is formed."""
    z = _np(Z, np.float64)
    vh = _np(Vhat, np.float64)
    w = _np(W, np.float64)
    do = _np(dO, np.float64)
    out = np.empty((len(tokens), z.shape[1]))
    for n, t in enumerate(tokens):
        i = t // C
        lo, hi = i * C, (i + 1) * C
        row = do[t] @ w + lr * ((vh[:lo] @ do[t]) @ z[:lo])
        if dW_final is not None:
            row = row + lr * (vh[t] @ _np(dW_final, np.float64))
        row = row + lr * ((do[hi:] @ vh[t]) @ z[hi:])
        out[n] = row
    return out


def inplace_target(X0, conv_w, W_target):
    """NTP-aligned target of In-Place TTT (page "In-Place Test-Time Training", section
    "核心方法和技术细节": Vhat = Conv1D(X0) W_target, the convolution reading nearby future
    tokens), in fp64. Reading: a depthwise convolution over the current and the next k - 1
    tokens, Y_t = sum_{j<k} conv_w[j] * X0_{t+j} (per channel, zero past the last token), then
    Vhat = Y W_target with row vectors.
    X0: [T, d]; conv_w: [k, d]; W_target: [d, d_out]. Returns (Vhat [T, d_out], Y [T, d])."""
    x = _np(X0, np.float64)
    w = _np(conv_w, np.float64)
    wt = _np(W_target, np.float64)
    T = x.shape[0]
    y = np.zeros_like(x)
    for j in range(w.shape[0]):
        y[: T - j] += w[j] * x[j:]
    return y @ wt, y


def inplace_target_bwd(X0, conv_w, W_target, dVhat, channels=None):
    """Reverse-mode of inplace_target for J = <dVhat, Vhat> (fp64): returns dict dX0 [T, d],
    dconv_w [k, d] and dW_target [d, d_out]. `channels` (index array into d) restricts all
    three to those input channels (columns of dX0 and dconv_w, rows of dW_target); every
    channel's gradients depend only on its own column of X0 and conv_w and its row of W_target,
    so the restricted result is exact."""
    x = _np(X0, np.float64)
    w = _np(conv_w, np.float64)
    wt = _np(W_target, np.float64)
    dv = _np(dVhat, np.float64)
    if channels is not None:
        channels = np.asarray(channels)
        x, w, wt = x[:, channels], w[:, channels], wt[channels]
    _, y = inplace_target(x, w, wt)
    dy = dv @ wt.T
    T = x.shape[0]
    dx = np.zeros_like(x)
    dw = np.zeros_like(w)
    for j in range(w.shape[0]):
        dx[j:] += w[j] * dy[: T - j]
        dw[j] = (dy[: T - j] * x[j:]).sum(axis=0)
    return dict(dX0=dx, dconv_w=dw, dW_target=y.T @ dv)


# --------------------------------------------------------------------------------- TTT-MLP
def _act_t(act, z):
    import torch
    return z * torch.sigmoid(z) if act == "silu" else z


def ttt_mlp_fwd(Q, K, V, beta, gamma, W1, W2, *, C: int, loss: str = "mse", act: str = "silu",
                lr_bias: float, keep_graph: bool = False):
    """TTT-MLP: the fast weight is a two-layer network vhat = act(k W1) W2 (page "Modular TTT:
    Rethinking Test-Time Training as Composable Modules": TTT-MLP, the two-layer fast weight of
    its throughput table; deeper learners factor an effective W = W1 W2), evolved per token in
    fp64 on the CPU with plain PyTorch ops. Readings, as for the single Linear: both layers
    decay by gamma_t and take one gradient step with eta_t = 2 sigmoid(beta_t + b); every
    gradient of a chunk is taken at the chunk-start weights (W1_0, W2_0); the token reads its own
    write, o_t = act(q_t W1_t) W2_t; MSE is 1/2 ||vhat - v||^2, IP is -<vhat, v>.
    Per token t of a chunk:
        z = k W1_0, a = act(z), vhat = a W2_0, g2 = vhat - v (MSE) or -v (IP),
        g1 = (g2 W2_0^T) * act'(z),
        W1 <- gamma W1 - eta k^T g1,   W2 <- gamma W2 - eta a^T g2,   o = act(q W1) W2.
    Q, K: [B,H,T,dk]; V: [B,H,T,dv]; beta, gamma: [B,H,T] (gamma None: no decay);
    W1: [B,H,dk,h]; W2: [B,H,h,dv]. Returns (O, W1_final, W2_final) as torch fp64 tensors
    (with keep_graph, still attached to the autograd graph of the inputs)."""
    import torch
    t = lambda x: x if isinstance(x, torch.Tensor) and x.dtype == torch.float64 and x.device.type == "cpu" \
        else torch.as_tensor(np.asarray(_np(x, np.float64)), dtype=torch.float64)
    q, k, v, b, w1, w2 = t(Q), t(K), t(V), t(beta), t(W1), t(W2)
    g = None if gamma is None else t(gamma)
    B, H, T, _ = q.shape
    if T % C:
        raise ValueError("T must be a multiple of C")
    outs, w1f, w2f = [], [], []
    for bi in range(B):
        ob, w1b, w2b = [], [], []
        for hi in range(H):
            A, Bw = w1[bi, hi], w2[bi, hi]
            orows = []
            for c in range(T // C):
                A0, B0 = A, Bw
                for s_ in range(C):
                    tt = c * C + s_
                    kt, qt, vt = k[bi, hi, tt], q[bi, hi, tt], v[bi, hi, tt]
                    eta = 2 * torch.sigmoid(b[bi, hi, tt] + lr_bias)
                    gam = 1.0 if g is None else g[bi, hi, tt]
                    z = kt @ A0
                    a = _act_t(act, z)
                    vh = a @ B0
                    g2 = vh - vt if loss == "mse" else -vt
                    if act == "silu":
                        sg = torch.sigmoid(z)
                        d1 = sg * (1 + z * (1 - sg))
                    else:
                        d1 = torch.ones_like(z)
                    g1 = (B0 @ g2) * d1
                    A = gam * A - eta * torch.outer(kt, g1)
                    Bw = gam * Bw - eta * torch.outer(a, g2)
                    orows.append(_act_t(act, qt @ A) @ Bw)
            ob.append(torch.stack(orows))
            w1b.append(A)
            w2b.append(Bw)
        outs.append(torch.stack(ob))
        w1f.append(torch.stack(w1b))
        w2f.append(torch.stack(w2b))
    O, W1f, W2f = torch.stack(outs), torch.stack(w1f), torch.stack(w2f)
    if not keep_graph:
        O, W1f, W2f = O.detach(), W1f.detach(), W2f.detach()
    return O, W1f, W2f


def ttt_mlp_bwd(Q, K, V, beta, gamma, W1, W2, dO, dW1_T=None, dW2_T=None, *, C: int,
                loss: str = "mse", act: str = "silu", lr_bias: float):
    """Gradients of J = <dO, O> + <dW1_T, W1_final> + <dW2_T, W2_final> through ttt_mlp_fwd's
    per-token loop, by reverse-mode automatic differentiation of the fp64 CPU loop (a library
    primitive standing in for the hand derivation). Returns numpy fp64 dQ, dK, dV, dbeta,
    dW1 (initial W1), dW2 (initial W2), and dgamma when gamma is given."""
    import torch
    names = ["Q", "K", "V", "beta", "W1", "W2"] + (["gamma"] if gamma is not None else [])
    vals = dict(Q=Q, K=K, V=V, beta=beta, W1=W1, W2=W2, gamma=gamma)
    leaves = {n: torch.as_tensor(np.asarray(_np(vals[n], np.float64)), dtype=torch.float64).requires_grad_(True)
              for n in names}
    O, W1f, W2f = ttt_mlp_fwd(leaves["Q"], leaves["K"], leaves["V"], leaves["beta"],
                              leaves.get("gamma"), leaves["W1"], leaves["W2"], C=C, loss=loss,
                              act=act, lr_bias=lr_bias, keep_graph=True)
    J = (O * torch.as_tensor(_np(dO, np.float64))).sum()
    if dW1_T is not None:
        J = J + (W1f * torch.as_tensor(_np(dW1_T, np.float64))).sum()
    if dW2_T is not None:
        J = J + (W2f * torch.as_tensor(_np(dW2_T, np.float64))).sum()
    grads = torch.autograd.grad(J, [leaves[n] for n in names])
    key = dict(Q="dQ", K="dK", V="dV", beta="dbeta", W1="dW1", W2="dW2", gamma="dgamma")
    return {key[n]: gr.numpy() for n, gr in zip(names, grads)}
