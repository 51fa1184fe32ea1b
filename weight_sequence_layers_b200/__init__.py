"""Python binding of the B200 chunkwise-TTT library (libttt.so, C ABI in include/ttt.h).

Argument marshalling only: every function here forwards torch tensors' device pointers,
sizes and the current CUDA stream to the C entry point of the same name and raises
TTTError on a non-OK status. Every step of the computation runs in the library's CUDA
kernels; there is no fallback of any kind. Importing fails loudly if libttt.so has not
been built (python weight_sequence_layers_b200/build.py).
"""
from __future__ import annotations

import ctypes
import os
import re

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libttt.so")
HEADER = os.path.join(os.path.dirname(_PKG), "include", "ttt.h")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with python weight_sequence_layers_b200/build.py")

_lib = ctypes.CDLL(LIB_PATH)

(OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_ALIGNMENT, ERR_WORKSPACE, ERR_CUDA, ERR_TIMEOUT,
 ERR_RANGE) = range(8)
F32, BF16 = 0, 1
LOSS = {"mse": 0, "ip": 1}
ACT = {"id": 0, "silu": 1}
DECAY = {"scalar": 0, "vector": 1}


class TTTError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} ({status})")


class ttt_config(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("T", ctypes.c_int),
                ("dk", ctypes.c_int), ("dv", ctypes.c_int), ("C", ctypes.c_int),
                ("dtype", ctypes.c_int), ("loss", ctypes.c_int), ("act", ctypes.c_int),
                ("lr_bias", ctypes.c_float), ("decay", ctypes.c_int),
                ("w0_shared", ctypes.c_int)]


_p, _i, _u, _f, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_uint, ctypes.c_float, ctypes.c_size_t
_cfgp = ctypes.POINTER(ttt_config)
_SIGS = {
    "ttt_workspace_bytes": ([_cfgp, _i], _sz),
    "ttt_saved_bytes": ([_cfgp], _sz),
    "ttt_chunk_fwd": ([_cfgp] + [_p] * 11 + [_sz, _p], _i),
    "ttt_chunk_bwd": ([_cfgp] + [_p] * 19 + [_sz, _p], _i),
    "inplace_ttt_workspace_bytes": ([_i] * 4, _sz),
    "ttt_mlp_workspace_bytes": ([_cfgp, _i], _sz),
    "ttt_mlp_fwd": ([_cfgp, _i] + [_p] * 13 + [_sz, _p], _i),
    "ttt_mlp_bwd": ([_cfgp, _i] + [_p] * 17 + [_sz, _p], _i),
    "inplace_ttt_fwd": ([_i] * 4 + [_f] + [_p] * 6 + [_sz, _p], _i),
    "inplace_ttt_bwd": ([_i] * 4 + [_f] + [_p] * 9 + [_sz, _p], _i),
    "inplace_ttt_target_workspace_bytes": ([_i] * 2, _sz),
    "inplace_ttt_docs_workspace_bytes": ([_i] * 4, _sz),
    "inplace_ttt_delta": ([_i] * 3 + [_f] + [_p] * 4 + [_sz, _p], _i),
    "ttt_add_f32": ([_p, _p, _sz, _p], _i),
    "inplace_ttt_fwd_docs": ([_i] * 4 + [_f] + [_p] * 6 + [_i, _p, _sz, _p], _i),
    "inplace_ttt_bwd_docs": ([_i] * 4 + [_f] + [_p] * 9 + [_i, _p, _sz, _p], _i),
    "inplace_ttt_target": ([_i] * 3 + [_p] * 5 + [_sz, _p], _i),
    "inplace_ttt_target_bwd_workspace_bytes": ([_i] * 3, _sz),
    "inplace_ttt_target_bwd": ([_i] * 3 + [_p] * 8 + [_sz, _p], _i),
    "ttt_get_device_error": ([_p], _i),
    "ttt_selftest_bounded_wait": ([_u, _p], _i),
    "ttt_status_string": ([_i], ctypes.c_char_p),
    "ttt_kernel_launches": ([], ctypes.c_ulonglong),
    "ttt_chunk_bwd_noalloc": ([_cfgp] + [_p] * 18 + [_p], _i),
}
for _name, (_args, _ret) in _SIGS.items():
    _fn = getattr(_lib, _name)
    _fn.argtypes = _args
    _fn.restype = _ret


def header_functions() -> list[str]:
    """Names of the functions include/ttt.h declares."""
    text = open(HEADER).read()
    # a declaration starts in column 0 with its return type (one or more words, pointers
    # included), then the name and "("; comments, macros and continuation lines do not
    return re.findall(r"^(?!typedef\b)(?:[A-Za-z_]\w*[ \t\*]+)+([A-Za-z_]\w*)\s*\(", text,
                      flags=re.M)


def status_string(status: int) -> str:
    return _lib.ttt_status_string(int(status)).decode()


def _ptr(t):
    """Device address of a tensor argument; None and raw integer addresses pass through.

    The library reads and writes every array argument as a dense row-major array on the
    current CUDA device. A strided view, a host tensor or a tensor on another device would
    give wrong results or a memory fault, so they are refused here, before any library call.
    """
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_contiguous():
        raise ValueError("tensor arguments must be contiguous (dense row-major, no strided views)")
    if not t.is_cuda:
        raise ValueError("tensor arguments must be CUDA tensors: the library takes device pointers")
    import torch
    if t.device.index != torch.cuda.current_device():
        raise ValueError(f"tensor on {t.device}, but the library runs on the current device "
                         f"cuda:{torch.cuda.current_device()}")
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(status: int, where: str):
    if status != OK:
        raise TTTError(status, where)


def make_config(B, H, T, dk, dv, C, dtype="bf16", loss="mse", act="id", lr_bias=0.0,
                decay="scalar", w0_shared=False) -> ttt_config:
    """decay: "scalar" (gamma [B,H,T], or no gamma) or "vector" (gamma [B,H,T,dk]).
    w0_shared: W0 (W1_0, W2_0 for TTT-MLP) is [H, ...], one initial state per head shared by
    the batch, instead of [B, H, ...]."""
    return ttt_config(B, H, T, dk, dv, C, F32 if dtype in ("f32", F32) else BF16,
                      LOSS.get(loss, loss), ACT.get(act, act), float(lr_bias),
                      DECAY.get(decay, decay), int(bool(w0_shared)))


def ttt_saved_bytes(cfg: ttt_config) -> int:
    """Bytes of the forward's G_saved buffer (G, and Zq with SiLU)."""
    n = _lib.ttt_saved_bytes(ctypes.byref(cfg))
    if n == ctypes.c_size_t(-1).value:
        raise TTTError(ERR_INVALID_ARG, "ttt_saved_bytes")
    return n


def ttt_workspace_bytes(cfg: ttt_config, for_bwd: int) -> int:
    """for_bwd: 0 forward, 1 backward without G_saved, 2 backward given G_saved."""
    n = _lib.ttt_workspace_bytes(ctypes.byref(cfg), int(for_bwd))
    if n == ctypes.c_size_t(-1).value:
        raise TTTError(ERR_INVALID_ARG, "ttt_workspace_bytes")
    return n


def _check_size(t, nbytes: int, name: str):
    """A buffer the library fills or reads for this config must hold nbytes; the C ABI cannot
    tell, and a short buffer would be written past its end."""
    if t is not None and not isinstance(t, int) and t.numel() * t.element_size() < nbytes:
        raise ValueError(f"{name} holds {t.numel() * t.element_size()} bytes, the config needs "
                         f"{nbytes}")


def _chunks_bytes(cfg) -> int:
    return cfg.B * cfg.H * (cfg.T // cfg.C) * cfg.dk * cfg.dv * (2 if cfg.dtype == BF16 else 4)


def ttt_chunk_fwd(cfg, Q, K, V, beta, gamma, W0, O, W_final=None, W_chunks=None, G_saved=None,
                  workspace=None, workspace_bytes=0, stream=None):
    """Forward of the chunkwise TTT layer on the current device and stream.

    Q, K [B,H,T,dk]; V, O [B,H,T,dv] in cfg's dtype; beta [B,H,T] and W0, W_final [B,H,dk,dv]
    float32; gamma [B,H,T] or [B,H,T,dk] float32, or None (no decay). W_chunks
    [B,H,T/C,dk,dv] in cfg's dtype and G_saved (ttt_saved_bytes) are optional outputs that
    ttt_chunk_bwd reads. Workspace: ttt_workspace_bytes(cfg, 0) bytes. Raises TTTError on a
    non-OK status."""
    if G_saved is not None:
        _check_size(G_saved, ttt_saved_bytes(cfg), "G_saved")
    if W_chunks is not None:
        _check_size(W_chunks, _chunks_bytes(cfg), "W_chunks")
    st = _lib.ttt_chunk_fwd(ctypes.byref(cfg), _ptr(Q), _ptr(K), _ptr(V), _ptr(beta), _ptr(gamma),
                            _ptr(W0), _ptr(O), _ptr(W_final), _ptr(W_chunks), _ptr(G_saved),
                            _ptr(workspace), int(workspace_bytes), _stream(stream))
    _check(st, "ttt_chunk_fwd")


def ttt_chunk_bwd(cfg, Q, K, V, beta, gamma, W0, W_chunks, G_saved, dO, dW_final, O, W_final, dQ,
                  dK, dV, dbeta, dW0, dgamma, workspace=None, workspace_bytes=0, stream=None):
    """Analytic backward of the layer for J = <dO, O> + <dW_final, W_final>.

    Takes the forward's inputs, its W_chunks and (optionally) G_saved, dO and dW_final (or
    None), and writes dQ, dK, dV, dbeta, dW0 and, when dgamma is given, the decay gradient
    (which also needs the forward's O, and W_final when dW_final is given). Workspace:
    ttt_workspace_bytes(cfg, 2 if G_saved is passed else 1) bytes."""
    if G_saved is not None:
        _check_size(G_saved, ttt_saved_bytes(cfg), "G_saved")
    st = _lib.ttt_chunk_bwd(ctypes.byref(cfg), _ptr(Q), _ptr(K), _ptr(V), _ptr(beta), _ptr(gamma),
                            _ptr(W0), _ptr(W_chunks), _ptr(G_saved), _ptr(dO), _ptr(dW_final),
                            _ptr(O), _ptr(W_final), _ptr(dQ), _ptr(dK), _ptr(dV), _ptr(dbeta),
                            _ptr(dW0), _ptr(dgamma), _ptr(workspace), int(workspace_bytes),
                            _stream(stream))
    _check(st, "ttt_chunk_bwd")


NOALLOC_SCRATCH_BYTES = 8 << 20


def ttt_chunk_bwd_noalloc(cfg, Q, K, V, beta, gamma, W0, W_chunks, G_saved, dO, dW_final, O,
                          W_final, dQ, dK, dV, dbeta, dW0, dgamma, stream=None):
    """ttt_chunk_bwd for callers that cannot allocate: scratch is the library's fixed array."""
    if G_saved is not None:
        _check_size(G_saved, ttt_saved_bytes(cfg), "G_saved")
    st = _lib.ttt_chunk_bwd_noalloc(ctypes.byref(cfg), _ptr(Q), _ptr(K), _ptr(V), _ptr(beta),
                                    _ptr(gamma), _ptr(W0), _ptr(W_chunks), _ptr(G_saved),
                                    _ptr(dO), _ptr(dW_final), _ptr(O), _ptr(W_final), _ptr(dQ),
                                    _ptr(dK), _ptr(dV), _ptr(dbeta), _ptr(dW0), _ptr(dgamma),
                                    _stream(stream))
    _check(st, "ttt_chunk_bwd_noalloc")


def ttt_mlp_workspace_bytes(cfg: ttt_config, hidden: int) -> int:
    n = _lib.ttt_mlp_workspace_bytes(ctypes.byref(cfg), int(hidden))
    if n == ctypes.c_size_t(-1).value:
        raise TTTError(ERR_INVALID_ARG, "ttt_mlp_workspace_bytes")
    return n


def ttt_mlp_fwd(cfg, hidden, Q, K, V, beta, gamma, W1_0, W2_0, O, W1_final, W2_final, W1_chunks,
                W2_chunks, workspace, workspace_bytes, stream=None):
    """TTT-MLP forward: the fast weight act(k W1) W2 with W1 [B,H,dk,hidden] and W2
    [B,H,hidden,dv] float32; W1_chunks / W2_chunks keep the chunk-start weights for the
    backward. Workspace: ttt_mlp_workspace_bytes(cfg, hidden)."""
    st = _lib.ttt_mlp_fwd(ctypes.byref(cfg), int(hidden), _ptr(Q), _ptr(K), _ptr(V), _ptr(beta),
                          _ptr(gamma), _ptr(W1_0), _ptr(W2_0), _ptr(O), _ptr(W1_final),
                          _ptr(W2_final), _ptr(W1_chunks), _ptr(W2_chunks), _ptr(workspace),
                          int(workspace_bytes), _stream(stream))
    _check(st, "ttt_mlp_fwd")


def ttt_mlp_bwd(cfg, hidden, Q, K, V, beta, gamma, W1_chunks, W2_chunks, dO, dW1_final, dW2_final,
                dQ, dK, dV, dbeta, dW1_0, dW2_0, workspace, workspace_bytes, stream=None):
    """TTT-MLP backward for J = <dO, O> + <dW1_final, W1_final> + <dW2_final, W2_final>."""
    st = _lib.ttt_mlp_bwd(ctypes.byref(cfg), int(hidden), _ptr(Q), _ptr(K), _ptr(V), _ptr(beta),
                          _ptr(gamma), _ptr(W1_chunks), _ptr(W2_chunks), _ptr(dO), _ptr(dW1_final),
                          _ptr(dW2_final), _ptr(dQ), _ptr(dK), _ptr(dV), _ptr(dbeta), _ptr(dW1_0),
                          _ptr(dW2_0), _ptr(workspace), int(workspace_bytes), _stream(stream))
    _check(st, "ttt_mlp_bwd")


def inplace_ttt_workspace_bytes(T, d_ff, d_model, C) -> int:
    n = _lib.inplace_ttt_workspace_bytes(T, d_ff, d_model, C)
    if n == ctypes.c_size_t(-1).value:
        raise TTTError(ERR_INVALID_ARG, "inplace_ttt_workspace_bytes")
    return n


def inplace_ttt_fwd(T, d_ff, d_model, C, lr, Z, Vhat, W, O, workspace=None, workspace_bytes=0,
                    stream=None, W_chunks=None):
    """In-Place TTT forward: per chunk of C tokens O_i = Z_i W^T, then W += lr Vhat_i^T Z_i.

    Z [T,d_ff] and Vhat [T,d_model] bf16; W [d_model,d_ff] float32 in/out; O [T,d_model] bf16;
    W_chunks [T/C,d_model,d_ff] bf16 (optional) keeps the weight each chunk applied, for
    inplace_ttt_bwd. Workspace: inplace_ttt_workspace_bytes(T, d_ff, d_model, C)."""
    st = _lib.inplace_ttt_fwd(T, d_ff, d_model, C, float(lr), _ptr(Z), _ptr(Vhat), _ptr(W),
                              _ptr(O), _ptr(W_chunks), _ptr(workspace), int(workspace_bytes),
                              _stream(stream))
    _check(st, "inplace_ttt_fwd")


def _int_array(xs):
    xs = [int(x) for x in xs]
    return (ctypes.c_int * max(1, len(xs)))(*xs), len(xs)


def inplace_ttt_docs_workspace_bytes(T, d_ff, d_model, C) -> int:
    n = _lib.inplace_ttt_docs_workspace_bytes(T, d_ff, d_model, C)
    if n == ctypes.c_size_t(-1).value:
        raise TTTError(ERR_INVALID_ARG, "inplace_ttt_docs_workspace_bytes")
    return n


def inplace_ttt_fwd_docs(T, d_ff, d_model, C, lr, Z, Vhat, W, O, W_chunks, doc_starts, workspace,
                         workspace_bytes, stream=None):
    arr, n = _int_array(doc_starts)
    st = _lib.inplace_ttt_fwd_docs(T, d_ff, d_model, C, float(lr), _ptr(Z), _ptr(Vhat), _ptr(W),
                                   _ptr(O), _ptr(W_chunks), arr, n, _ptr(workspace),
                                   int(workspace_bytes), _stream(stream))
    _check(st, "inplace_ttt_fwd_docs")


def inplace_ttt_bwd_docs(T, d_ff, d_model, C, lr, Z, Vhat, W_chunks, dO, dW_final, dZ, dVhat, dW,
                         doc_starts, workspace, workspace_bytes, stream=None):
    arr, n = _int_array(doc_starts)
    st = _lib.inplace_ttt_bwd_docs(T, d_ff, d_model, C, float(lr), _ptr(Z), _ptr(Vhat),
                                   _ptr(W_chunks), _ptr(dO), _ptr(dW_final), _ptr(dZ), _ptr(dVhat),
                                   _ptr(dW), arr, n, _ptr(workspace), int(workspace_bytes),
                                   _stream(stream))
    _check(st, "inplace_ttt_bwd_docs")


def inplace_ttt_target_workspace_bytes(T, d_model) -> int:
    n = _lib.inplace_ttt_target_workspace_bytes(T, d_model)
    if n == ctypes.c_size_t(-1).value:
        raise TTTError(ERR_INVALID_ARG, "inplace_ttt_target_workspace_bytes")
    return n


def inplace_ttt_target(T, d_model, k, X0, conv_w, W_target, Vhat, workspace=None,
                       workspace_bytes=0, stream=None):
    st = _lib.inplace_ttt_target(T, d_model, k, _ptr(X0), _ptr(conv_w), _ptr(W_target), _ptr(Vhat),
                                 _ptr(workspace), int(workspace_bytes), _stream(stream))
    _check(st, "inplace_ttt_target")


def inplace_ttt_target_bwd_workspace_bytes(T, d_model, k) -> int:
    n = _lib.inplace_ttt_target_bwd_workspace_bytes(T, d_model, k)
    if n == ctypes.c_size_t(-1).value:
        raise TTTError(ERR_INVALID_ARG, "inplace_ttt_target_bwd_workspace_bytes")
    return n


def inplace_ttt_target_bwd(T, d_model, k, X0, conv_w, W_target, dVhat, dX0, dconv_w, dW_target,
                           workspace=None, workspace_bytes=0, stream=None):
    st = _lib.inplace_ttt_target_bwd(T, d_model, k, _ptr(X0), _ptr(conv_w), _ptr(W_target),
                                     _ptr(dVhat), _ptr(dX0), _ptr(dconv_w), _ptr(dW_target),
                                     _ptr(workspace), int(workspace_bytes), _stream(stream))
    _check(st, "inplace_ttt_target_bwd")


def inplace_ttt_bwd(T, d_ff, d_model, C, lr, Z, Vhat, W_chunks, dO, dW_final, dZ, dVhat, dW,
                    workspace=None, workspace_bytes=0, stream=None):
    """In-Place TTT backward for J = sum_i <dO_i, O_i> + <dW_final, W_final> (dW_final may
    be None): writes dZ [T,d_ff] and dVhat [T,d_model] bf16 and dW, the float32 gradient of the
    initial W, from the forward's W_chunks."""
    st = _lib.inplace_ttt_bwd(T, d_ff, d_model, C, float(lr), _ptr(Z), _ptr(Vhat), _ptr(W_chunks),
                              _ptr(dO), _ptr(dW_final), _ptr(dZ), _ptr(dVhat), _ptr(dW),
                              _ptr(workspace), int(workspace_bytes), _stream(stream))
    _check(st, "inplace_ttt_bwd")


def ttt_get_device_error(stream=None) -> int:
    """Returns the status (OK, ERR_TIMEOUT, ERR_RANGE or ERR_CUDA) instead of raising."""
    return _lib.ttt_get_device_error(_stream(stream))


def ttt_selftest_bounded_wait(spin_limit: int, stream=None):
    _check(_lib.ttt_selftest_bounded_wait(int(spin_limit), _stream(stream)), "ttt_selftest_bounded_wait")


def ttt_kernel_launches() -> int:
    return int(_lib.ttt_kernel_launches())


# Raw C entry points (for callers that marshal pointers themselves).
lib = _lib


def inplace_ttt_delta(T, d_ff, d_model, lr, Z, Vhat, dW, workspace, workspace_bytes, stream=None):
    """dW = lr Vhat^T Z over all T tokens (the summed chunk updates of one shard)."""
    st = _lib.inplace_ttt_delta(T, d_ff, d_model, float(lr), _ptr(Z), _ptr(Vhat), _ptr(dW),
                                _ptr(workspace), int(workspace_bytes), _stream(stream))
    _check(st, "inplace_ttt_delta")


def ttt_add_f32(dst, src, stream=None):
    st = _lib.ttt_add_f32(_ptr(dst), _ptr(src), int(dst.numel()), _stream(stream))
    _check(st, "ttt_add_f32")


class _CudaOps:
    """The library calls the context-parallel In-Place forward is made of."""

    @staticmethod
    def delta(T, d_ff, d_model, lr, Z, Vhat, dW, workspace, workspace_bytes):
        inplace_ttt_delta(T, d_ff, d_model, lr, Z, Vhat, dW, workspace, workspace_bytes)

    @staticmethod
    def add(dst, src):
        ttt_add_f32(dst, src)

    @staticmethod
    def fwd(T, d_ff, d_model, C, lr, Z, Vhat, W, O, workspace, workspace_bytes):
        inplace_ttt_fwd(T, d_ff, d_model, C, lr, Z, Vhat, W, O, workspace, workspace_bytes)


def inplace_cp_fwd(T, d_ff, d_model, C, lr, Z, Vhat, W, O, workspace, workspace_bytes,
                   group=None, ops=None):
    """Context-parallel In-Place forward (page "In-Place Test-Time Training", section "核心方法和
    技术细节": the update is associative, so the chunk loop runs as a parallel scan across
    devices). The sequence is split in order across the ranks of `group`; this rank holds its
    T tokens (Z [T, d_ff], Vhat [T, d_model]), and W holds the initial W_down on every rank.
    Each rank computes its shard's summed update dW_g = lr Vhat_g^T Z_g, the ranks exchange
    them (all-gather), rank g adds dW_h for h < g to W and runs inplace_ttt_fwd on its tokens.
    On return O holds this shard's outputs and W its end state (the last rank's W is the
    sequence's final W_down). `ops` replaces the library calls (the CPU tests of the exchange
    pass an implementation built on the oracle); by default they are the C ABI's."""
    import torch
    import torch.distributed as dist
    ops = ops or _CudaOps
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    dW = torch.empty_like(W)
    ops.delta(T, d_ff, d_model, lr, Z, Vhat, dW, workspace, workspace_bytes)
    parts = [torch.empty_like(dW) for _ in range(world)]
    dist.all_gather(parts, dW, group=group)
    for h in range(rank):
        ops.add(W, parts[h])
    ops.fwd(T, d_ff, d_model, C, lr, Z, Vhat, W, O, workspace, workspace_bytes)
