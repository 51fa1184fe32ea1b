"""The C-ABI library loads, exports every function include/ttt.h declares, and rejects bad
arguments on the host before touching a GPU (these run without one)."""
import ctypes
import os
import subprocess

import pytest

import weight_sequence_layers_b200 as ttt

FWD_NAMES = {"ttt_workspace_bytes", "ttt_chunk_fwd", "ttt_chunk_bwd", "inplace_ttt_workspace_bytes",
             "inplace_ttt_fwd", "inplace_ttt_bwd", "inplace_ttt_target", "inplace_ttt_target_workspace_bytes",
             "inplace_ttt_target_bwd", "inplace_ttt_target_bwd_workspace_bytes",
             "ttt_mlp_fwd", "ttt_mlp_bwd", "ttt_mlp_workspace_bytes",
             "inplace_ttt_fwd_docs", "inplace_ttt_bwd_docs", "inplace_ttt_docs_workspace_bytes",
             "inplace_ttt_delta", "ttt_add_f32", "ttt_saved_bytes", "ttt_get_device_error", "ttt_selftest_bounded_wait",
             "ttt_status_string", "ttt_kernel_launches", "ttt_chunk_bwd_noalloc"}


def test_binding_gives_every_declared_function_its_signature():
    # ctypes would otherwise pass every argument as a C int
    assert set(ttt.header_functions()) == set(ttt._SIGS)


def test_header_declares_the_entry_points():
    assert FWD_NAMES <= set(ttt.header_functions())


def test_every_declared_symbol_is_exported():
    out = subprocess.run(["nm", "-D", "--defined-only", ttt.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    for name in ttt.header_functions():
        assert name in exported, name
        assert getattr(ttt.lib, name) is not None


def test_library_links_no_libcuda():
    out = subprocess.run(["ldd", ttt.LIB_PATH], capture_output=True, text=True).stdout
    assert "libcuda.so" not in out and "libcudart.so" not in out


def test_status_strings():
    for s in range(8):
        assert ttt.status_string(s)
    assert ttt.status_string(99) == "unknown status"


def _cfg(**kw):
    base = dict(B=2, H=3, T=256, dk=64, dv=64, C=64, dtype="f32", loss="mse", act="id", lr_bias=-2.9)
    base.update(kw)
    return ttt.make_config(**base)


def test_workspace_query_validates_config():
    assert ttt.ttt_workspace_bytes(_cfg(), 0) == 0
    assert ttt.ttt_workspace_bytes(_cfg(), 1) > 0
    # the tensor-core backward keeps G in its workspace only when the forward's saved tensors
    # are not passed
    tc = _cfg(dtype="bf16", dk=128, dv=128, C=256, T=512)
    assert 0 < ttt.ttt_workspace_bytes(tc, 2) < ttt.ttt_workspace_bytes(tc, 1)
    with pytest.raises(ttt.TTTError):
        ttt.ttt_workspace_bytes(tc, 3)
    for bad in (dict(T=250), dict(C=0), dict(B=0), dict(dk=0),
                dict(B=1 << 14, H=1 << 10, T=1 << 7, C=128, dk=1, dv=1)):  # B*H*T = 2^31
        with pytest.raises(ttt.TTTError):
            ttt.ttt_workspace_bytes(_cfg(**bad), False)
    cfg = _cfg()
    cfg.loss = 7
    with pytest.raises(ttt.TTTError):
        ttt.ttt_workspace_bytes(cfg, False)


def test_unsupported_shapes_are_reported():
    cfg = _cfg(dk=256)
    assert ttt.lib.ttt_workspace_bytes(ctypes.byref(cfg), 0) == ctypes.c_size_t(-1).value
    st = ttt.lib.ttt_chunk_fwd(ctypes.byref(cfg), *([16] * 3), 16, None, 16, 16, None, None, None,
                               None, 0, None)
    assert st == ttt.ERR_UNSUPPORTED


def test_fwd_argument_errors_before_launch():
    cfg = _cfg()
    call = lambda *p: ttt.lib.ttt_chunk_fwd(ctypes.byref(cfg), *p, None)
    A = 4096  # a 16-byte aligned fake address: never dereferenced on these paths
    assert call(None, A, A, A, None, A, A, None, None, None, None, 0) == ttt.ERR_INVALID_ARG
    assert call(A, A, A, A, None, A, None, None, None, None, None, 0) == ttt.ERR_INVALID_ARG
    assert call(A + 4, A, A, A, None, A, A, None, None, None, None, 0) == ttt.ERR_ALIGNMENT
    assert call(A, A, A, A, A + 8, A, A, None, None, None, None, 0) == ttt.ERR_ALIGNMENT
    assert call(A, A, A, A, None, A, A, None, None, A + 2, None, 0) == ttt.ERR_ALIGNMENT  # G_saved
    bad = _cfg(T=100)
    assert ttt.lib.ttt_chunk_fwd(ctypes.byref(bad), A, A, A, A, None, A, A, None, None, None, None,
                                 0, None) == ttt.ERR_INVALID_ARG
    assert ttt.lib.ttt_chunk_fwd(None, A, A, A, A, None, A, A, None, None, None, None, 0,
                                 None) == ttt.ERR_INVALID_ARG


def test_bwd_requires_chunk_states_and_workspace():
    cfg = _cfg()
    A = 4096
    # Q K V beta gamma W0 W_chunks G_saved dO dW_final O W_final dQ dK dV dbeta dW0 dgamma
    base = [A, A, A, A, None, A, A, None, A, None, None, None, A, A, A, A, A, None]
    args = list(base)
    args[6] = None  # W_chunks
    assert ttt.lib.ttt_chunk_bwd(ctypes.byref(cfg), *args, None, 0, None) == ttt.ERR_INVALID_ARG
    assert ttt.lib.ttt_chunk_bwd(ctypes.byref(cfg), *base, None, 0, None) == ttt.ERR_WORKSPACE
    need = ttt.ttt_workspace_bytes(cfg, 1)
    assert ttt.lib.ttt_chunk_bwd(ctypes.byref(cfg), *base, A, need - 1, None) == ttt.ERR_WORKSPACE
    # the decay gradient needs gamma and the forward's O (and W_final with dW_final)
    dg = list(base)
    dg[17] = A  # dgamma without gamma
    assert ttt.lib.ttt_chunk_bwd(ctypes.byref(cfg), *dg, A, need, None) == ttt.ERR_INVALID_ARG
    dg[4] = A   # gamma, but no O
    assert ttt.lib.ttt_chunk_bwd(ctypes.byref(cfg), *dg, A, need, None) == ttt.ERR_INVALID_ARG
    dg[10] = A  # O; dW_final set without W_final
    dg[9] = A
    assert ttt.lib.ttt_chunk_bwd(ctypes.byref(cfg), *dg, A, need, None) == ttt.ERR_INVALID_ARG


def test_decay_kind_is_checked_and_vector_decay_leaves_the_tensor_core_path():
    bad = _cfg()
    bad.decay = 2
    with pytest.raises(ttt.TTTError):
        ttt.ttt_workspace_bytes(bad, 0)
    # a shape the tensor-core backward takes with a scalar decay needs its chunk-end adjoint
    # scratch; with a vector decay the SIMT backward's per-head scratch is sized instead
    tc = _cfg(dtype="bf16", dk=128, dv=128, C=256, T=512)
    vec = _cfg(dtype="bf16", dk=128, dv=128, C=256, T=512, decay="vector")
    assert ttt.ttt_workspace_bytes(vec, 1) != ttt.ttt_workspace_bytes(tc, 1)
    # the fixed-scratch backward serves tensor-core configs only
    A = 4096
    st = ttt.lib.ttt_chunk_bwd_noalloc(ctypes.byref(vec), A, A, A, A, A, A, A, None, A, None, None,
                                       None, A, A, A, A, A, None, None)
    assert st == ttt.ERR_UNSUPPORTED
    # a valid config that no backward path serves (dk = dv = 256) is unsupported, not invalid;
    # an invalid one is invalid
    wide = _cfg(dtype="bf16", dk=256, dv=256, C=256, T=512)
    st = ttt.lib.ttt_chunk_bwd_noalloc(ctypes.byref(wide), A, A, A, A, A, A, A, None, A, None, None,
                                       None, A, A, A, A, A, None, None)
    assert st == ttt.ERR_UNSUPPORTED
    st = ttt.lib.ttt_chunk_bwd_noalloc(ctypes.byref(_cfg(T=250)), A, A, A, A, A, A, A, None, A, None,
                                       None, None, A, A, A, A, A, None, None)
    assert st == ttt.ERR_INVALID_ARG


def test_tc_bwd_workspace_covers_the_decay_gradient():
    # the query's backward figure includes the float per token that only dgamma calls use
    tc = _cfg(dtype="bf16", dk=128, dv=128, C=256, T=512)
    need = ttt.ttt_workspace_bytes(tc, 2)
    A = 4096
    # Q K V beta gamma W0 W_chunks G_saved dO dW_final O W_final dQ dK dV dbeta dW0 dgamma
    args = [A, A, A, A, A, A, A, A, A, None, A, None, A, A, A, A, A, A]
    short = need - tc.B * tc.H * tc.T * 4
    assert ttt.lib.ttt_chunk_bwd(ctypes.byref(tc), *args, A, short, None) == ttt.ERR_WORKSPACE


def test_inplace_argument_errors():
    A = 4096
    f = ttt.lib.inplace_ttt_fwd
    # T d_ff d_model C lr Z Vhat W O W_chunks workspace bytes stream
    assert f(1000, 256, 256, 128, 1e-3, A, A, A, A, None, A, 1 << 30, None) == ttt.ERR_INVALID_ARG  # T % C
    assert f(960, 256, 256, 96, 1e-3, A, A, A, A, None, A, 1 << 30, None) == ttt.ERR_UNSUPPORTED    # C % 128
    assert f(1024, 250, 256, 128, 1e-3, A, A, A, A, None, A, 1 << 30, None) == ttt.ERR_UNSUPPORTED  # d_ff % 64
    assert f(1024, 256, 256, 128, float("nan"), A, A, A, A, None, A, 1 << 30, None) == ttt.ERR_INVALID_ARG
    assert f(1024, 256, 256, 128, 1e-3, None, A, A, A, None, A, 1 << 30, None) == ttt.ERR_INVALID_ARG
    assert f(1024, 256, 256, 128, 1e-3, A, A, A + 4, A, None, A, 1 << 30, None) == ttt.ERR_ALIGNMENT
    assert f(1024, 256, 256, 128, 1e-3, A, A, A, A, A + 8, A, 1 << 30, None) == ttt.ERR_ALIGNMENT
    need = ttt.inplace_ttt_workspace_bytes(1024, 256, 256, 128)
    assert need >= 2 * 256 * 256 * 2
    assert f(1024, 256, 256, 128, 1e-3, A, A, A, A, None, A, need - 1, None) == ttt.ERR_WORKSPACE
    with pytest.raises(ttt.TTTError):
        ttt.inplace_ttt_workspace_bytes(1000, 256, 256, 128)


def test_inplace_bwd_argument_errors():
    A = 4096
    b = ttt.lib.inplace_ttt_bwd
    need = ttt.inplace_ttt_workspace_bytes(1024, 256, 256, 128)
    # T d_ff d_model C lr Z Vhat W_chunks dO dW_final dZ dVhat dW workspace bytes stream
    ok = [A, A, A, A, None, A, A, A, A, need, None]
    assert b(1000, 256, 256, 128, 1e-3, *ok) == ttt.ERR_INVALID_ARG        # T % C
    assert b(1024, 256, 192, 128, 1e-3, *ok) == ttt.ERR_UNSUPPORTED        # d_model % 128
    args = list(ok)
    args[2] = None                                                          # W_chunks is required
    assert b(1024, 256, 256, 128, 1e-3, *args) == ttt.ERR_INVALID_ARG
    args = list(ok)
    args[4] = A + 4                                                         # dW_final misaligned
    assert b(1024, 256, 256, 128, 1e-3, *args) == ttt.ERR_ALIGNMENT
    args = list(ok)
    args[9] = need - 1
    assert b(1024, 256, 256, 128, 1e-3, *args) == ttt.ERR_WORKSPACE


def test_valid_call_without_a_gpu_reports_cuda_error():
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    cfg = _cfg()
    A = 4096
    st = ttt.lib.ttt_chunk_fwd(ctypes.byref(cfg), A, A, A, A, None, A, A, None, None, None, None, 0,
                               None)
    assert st == ttt.ERR_CUDA


def test_inplace_target_argument_errors():
    A = 4096
    f = ttt.lib.inplace_ttt_target
    need = ttt.inplace_ttt_target_workspace_bytes(256, 128)
    assert need >= 256 * 128 * 2
    # T d_model k X0 conv_w W_target Vhat workspace bytes stream
    assert f(256, 128, 0, A, A, A, A, A, need, None) == ttt.ERR_INVALID_ARG     # k < 1
    assert f(256, 128, 9, A, A, A, A, A, need, None) == ttt.ERR_UNSUPPORTED     # k > 8
    assert f(200, 128, 4, A, A, A, A, A, need, None) == ttt.ERR_UNSUPPORTED     # T % 128
    assert f(256, 128, 4, None, A, A, A, A, need, None) == ttt.ERR_INVALID_ARG
    assert f(256, 128, 4, A, A + 4, A, A, A, need, None) == ttt.ERR_ALIGNMENT
    assert f(256, 128, 4, A, A, A, A, A, need - 1, None) == ttt.ERR_WORKSPACE
    with pytest.raises(ttt.TTTError):
        ttt.inplace_ttt_target_workspace_bytes(256, 100)


def test_inplace_target_bwd_argument_errors():
    A = 4096
    f = ttt.lib.inplace_ttt_target_bwd
    need = ttt.inplace_ttt_target_bwd_workspace_bytes(256, 128, 4)
    # T d_model k X0 conv_w W_target dVhat dX0 dconv_w dW_target workspace bytes stream
    ok = [A, A, A, A, A, A, A, A, need, None]
    assert f(256, 128, 9, *ok) == ttt.ERR_UNSUPPORTED
    args = list(ok)
    args[5] = None  # dconv_w
    assert f(256, 128, 4, *args) == ttt.ERR_INVALID_ARG
    args = list(ok)
    args[8] = need - 1
    assert f(256, 128, 4, *args) == ttt.ERR_WORKSPACE
    with pytest.raises(ttt.TTTError):
        ttt.inplace_ttt_target_bwd_workspace_bytes(256, 128, 0)


def test_ttt_mlp_argument_errors():
    cfg = _cfg()
    A = 4096
    need = ttt.ttt_mlp_workspace_bytes(cfg, 96)
    assert need > 0
    with pytest.raises(ttt.TTTError):
        ttt.ttt_mlp_workspace_bytes(cfg, 600)                     # hidden > 512
    vec = _cfg(decay="vector")
    with pytest.raises(ttt.TTTError):
        ttt.ttt_mlp_workspace_bytes(vec, 96)                      # scalar decay only
    f = ttt.lib.ttt_mlp_fwd
    # cfg hidden Q K V beta gamma W1_0 W2_0 O W1_final W2_final W1_chunks W2_chunks ws bytes stream
    ok = [A, A, A, A, None, A, A, A, None, None, None, None, A, need, None]
    assert f(ctypes.byref(cfg), 0, *ok) == ttt.ERR_UNSUPPORTED
    args = list(ok)
    args[5] = None  # W1_0
    assert f(ctypes.byref(cfg), 96, *args) == ttt.ERR_INVALID_ARG
    args = list(ok)
    args[13] = need - 1
    assert f(ctypes.byref(cfg), 96, *args) == ttt.ERR_WORKSPACE
    b = ttt.lib.ttt_mlp_bwd
    # cfg hidden Q K V beta gamma W1c W2c dO dW1f dW2f dQ dK dV dbeta dW1 dW2 ws bytes stream
    okb = [A, A, A, A, None, None, A, A, None, None, A, A, A, A, A, A, A, need, None]
    assert b(ctypes.byref(cfg), 96, *okb) == ttt.ERR_INVALID_ARG  # W1_chunks is required


def test_inplace_document_list_is_checked():
    A = 4096
    f = ttt.lib.inplace_ttt_fwd_docs
    need = ttt.inplace_ttt_docs_workspace_bytes(1024, 256, 256, 128)
    assert need > ttt.inplace_ttt_workspace_bytes(1024, 256, 256, 128)
    # T d_ff d_model C lr Z Vhat W O W_chunks doc_starts n_docs workspace bytes stream
    for bad in ([0], [8], [3, 3], [4, 2], [-1]):  # 8 chunks: starts must be in 1..7, increasing
        arr = (ctypes.c_int * len(bad))(*bad)
        assert f(1024, 256, 256, 128, 1e-3, A, A, A, A, None, arr, len(bad), A, need, None) == \
            ttt.ERR_INVALID_ARG, bad
    arr = (ctypes.c_int * 1)(3)
    short = ttt.inplace_ttt_workspace_bytes(1024, 256, 256, 128)
    assert f(1024, 256, 256, 128, 1e-3, A, A, A, A, None, arr, 1, A, short, None) == ttt.ERR_WORKSPACE


def test_context_parallel_calls_check_arguments():
    A = 4096
    d = ttt.lib.inplace_ttt_delta
    # T d_ff d_model lr Z Vhat dW workspace bytes stream
    assert d(200, 256, 256, 1e-3, A, A, A, A, 256, None) == ttt.ERR_UNSUPPORTED   # T % 128
    assert d(256, 256, 256, float("nan"), A, A, A, A, 256, None) == ttt.ERR_INVALID_ARG
    assert d(256, 256, 256, 1e-3, A, A, None, A, 256, None) == ttt.ERR_INVALID_ARG
    assert d(256, 256, 256, 1e-3, A, A, A, A, 255, None) == ttt.ERR_WORKSPACE
    a = ttt.lib.ttt_add_f32
    assert a(A, A, 6, None) == ttt.ERR_INVALID_ARG      # n % 4
    assert a(A + 4, A, 8, None) == ttt.ERR_ALIGNMENT
    assert a(None, A, 8, None) == ttt.ERR_INVALID_ARG


def test_shared_initial_state_flag_is_validated():
    c = _cfg()
    c.w0_shared = 1
    assert ttt.ttt_workspace_bytes(c, 0) == 0
    c.w0_shared = 2
    with pytest.raises(ttt.TTTError):
        ttt.ttt_workspace_bytes(c, 0)
    assert _cfg(w0_shared=True).w0_shared == 1


def test_saved_buffer_size():
    cfg = _cfg(dtype="bf16", dk=128, dv=96, C=128, T=512)
    assert ttt.ttt_saved_bytes(cfg) == 2 * 3 * 512 * 96 * 2
    assert ttt.ttt_saved_bytes(_cfg(dtype="bf16", dk=128, dv=96, C=128, T=512, act="silu")) == \
        2 * 2 * 3 * 512 * 96 * 2
    assert ttt.ttt_saved_bytes(_cfg()) == 2 * 3 * 256 * 64 * 4
    # vector decay on the tensor cores: G first, then the forward's decayed operands and R
    vec = _cfg(dtype="bf16", dk=64, dv=64, C=256, T=512, decay="vector")
    g_plane = 2 * 3 * 512 * 64 * 2
    assert ttt.ttt_saved_bytes(vec) > 4 * g_plane
    # (the vector decay outside that path keeps G alone)
    assert ttt.ttt_saved_bytes(_cfg(dtype="bf16", dk=64, dv=64, C=64, T=512, decay="vector")) == \
        2 * 3 * 512 * 64 * 2
    with pytest.raises(ttt.TTTError):
        ttt.ttt_saved_bytes(_cfg(T=250))


def test_binding_refuses_host_and_strided_tensors():
    # the library takes dense device arrays; the binding refuses anything else before calling it
    import torch
    cfg = _cfg(B=1, H=1, T=64, dk=16, dv=16, C=16)
    x = torch.zeros((1, 1, 64, 16))
    beta, W0 = torch.zeros((1, 1, 64)), torch.zeros((1, 1, 16, 16))
    n0 = ttt.ttt_kernel_launches()
    with pytest.raises(ValueError, match="CUDA tensors"):
        ttt.ttt_chunk_fwd(cfg, x, x, x, beta, None, W0, x)
    with pytest.raises(ValueError, match="contiguous"):
        ttt.ttt_chunk_fwd(cfg, x.transpose(2, 3), x, x, beta, None, W0, x)
    with pytest.raises(ValueError, match="CUDA tensors"):
        ttt.ttt_add_f32(torch.zeros(8), torch.zeros(8))
    Zt = torch.zeros((128, 256)).t()  # [T, d_ff] = [256, 128], column-major
    Vh, W, O = (torch.zeros(s) for s in ((256, 128), (128, 128), (256, 128)))
    with pytest.raises(ValueError, match="contiguous"):
        ttt.inplace_ttt_fwd(256, 128, 128, 128, 1e-3, Zt, Vh, W, O)
    assert ttt.ttt_kernel_launches() == n0


C_CLIENT = r"""
#include "ttt.h"
#include <stdio.h>
#include <string.h>

/* A plain C99 caller of the library: the header must compile as C, the entry points must
   link, and argument errors must come back as statuses with nothing launched. */
int main(void) {
  ttt_config c = {2, 3, 256, 64, 64, 64, TTT_F32, TTT_LOSS_MSE, TTT_ACT_ID, -2.9f,
                  TTT_DECAY_SCALAR, 0};
  char a[64];
  void* p = (void*)(((unsigned long)a + 15) & ~15ul); /* aligned, never dereferenced */
  int bad = 0;
  bad |= strcmp(ttt_status_string(TTT_OK), "ok") != 0;
  bad |= ttt_workspace_bytes(&c, 0) != 0;
  bad |= ttt_workspace_bytes(&c, 1) == 0 || ttt_workspace_bytes(&c, 1) == (size_t)-1;
  /* Q missing */
  bad |= ttt_chunk_fwd(&c, NULL, p, p, (const float*)p, NULL, (const float*)p, p, NULL, NULL,
                       NULL, NULL, 0, NULL) != TTT_ERR_INVALID_ARG;
  /* misaligned K */
  bad |= ttt_chunk_fwd(&c, p, (char*)p + 4, p, (const float*)p, NULL, (const float*)p, p, NULL,
                       NULL, NULL, NULL, 0, NULL) != TTT_ERR_ALIGNMENT;
  /* T not a multiple of C */
  c.T = 250;
  bad |= ttt_workspace_bytes(&c, 0) != (size_t)-1;
  bad |= inplace_ttt_workspace_bytes(1000, 256, 256, 128) != (size_t)-1;
  printf("%s\n", bad ? "FAIL" : "PASS");
  return bad;
}
"""


def test_header_compiles_and_links_as_plain_c(tmp_path):
    src = tmp_path / "client.c"
    src.write_text(C_CLIENT)
    exe = tmp_path / "client"
    pkg = os.path.dirname(ttt.LIB_PATH)
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror",
                    "-I", os.path.dirname(ttt.HEADER), str(src), "-L", pkg, "-lttt",
                    f"-Wl,-rpath,{pkg}", "-o", str(exe)], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True)
    assert r.returncode == 0 and r.stdout.strip() == "PASS", r.stdout + r.stderr


def _declared_parameters():
    """name -> list of parameter declarations, parsed from include/ttt.h."""
    import re
    text = open(ttt.HEADER).read()
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)  # drop comments
    out = {}
    for name in ttt.header_functions():
        m = re.search(r"\b" + name + r"\s*\(([^)]*)\)\s*;", text)
        assert m, name
        params = [p.strip() for p in m.group(1).split(",")]
        out[name] = [] if params == ["void"] else params
    return out


def _kind_of_declaration(p):
    if "*" in p:
        return "pointer"
    words = p.split()[:-1]  # drop the parameter name
    if words == ["size_t"]:
        return "size_t"
    if words == ["float"]:
        return "float"
    if words in (["int"], ["unsigned"], ["ttt_status"]):
        return "int"
    raise AssertionError(f"unexpected parameter {p!r}")


def _kind_of_ctype(t):
    if t in (ctypes.c_void_p,) or (isinstance(t, type) and issubclass(t, ctypes._Pointer)):
        return "pointer"
    if t is ctypes.c_size_t:
        return "size_t"
    if t is ctypes.c_float:
        return "float"
    if t in (ctypes.c_int, ctypes.c_uint):
        return "int"
    raise AssertionError(f"unexpected ctypes type {t!r}")


def test_binding_signatures_match_the_header():
    # the number and kind (pointer, size_t, float, int) of every argument ctypes passes agree
    # with the declaration; a mismatch would shift every later argument
    for name, params in _declared_parameters().items():
        argtypes, _ = ttt._SIGS[name]
        assert [_kind_of_declaration(p) for p in params] == \
            [_kind_of_ctype(t) for t in argtypes], name


def test_binding_return_types_match_the_header():
    import re
    text = open(ttt.HEADER).read()
    want = {"size_t": ctypes.c_size_t, "ttt_status": ctypes.c_int, "const char*": ctypes.c_char_p,
            "unsigned long long": ctypes.c_ulonglong}
    for name in ttt.header_functions():
        m = re.search(r"^([A-Za-z_][\w \t\*]*?)\s*\b" + name + r"\s*\(", text, flags=re.M)
        ret = " ".join(m.group(1).replace("*", " * ").split()).replace(" *", "*")
        assert ttt._SIGS[name][1] is want[ret], (name, ret)


def test_config_struct_matches_the_header():
    # field order and types of ttt_config in the binding are the header's, and so are the
    # enum values the binding passes
    import re
    text = re.sub(r"/\*.*?\*/", " ", open(ttt.HEADER).read(), flags=re.S)
    body = re.search(r"typedef struct \{(.*?)\} ttt_config;", text, flags=re.S).group(1)
    fields = []
    for decl in body.split(";"):
        words = decl.replace(",", " ").split()
        if words:
            fields += [(name, words[0]) for name in words[1:]]
    ctype = {"int": ctypes.c_int, "float": ctypes.c_float}
    assert [(n, ctype[t]) for n, t in fields] == list(ttt.ttt_config._fields_)
    enums = dict(re.findall(r"\b(TTT_[A-Z0-9_]+)\s*=\s*(\d+)", text))
    assert int(enums["TTT_F32"]) == ttt.F32 and int(enums["TTT_BF16"]) == ttt.BF16
    assert {k: int(enums["TTT_LOSS_" + k.upper()]) for k in ttt.LOSS} == ttt.LOSS
    assert {k: int(enums["TTT_ACT_" + k.upper()]) for k in ttt.ACT} == ttt.ACT
    assert {k: int(enums["TTT_DECAY_" + k.upper()]) for k in ttt.DECAY} == ttt.DECAY
    names = ["TTT_OK", "TTT_ERR_INVALID_ARG", "TTT_ERR_UNSUPPORTED", "TTT_ERR_ALIGNMENT",
             "TTT_ERR_WORKSPACE", "TTT_ERR_CUDA", "TTT_ERR_TIMEOUT", "TTT_ERR_RANGE"]
    assert [int(enums[n]) for n in names] == [ttt.OK, ttt.ERR_INVALID_ARG, ttt.ERR_UNSUPPORTED,
                                             ttt.ERR_ALIGNMENT, ttt.ERR_WORKSPACE, ttt.ERR_CUDA,
                                             ttt.ERR_TIMEOUT, ttt.ERR_RANGE]
    m = re.search(r"#define TTT_NOALLOC_SCRATCH_BYTES \(\(size_t\)(\d+) << (\d+)\)", text)
    assert int(m.group(1)) << int(m.group(2)) == ttt.NOALLOC_SCRATCH_BYTES


@pytest.mark.parametrize("act", ["id", "silu"])
@pytest.mark.parametrize("d,C", [(64, 256), (128, 128), (128, 256)])
def test_tensor_core_backward_workspace_is_the_documented_sum(act, d, C):
    # the bf16 chunk-end adjoints, G when the forward's G is not passed, a float per token for
    # the decay gradient, and with SiLU four bf16 planes (include/ttt.h, ttt_chunk_bwd_noalloc)
    B, H, T = 2, 3, 4 * C
    cfg = _cfg(B=B, H=H, T=T, dk=d, dv=d, C=C, dtype="bf16", act=act)
    adj, G, dg = B * H * (T // C) * d * d * 2, B * H * T * d * 2, B * H * T * 4
    planes = 4 * B * H * T * d * 2 if act == "silu" else 0
    assert ttt.ttt_workspace_bytes(cfg, 2) == adj + dg + planes
    if act == "id":
        assert ttt.ttt_workspace_bytes(cfg, 1) == adj + G + dg
    else:  # the SiLU backward without the forward's G and Zq is refused on these shapes
        with pytest.raises(ttt.TTTError):
            ttt.ttt_workspace_bytes(cfg, 1)


def test_silu_tensor_core_backward_without_saved_tensors_is_refused():
    # a SiLU backward on a tensor-core shape needs the forward's G and Zq; without them the call
    # returns TTT_ERR_UNSUPPORTED before anything is launched (the pointers are never read)
    cfg = _cfg(dtype="bf16", dk=128, dv=128, C=256, T=512, act="silu")
    A = 4096
    ws = ttt.ttt_workspace_bytes(cfg, 2)
    args = [A] * 7 + [None, A, None, None, None] + [A] * 5 + [None]  # ... G_saved = NULL ...
    assert ttt.lib.ttt_chunk_bwd(ctypes.byref(cfg), *args, A, ws, None) == ttt.ERR_UNSUPPORTED
    # with G_saved the same call passes the host checks (it would launch; not run here)
    assert ttt.ttt_workspace_bytes(cfg, 2) > 0
