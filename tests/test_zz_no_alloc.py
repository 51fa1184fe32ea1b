"""ttt_chunk_bwd_noalloc: the backward for callers that cannot allocate device memory when they
call the library (a host framework that owns all device memory, a plugin handed only its
buffers). It must give the same gradients as ttt_chunk_bwd with a caller workspace, bit for
bit, on consecutive calls that share its fixed scratch array (each call finds the bytes the
previous one left behind), and refuse configs whose scratch would not fit. This file is
collected last on purpose."""
import ctypes

import pytest
import torch

import synth
import weight_sequence_layers_b200 as ttt
from _runners import abi_config, run_bwd, run_fwd
from _util import rel_err

pytestmark = pytest.mark.gpu

TOL = 2e-2
GRADS = ("dQ", "dK", "dV", "dbeta", "dW0", "dgamma")


def noalloc_bwd(cfg, inp, W_chunks, G, fwd):
    c = abi_config(cfg)
    sd = synth.storage_dtype(cfg)
    B, H, T, dk, dv = cfg.B, cfg.H, cfg.T, cfg.dk, cfg.dv
    out = dict(dQ=torch.full((B, H, T, dk), float("nan"), device="cuda", dtype=sd),
               dK=torch.full((B, H, T, dk), float("nan"), device="cuda", dtype=sd),
               dV=torch.full((B, H, T, dv), float("nan"), device="cuda", dtype=sd),
               dbeta=torch.full((B, H, T), float("nan"), device="cuda"),
               dW0=torch.full((B, H, dk, dv), float("nan"), device="cuda"),
               dgamma=torch.full((B, H, T), float("nan"), device="cuda"))
    st = ttt.lib.ttt_chunk_bwd_noalloc(
        ctypes.byref(c), inp["Q"].data_ptr(), inp["K"].data_ptr(), inp["V"].data_ptr(),
        inp["beta"].data_ptr(), inp["gamma"].data_ptr(), inp["W0"].data_ptr(), W_chunks.data_ptr(),
        G.data_ptr() if G is not None else None, inp["dO"].data_ptr(), inp["dW_T"].data_ptr(),
        fwd["O"].data_ptr(), fwd["W_final"].data_ptr(), out["dQ"].data_ptr(),
        out["dK"].data_ptr(), out["dV"].data_ptr(), out["dbeta"].data_ptr(),
        out["dW0"].data_ptr(), out["dgamma"].data_ptr(),
        torch.cuda.current_stream().cuda_stream)
    assert st == ttt.OK, ttt.status_string(st)
    torch.cuda.synchronize()
    assert ttt.ttt_get_device_error() == ttt.OK
    return out


def _same(got, ref, where):
    # the same kernels on the same inputs (no atomics): the results agree bit for bit
    for k in GRADS:
        assert torch.equal(got[k], ref[k]), (where, k, rel_err(got[k], ref[k]))
        assert rel_err(got[k], ref[k]) <= TOL, (where, k)


def test_noalloc_backward_matches_the_workspace_backward_call_after_call():
    # Scratch needed (limit 8 MiB): 4 heads x 4 chunks x 128 x 128 x 2 bytes = 512 KiB of
    # chunk-end adjoints, plus 1 MiB of G when the forward's saved tensors are not passed, plus
    # 16 KiB for dgamma, plus 4 MiB of SiLU planes. The calls run in an order that makes each
    # one start from the bytes an earlier call of another kind left behind: without the saved
    # tensors (fills the G region), with them, SiLU (fills the four planes), then without them
    # again, and the first one once more.
    cfg = synth.TRAIN_1P45B.replace(B=1, H=4, T=1024)
    silu = synth.SILU_IP_FWD.replace(B=1, H=4, T=1024, loss="mse")
    plan = [(cfg, 21, False), (cfg, 22, True), (silu, 23, True), (cfg, 24, False), (cfg, 21, False)]
    for c, seed, saved in plan:
        inp = synth.ttt_inputs(c, device="cuda", seed=seed)
        inp["dW_T"].normal_(generator=torch.Generator("cuda").manual_seed(seed))
        fwd = run_fwd(c, inp, save_g=saved)
        ref = run_bwd(c, inp, fwd["W_chunks"], fwd["G_saved"], fwd=fwd)
        got = noalloc_bwd(c, inp, fwd["W_chunks"], fwd["G_saved"], fwd)
        _same(got, ref, (c.name, seed, saved))


def test_noalloc_backward_refuses_configs_beyond_its_scratch():
    big = abi_config(synth.TRAIN_1P45B)  # needs 32 MiB of scratch even with G passed in
    A = 4096  # never dereferenced: the size check comes first
    # Q K V beta gamma W0 W_chunks G_saved dO dW_final O W_final dQ dK dV dbeta dW0 dgamma stream
    st = ttt.lib.ttt_chunk_bwd_noalloc(ctypes.byref(big), A, A, A, A, A, A, A, A, A, None, None, None,
                                       A, A, A, A, A, None, None)
    assert st == ttt.ERR_WORKSPACE
    silu = abi_config(synth.TRAIN_1P45B.replace(B=1, H=1, T=256, act="silu"))
    st = ttt.lib.ttt_chunk_bwd_noalloc(ctypes.byref(silu), A, A, A, A, A, A, A, None, A, None, None,
                                       None, A, A, A, A, A, None, None)
    assert st == ttt.ERR_UNSUPPORTED
