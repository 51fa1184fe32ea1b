"""GPU checks of two properties the layer's contract promises beyond parity.

* Streaming (checkpoint and resume): the state is explicit, so running the forward over
  [0, T1) and then over [T1, T) from the first call's W_final equals one call over [0, T) when
  T1 is a chunk boundary; the backward likewise runs the second half first and hands its dW0
  (the adjoint of the state at T1) to the first half as dW_final.
* No writes outside the outputs: every output is placed between guard regions filled with a
  byte pattern, and the patterns must be intact after the calls (the library has no debug
  build with device-side bounds checks; this is the check that stands in for one).
"""
import numpy as np
import pytest
import torch

import synth
import weight_sequence_layers_b200 as ttt
from _runners import abi_config, oracle_bwd, oracle_fwd, run_bwd, run_fwd
from _util import rel_err

pytestmark = pytest.mark.gpu

TOL = 2e-2       # against the oracle (bf16 storage)
F32_TOL = 1e-4
SPLIT_TOL = 1e-3  # one call against two: the same kernels on the same values


def _cut(inp, a, b):
    out = {}
    for k, v in inp.items():
        if v is None:
            out[k] = None
        elif k in ("W0", "dW_T"):
            out[k] = v.clone()
        else:
            out[k] = v[:, :, a:b].contiguous()
    return out


CASES = [
    # (workload, overrides): identity and SiLU on the tensor cores, float32 on SIMT, and the
    # per-feature decay on the tensor cores
    (synth.TRAIN_1P45B, dict(B=1, H=2, T=1024)),
    (synth.SILU_IP_FWD, dict(B=1, H=2, T=1024, loss="mse")),
    (synth.TINY_FP32, dict(B=1, H=2, T=512)),
    (synth.FWD_410M, dict(B=1, H=2, T=1024, decay="vector", w0_std=0.05)),
]
IDS = ["tc-id", "tc-silu", "simt-f32", "tc-vector"]


@pytest.mark.parametrize("base,kw", CASES, ids=IDS)
def test_two_calls_with_the_state_carried_equal_one_call(base, kw):
    cfg = base.replace(**kw)
    T1 = cfg.T // 2
    assert T1 % cfg.C == 0
    inp = synth.ttt_inputs(cfg, device="cuda", seed=101)
    inp["dW_T"].normal_(generator=torch.Generator("cuda").manual_seed(102))
    full = run_fwd(cfg, inp)
    half = cfg.replace(T=T1)
    a, b = _cut(inp, 0, T1), _cut(inp, T1, cfg.T)
    fa = run_fwd(half, a)
    b["W0"] = fa["W_final"].clone()
    fb = run_fwd(half, b)
    tol = F32_TOL if cfg.dtype == "f32" else SPLIT_TOL
    assert rel_err(torch.cat([fa["O"], fb["O"]], 2), full["O"]) <= tol
    assert rel_err(fb["W_final"], full["W_final"]) <= tol
    ref = oracle_fwd(cfg, inp)
    assert rel_err(torch.cat([fa["O"], fb["O"]], 2), ref["O"]) <= (F32_TOL if cfg.dtype == "f32" else TOL)
    # backward: the second half first, its dW0 is the first half's dW_final
    g_full = run_bwd(cfg, inp, full["W_chunks"], full["G_saved"])
    b["dW_T"] = inp["dW_T"]
    gb = run_bwd(half, b, fb["W_chunks"], fb["G_saved"])
    a["dW_T"] = gb["dW0"].clone()
    ga = run_bwd(half, a, fa["W_chunks"], fa["G_saved"])
    for k in ("dQ", "dK", "dV", "dbeta"):
        got = torch.cat([ga[k], gb[k]], 2)
        assert rel_err(got, g_full[k]) <= tol, (k, rel_err(got, g_full[k]))
    assert rel_err(ga["dW0"], g_full["dW0"]) <= tol
    r = oracle_bwd(cfg, inp)
    assert rel_err(ga["dW0"], r["dW0"]) <= (F32_TOL if cfg.dtype == "f32" else TOL)


PATTERN = 0xA5
PAD = 4096


def _guarded(shape, dtype):
    """A tensor of `shape` inside a byte buffer with PAD pattern bytes on each side."""
    n = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
    buf = torch.full((PAD + n + PAD,), PATTERN, device="cuda", dtype=torch.uint8)
    return buf, buf[PAD:PAD + n].view(dtype).view(shape)


def _intact(buf):
    return bool((buf[:PAD] == PATTERN).all()) and bool((buf[-PAD:] == PATTERN).all())


@pytest.mark.parametrize("base,kw", CASES, ids=IDS)
def test_no_output_is_written_past_its_ends(base, kw):
    cfg = base.replace(**kw)
    inp = synth.ttt_inputs(cfg, device="cuda", seed=103)
    c = abi_config(cfg)
    sd = synth.storage_dtype(cfg)
    B, H, T, dk, dv, C = cfg.B, cfg.H, cfg.T, cfg.dk, cfg.dv, cfg.C
    bufs = {}

    def out(name, shape, dtype):
        bufs[name], t = _guarded(shape, dtype)
        return t

    O = out("O", (B, H, T, dv), sd)
    Wf = out("W_final", (B, H, dk, dv), torch.float32)
    Wc = out("W_chunks", (B, H, T // C, dk, dv), sd)
    Gs = out("G_saved", (-(-ttt.ttt_saved_bytes(c) // (B * H * T * dv * sd.itemsize)), B, H, T, dv),
             sd)
    n = ttt.ttt_workspace_bytes(c, 0)
    ws = out("ws_fwd", (max(n, 16),), torch.uint8)
    ttt.ttt_chunk_fwd(c, inp["Q"], inp["K"], inp["V"], inp["beta"], inp["gamma"], inp["W0"], O, Wf,
                      Wc, Gs, ws, n)
    dQ = out("dQ", (B, H, T, dk), sd)
    dK = out("dK", (B, H, T, dk), sd)
    dV = out("dV", (B, H, T, dv), sd)
    dbeta = out("dbeta", (B, H, T), torch.float32)
    dW0 = out("dW0", (B, H, dk, dv), torch.float32)
    dg = out("dgamma", tuple(inp["gamma"].shape), torch.float32) if inp["gamma"] is not None else None
    nb = ttt.ttt_workspace_bytes(c, 2)
    wsb = out("ws_bwd", (max(nb, 16),), torch.uint8)
    ttt.ttt_chunk_bwd(c, inp["Q"], inp["K"], inp["V"], inp["beta"], inp["gamma"], inp["W0"], Wc, Gs,
                      inp["dO"], inp["dW_T"], O if dg is not None else None,
                      Wf if dg is not None else None, dQ, dK, dV, dbeta, dW0, dg, wsb, nb)
    torch.cuda.synchronize()
    assert ttt.ttt_get_device_error() == ttt.OK
    bad = [k for k, v in bufs.items() if not _intact(v)]
    assert not bad, bad
    # and the outputs themselves are the right ones
    ref = oracle_fwd(cfg, inp)
    tol = F32_TOL if cfg.dtype == "f32" else TOL
    assert rel_err(O, ref["O"]) <= tol


def test_inplace_outputs_are_not_written_past_their_ends():
    icfg = synth.INPLACE_QWEN4B.replace(T=512, d_ff=512, d_model=256, C=256, lr=0.05)
    iin = synth.inplace_inputs(icfg, device="cuda")
    bufs = {}
    bufs["W"], W = _guarded((icfg.d_model, icfg.d_ff), torch.float32)
    W.copy_(iin["W"])
    bufs["O"], O = _guarded((icfg.T, icfg.d_model), torch.bfloat16)
    bufs["Wc"], Wc = _guarded((icfg.T // icfg.C, icfg.d_model, icfg.d_ff), torch.bfloat16)
    n = ttt.inplace_ttt_workspace_bytes(icfg.T, icfg.d_ff, icfg.d_model, icfg.C)
    bufs["ws"], ws = _guarded((n,), torch.uint8)
    ttt.inplace_ttt_fwd(icfg.T, icfg.d_ff, icfg.d_model, icfg.C, icfg.lr, iin["Z"], iin["Vhat"], W,
                        O, ws, n, W_chunks=Wc)
    bufs["dZ"], dZ = _guarded((icfg.T, icfg.d_ff), torch.bfloat16)
    bufs["dVh"], dVh = _guarded((icfg.T, icfg.d_model), torch.bfloat16)
    bufs["dW"], dW = _guarded((icfg.d_model, icfg.d_ff), torch.float32)
    dO = torch.randn((icfg.T, icfg.d_model), device="cuda").to(torch.bfloat16)
    ttt.inplace_ttt_bwd(icfg.T, icfg.d_ff, icfg.d_model, icfg.C, icfg.lr, iin["Z"], iin["Vhat"], Wc,
                        dO, None, dZ, dVh, dW, ws, n)
    torch.cuda.synchronize()
    assert ttt.ttt_get_device_error() == ttt.OK
    bad = [k for k, v in bufs.items() if not _intact(v)]
    assert not bad, bad
