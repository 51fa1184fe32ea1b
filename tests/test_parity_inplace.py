"""GPU parity of the In-Place TTT tensor-core kernel against the oracle."""
import numpy as np
import pytest
import torch

import oracle
import synth
import weight_sequence_layers_b200 as ttt
from _util import rel_err

pytestmark = pytest.mark.gpu

O_TOL = 2e-2     # bf16 output
W_TOL = 1e-4     # float32 state built from exact bf16 products


def run(cfg, inp, save=False):
    W = inp["W"].clone()
    O = torch.empty((cfg.T, cfg.d_model), device="cuda", dtype=torch.bfloat16)
    Wc = torch.empty((cfg.T // cfg.C, cfg.d_model, cfg.d_ff), device="cuda",
                     dtype=torch.bfloat16) if save else None
    n = ttt.inplace_ttt_workspace_bytes(cfg.T, cfg.d_ff, cfg.d_model, cfg.C)
    ws = torch.empty(n, device="cuda", dtype=torch.uint8)
    ttt.inplace_ttt_fwd(cfg.T, cfg.d_ff, cfg.d_model, cfg.C, cfg.lr, inp["Z"], inp["Vhat"], W, O, ws, n,
                        W_chunks=Wc)
    torch.cuda.synchronize()
    assert ttt.ttt_get_device_error() == ttt.OK
    return (O, W, Wc) if save else (O, W)


def run_bwd(cfg, inp, Wc, dWf):
    dZ = torch.full((cfg.T, cfg.d_ff), float("nan"), device="cuda", dtype=torch.bfloat16)
    dVh = torch.full((cfg.T, cfg.d_model), float("nan"), device="cuda", dtype=torch.bfloat16)
    dW = torch.full((cfg.d_model, cfg.d_ff), float("nan"), device="cuda", dtype=torch.float32)
    n = ttt.inplace_ttt_workspace_bytes(cfg.T, cfg.d_ff, cfg.d_model, cfg.C)
    ws = torch.empty(n, device="cuda", dtype=torch.uint8)
    ttt.inplace_ttt_bwd(cfg.T, cfg.d_ff, cfg.d_model, cfg.C, cfg.lr, inp["Z"], inp["Vhat"], Wc,
                        inp["dO"], dWf, dZ, dVh, dW, ws, n)
    torch.cuda.synchronize()
    assert ttt.ttt_get_device_error() == ttt.OK
    return dZ, dVh, dW


SMALL = [
    # T, d_ff, d_model, C, lr
    (512, 256, 256, 128, 0.1),
    (384, 320, 384, 128, 0.05),    # ragged N tiles on both GEMMs
    (1024, 512, 128, 256, 0.02),
    (128, 64, 128, 128, 0.1),      # one chunk: a plain GEMM
    (4096, 512, 256, 128, 0.05),   # 32 chunks: the forward's cross-chunk dependency counts
    (2048, 448, 640, 256, 0.05),   # 8 chunks, d_model = 2.5 pair tiles: a half-empty pair tile
]


@pytest.mark.parametrize("T,d_ff,d_model,C,lr", SMALL)
def test_inplace_small(T, d_ff, d_model, C, lr):
    cfg = synth.INPLACE_QWEN4B.replace(T=T, d_ff=d_ff, d_model=d_model, C=C, lr=lr)
    inp = synth.inplace_inputs(cfg, device="cuda", seed=T + d_ff)
    O, W = run(cfg, inp)
    Oref, Wref = oracle.inplace_fwd(inp["Z"], inp["Vhat"], inp["W"], C=C, lr=float(np.float32(lr)))
    assert rel_err(O, Oref) <= O_TOL
    assert rel_err(W, Wref) <= W_TOL


def test_inplace_full_size_sampled_rows():
    cfg = synth.INPLACE_QWEN4B
    inp = synth.inplace_inputs(cfg, device="cuda")
    O, W = run(cfg, inp)
    rows = np.sort(np.random.default_rng(0).choice(cfg.d_model, 24, replace=False))
    Oref, Wref = oracle.inplace_fwd(inp["Z"], inp["Vhat"], inp["W"], C=cfg.C,
                                    lr=float(np.float32(cfg.lr)), rows=rows)
    assert rel_err(O[:, rows], Oref) <= O_TOL
    assert rel_err(W[rows], Wref) <= W_TOL
    # associativity over all rows (page "In-Place Test-Time Training": the update is a sum)
    Wsum = inp["W"] + cfg.lr * (inp["Vhat"].float().T @ inp["Z"].float())
    assert rel_err(W, Wsum) <= 1e-3


@pytest.mark.parametrize("T,d_ff,d_model,C,lr", SMALL)
def test_inplace_forward_saves_the_applied_weights(T, d_ff, d_model, C, lr):
    cfg = synth.INPLACE_QWEN4B.replace(T=T, d_ff=d_ff, d_model=d_model, C=C, lr=lr)
    inp = synth.inplace_inputs(cfg, device="cuda", seed=T + d_ff)
    O, W = run(cfg, inp)
    O2, W2, Wc = run(cfg, inp, save=True)
    # the saved states are the operands the apply tiles read: outputs identical either way
    assert torch.equal(O, O2) and torch.equal(W, W2)
    lr32 = float(np.float32(lr))
    for i in range(T // C):
        # W_i: the state after the first i chunks (the initial W for i = 0)
        ref = inp["W"].double().cpu().numpy() if i == 0 else oracle.inplace_fwd(
            inp["Z"][: i * C], inp["Vhat"][: i * C], inp["W"], C=C, lr=lr32)[1]
        assert rel_err(Wc[i], ref) <= 4e-3, i  # bf16 rounding of an fp32 state


@pytest.mark.parametrize("T,d_ff,d_model,C,lr", SMALL)
@pytest.mark.parametrize("with_dwf", [False, True])
def test_inplace_backward_small(T, d_ff, d_model, C, lr, with_dwf):
    cfg = synth.INPLACE_QWEN4B.replace(T=T, d_ff=d_ff, d_model=d_model, C=C, lr=lr)
    inp = synth.inplace_inputs(cfg, device="cuda", seed=T + d_ff + 1)
    dWf = (0.1 * torch.randn((d_model, d_ff), device="cuda",
                             generator=torch.Generator("cuda").manual_seed(6))) if with_dwf else None
    _, _, Wc = run(cfg, inp, save=True)
    dZ, dVh, dW = run_bwd(cfg, inp, Wc, dWf)
    ref = oracle.inplace_bwd(inp["Z"], inp["Vhat"], inp["W"], inp["dO"], dWf, C=C,
                             lr=float(np.float32(lr)))
    assert rel_err(dZ, ref["dZ"]) <= O_TOL
    assert rel_err(dVh, ref["dVhat"]) <= O_TOL
    assert rel_err(dW, ref["dW"]) <= W_TOL


def test_inplace_backward_full_size_sampled():
    cfg = synth.INPLACE_QWEN4B
    inp = synth.inplace_inputs(cfg, device="cuda")
    _, _, Wc = run(cfg, inp, save=True)
    dZ, dVh, dW = run_bwd(cfg, inp, Wc, None)
    lr32 = float(np.float32(cfg.lr))
    rng = np.random.default_rng(1)
    rows = np.sort(rng.choice(cfg.d_model, 16, replace=False))
    ref = oracle.inplace_bwd(inp["Z"], inp["Vhat"], inp["W"], inp["dO"], None, C=cfg.C, lr=lr32,
                             rows=rows)
    assert rel_err(dVh[:, rows], ref["dVhat"]) <= O_TOL
    assert rel_err(dW[rows], ref["dW"]) <= W_TOL
    # tokens from the first, a middle and the last chunk
    tokens = [3, 1000, cfg.T // 2 + 17, cfg.T - 5]
    dz = oracle.inplace_bwd_dz_tokens(inp["Z"], inp["Vhat"], inp["W"], inp["dO"], None, C=cfg.C,
                                      lr=lr32, tokens=tokens)
    assert rel_err(dZ[tokens], dz) <= O_TOL


def run_target(T, d, k, tin):
    V = torch.full((T, d), float("nan"), device="cuda", dtype=torch.bfloat16)
    n = ttt.inplace_ttt_target_workspace_bytes(T, d)
    ws = torch.empty(n, device="cuda", dtype=torch.uint8)
    ttt.inplace_ttt_target(T, d, k, tin["X0"], tin["conv_w"], tin["W_target"], V, ws, n)
    torch.cuda.synchronize()
    assert ttt.ttt_get_device_error() == ttt.OK
    return V


@pytest.mark.parametrize("T,d,k", [(256, 128, 1), (256, 128, 2), (512, 256, 4), (384, 384, 8), (128, 640, 3)])
def test_inplace_target_small(T, d, k):
    cfg = synth.INPLACE_QWEN4B.replace(T=T, d_model=d)
    tin = synth.inplace_target_inputs(cfg, k=k, device="cuda", seed=T + d + k)
    V = run_target(T, d, k, tin)
    ref, _ = oracle.inplace_target(tin["X0"], tin["conv_w"], tin["W_target"])
    assert rel_err(V, ref) <= O_TOL


def test_inplace_target_full_size_sampled_tokens():
    cfg = synth.INPLACE_QWEN4B
    k = 4
    tin = synth.inplace_target_inputs(cfg, k=k, device="cuda")
    V = run_target(cfg.T, cfg.d_model, k, tin)
    # Vhat_t needs X0 rows t .. t+k-1 only: slice windows around sampled tokens, and the tail
    for t0 in (0, 4093, cfg.T // 2 + 5, cfg.T - 32):
        m = min(32, cfg.T - t0)
        hi = min(cfg.T, t0 + m + k - 1)
        ref, _ = oracle.inplace_target(tin["X0"][t0:hi], tin["conv_w"], tin["W_target"])
        assert rel_err(V[t0:t0 + m], ref[:m]) <= O_TOL, t0


def run_target_bwd(T, d, k, tin):
    dX0 = torch.full((T, d), float("nan"), device="cuda", dtype=torch.bfloat16)
    dw = torch.full((k, d), float("nan"), device="cuda", dtype=torch.float32)
    dWt = torch.full((d, d), float("nan"), device="cuda", dtype=torch.float32)
    n = ttt.inplace_ttt_target_bwd_workspace_bytes(T, d, k)
    ws = torch.empty(n, device="cuda", dtype=torch.uint8)
    ttt.inplace_ttt_target_bwd(T, d, k, tin["X0"], tin["conv_w"], tin["W_target"], tin["dVhat"],
                               dX0, dw, dWt, ws, n)
    torch.cuda.synchronize()
    assert ttt.ttt_get_device_error() == ttt.OK
    return dict(dX0=dX0, dconv_w=dw, dW_target=dWt)


@pytest.mark.parametrize("T,d,k", [(256, 128, 1), (256, 128, 2), (512, 256, 4), (384, 384, 8), (128, 640, 3)])
def test_inplace_target_backward_small(T, d, k):
    cfg = synth.INPLACE_QWEN4B.replace(T=T, d_model=d)
    tin = synth.inplace_target_inputs(cfg, k=k, device="cuda", seed=2 * T + d + k)
    got = run_target_bwd(T, d, k, tin)
    ref = oracle.inplace_target_bwd(tin["X0"], tin["conv_w"], tin["W_target"], tin["dVhat"])
    for key in ("dX0", "dconv_w", "dW_target"):
        assert rel_err(got[key], ref[key]) <= O_TOL, key


def test_inplace_target_backward_full_size_sampled_channels():
    cfg = synth.INPLACE_QWEN4B
    k = 4
    tin = synth.inplace_target_inputs(cfg, k=k, device="cuda")
    got = run_target_bwd(cfg.T, cfg.d_model, k, tin)
    ch = np.sort(np.random.default_rng(2).choice(cfg.d_model, 12, replace=False))
    ref = oracle.inplace_target_bwd(tin["X0"], tin["conv_w"], tin["W_target"], tin["dVhat"],
                                    channels=ch)
    assert rel_err(got["dX0"][:, ch], ref["dX0"]) <= O_TOL
    assert rel_err(got["dconv_w"][:, ch], ref["dconv_w"]) <= O_TOL
    assert rel_err(got["dW_target"][ch], ref["dW_target"]) <= O_TOL


@pytest.mark.parametrize("starts", [[2], [1, 3], [1, 2, 3]])
def test_inplace_document_resets(starts):
    cfg = synth.INPLACE_QWEN4B.replace(T=512, d_ff=256, d_model=256, C=128, lr=0.1)
    inp = synth.inplace_inputs(cfg, device="cuda", seed=61)
    T, F, M, C = cfg.T, cfg.d_ff, cfg.d_model, cfg.C
    n = ttt.inplace_ttt_docs_workspace_bytes(T, F, M, C)
    ws = torch.empty(n, device="cuda", dtype=torch.uint8)
    W = inp["W"].clone()
    O = torch.empty((T, M), device="cuda", dtype=torch.bfloat16)
    Wc = torch.empty((T // C, M, F), device="cuda", dtype=torch.bfloat16)
    ttt.inplace_ttt_fwd_docs(T, F, M, C, cfg.lr, inp["Z"], inp["Vhat"], W, O, Wc, starts, ws, n)
    dWf = 0.1 * torch.randn((M, F), device="cuda", generator=torch.Generator("cuda").manual_seed(7))
    dZ = torch.empty((T, F), device="cuda", dtype=torch.bfloat16)
    dVh = torch.empty((T, M), device="cuda", dtype=torch.bfloat16)
    dW = torch.empty((M, F), device="cuda")
    ttt.inplace_ttt_bwd_docs(T, F, M, C, cfg.lr, inp["Z"], inp["Vhat"], Wc, inp["dO"], dWf, dZ, dVh,
                             dW, starts, ws, n)
    torch.cuda.synchronize()
    assert ttt.ttt_get_device_error() == ttt.OK
    lr32 = float(np.float32(cfg.lr))
    Oref, Wref = oracle.inplace_fwd(inp["Z"], inp["Vhat"], inp["W"], C=C, lr=lr32, doc_starts=starts)
    assert rel_err(O, Oref) <= O_TOL
    assert rel_err(W, Wref) <= W_TOL
    ref = oracle.inplace_bwd(inp["Z"], inp["Vhat"], inp["W"], inp["dO"], dWf, C=C, lr=lr32,
                             doc_starts=starts)
    assert rel_err(dZ, ref["dZ"]) <= O_TOL
    assert rel_err(dVh, ref["dVhat"]) <= O_TOL
    assert rel_err(dW, ref["dW"]) <= W_TOL
    # the applied weights it saved: the state before each chunk, the initial W at a document start
    for i in range(T // C):
        s0 = max([0] + [s for s in starts if s <= i])  # the first chunk of chunk i's document
        ref_i = inp["W"].double().cpu().numpy() if i == s0 else oracle.inplace_fwd(
            inp["Z"][s0 * C: i * C], inp["Vhat"][s0 * C: i * C], inp["W"], C=C, lr=lr32)[1]
        assert rel_err(Wc[i], ref_i) <= 4e-3, i


@pytest.mark.parametrize("starts", [[2], [1, 3], [3, 5, 6]])
def test_inplace_document_resets_without_saved_weights(starts):
    # the forward alone (two rotating bf16 copies instead of the caller's chunk states), 8 chunks
    cfg = synth.INPLACE_QWEN4B.replace(T=1024, d_ff=320, d_model=384, C=128, lr=0.1)
    inp = synth.inplace_inputs(cfg, device="cuda", seed=63)
    T, F, M, C = cfg.T, cfg.d_ff, cfg.d_model, cfg.C
    n = ttt.inplace_ttt_docs_workspace_bytes(T, F, M, C)
    ws = torch.empty(n, device="cuda", dtype=torch.uint8)
    W = inp["W"].clone()
    O = torch.empty((T, M), device="cuda", dtype=torch.bfloat16)
    ttt.inplace_ttt_fwd_docs(T, F, M, C, cfg.lr, inp["Z"], inp["Vhat"], W, O, None, starts, ws, n)
    torch.cuda.synchronize()
    assert ttt.ttt_get_device_error() == ttt.OK
    lr32 = float(np.float32(cfg.lr))
    Oref, Wref = oracle.inplace_fwd(inp["Z"], inp["Vhat"], inp["W"], C=C, lr=lr32, doc_starts=starts)
    assert rel_err(O, Oref) <= O_TOL
    assert rel_err(W, Wref) <= W_TOL


def test_inplace_delta_and_single_rank_context_parallel():
    import datetime
    import os
    import socket

    import torch.distributed as dist
    cfg = synth.INPLACE_QWEN4B.replace(T=512, d_ff=256, d_model=256, C=128, lr=0.1)
    inp = synth.inplace_inputs(cfg, device="cuda", seed=71)
    T, F, M, C = cfg.T, cfg.d_ff, cfg.d_model, cfg.C
    n = ttt.inplace_ttt_workspace_bytes(T, F, M, C)
    ws = torch.empty(n, device="cuda", dtype=torch.uint8)
    dW = torch.empty((M, F), device="cuda")
    ttt.inplace_ttt_delta(T, F, M, cfg.lr, inp["Z"], inp["Vhat"], dW, ws, n)
    lr32 = float(np.float32(cfg.lr))
    _, WF = oracle.inplace_fwd(inp["Z"], inp["Vhat"], np.zeros((M, F)), C=T, lr=lr32)
    torch.cuda.synchronize()
    assert rel_err(dW, WF) <= W_TOL
    # one rank: the context-parallel forward is the plain forward
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=0, world_size=1, timeout=datetime.timedelta(seconds=60))
    try:
        W = inp["W"].clone()
        O = torch.empty((T, M), device="cuda", dtype=torch.bfloat16)
        ttt.inplace_cp_fwd(T, F, M, C, cfg.lr, inp["Z"], inp["Vhat"], W, O, ws, n)
    finally:
        dist.destroy_process_group()
    O2, W2 = run(cfg, inp)
    assert torch.equal(O, O2) and torch.equal(W, W2)
