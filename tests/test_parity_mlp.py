"""GPU parity of TTT-MLP (two-layer fast weight act(k W1) W2) against the oracle's fp64
per-token loop and its autograd backward: the SIMT kernels (float32, and bf16 shapes outside
the tensor-core envelope) and the batched tcgen05 GEMM program (bf16, d = 64, hidden 128 or 256,
C = 128 or 256)."""
import numpy as np
import pytest
import torch

import oracle
import synth
import weight_sequence_layers_b200 as ttt
from _runners import abi_config, head_slice, lr_bias32
from _util import rel_err

pytestmark = pytest.mark.gpu

F32_TOL = 1e-4
BF16_TOL = 2e-2


def run_mlp(cfg, hidden, inp, w):
    c = abi_config(cfg)
    sd = synth.storage_dtype(cfg)
    B, H, T, dk, dv, C = cfg.B, cfg.H, cfg.T, cfg.dk, cfg.dv, cfg.C
    dev = "cuda"
    f = dict(O=torch.empty((B, H, T, dv), device=dev, dtype=sd),
             W1_final=torch.empty_like(w["W1"]), W2_final=torch.empty_like(w["W2"]),
             W1c=torch.empty((B, H, T // C, dk, hidden), device=dev),
             W2c=torch.empty((B, H, T // C, hidden, dv), device=dev))
    n = ttt.ttt_mlp_workspace_bytes(c, hidden)
    ws = torch.empty(n, device=dev, dtype=torch.uint8)
    ttt.ttt_mlp_fwd(c, hidden, inp["Q"], inp["K"], inp["V"], inp["beta"], inp["gamma"], w["W1"],
                    w["W2"], f["O"], f["W1_final"], f["W2_final"], f["W1c"], f["W2c"], ws, n)
    g = dict(dQ=torch.empty((B, H, T, dk), device=dev, dtype=sd),
             dK=torch.empty((B, H, T, dk), device=dev, dtype=sd),
             dV=torch.empty((B, H, T, dv), device=dev, dtype=sd),
             dbeta=torch.empty((B, H, T), device=dev),
             dW1=torch.empty_like(w["W1"]), dW2=torch.empty_like(w["W2"]))
    ttt.ttt_mlp_bwd(c, hidden, inp["Q"], inp["K"], inp["V"], inp["beta"], inp["gamma"], f["W1c"],
                    f["W2c"], inp["dO"], w["dW1_T"], w["dW2_T"], g["dQ"], g["dK"], g["dV"],
                    g["dbeta"], g["dW1"], g["dW2"], ws, n)
    torch.cuda.synchronize()
    assert ttt.ttt_get_device_error() == ttt.OK
    return f, g


def reference(cfg, inp, w):
    kw = dict(C=cfg.C, loss=cfg.loss, act=cfg.act, lr_bias=lr_bias32(cfg))
    O, W1f, W2f = oracle.ttt_mlp_fwd(inp["Q"], inp["K"], inp["V"], inp["beta"], inp["gamma"],
                                     w["W1"], w["W2"], **kw)
    g = oracle.ttt_mlp_bwd(inp["Q"], inp["K"], inp["V"], inp["beta"], inp["gamma"], w["W1"],
                           w["W2"], inp["dO"], w["dW1_T"], w["dW2_T"], **kw)
    return dict(O=O.numpy(), W1_final=W1f.numpy(), W2_final=W2f.numpy()), g


COMBOS = [("mse", "id"), ("mse", "silu"), ("ip", "id"), ("ip", "silu")]


@pytest.mark.parametrize("loss,act", COMBOS)
@pytest.mark.parametrize("decay", [False, True])
def test_mlp_fp32(loss, act, decay):
    cfg = synth.TTT_MLP_410M.replace(B=1, H=2, T=64, dk=16, dv=24, C=16, dtype="f32", loss=loss,
                                     act=act, decay=decay, w0_std=0.2)
    hidden = 40
    inp = synth.ttt_inputs(cfg, device="cuda", seed=31)
    w = synth.ttt_mlp_weights(cfg, hidden, device="cuda", seed=31)
    w["dW1_T"].normal_(generator=torch.Generator("cuda").manual_seed(1))
    w["dW2_T"].normal_(generator=torch.Generator("cuda").manual_seed(2))
    f, g = run_mlp(cfg, hidden, inp, w)
    rf, rg = reference(cfg, inp, w)
    for k in ("O", "W1_final", "W2_final"):
        assert rel_err(f[k], rf[k]) <= F32_TOL, k
    for k in ("dQ", "dK", "dV", "dbeta", "dW1", "dW2"):
        assert rel_err(g[k], rg[k]) <= F32_TOL, (k, rel_err(g[k], rg[k]))


@pytest.mark.parametrize("loss", ["mse", "ip"])
def test_mlp_bf16(loss):
    cfg = synth.TTT_MLP_410M.replace(B=1, H=1, T=256, C=64, loss=loss, w0_std=0.05)
    hidden = 256
    inp = synth.ttt_inputs(cfg, device="cuda", seed=32)
    w = synth.ttt_mlp_weights(cfg, hidden, device="cuda", seed=32)
    f, g = run_mlp(cfg, hidden, inp, w)
    rf, rg = reference(cfg, inp, w)
    for k in ("O", "W1_final", "W2_final"):
        assert rel_err(f[k], rf[k]) <= BF16_TOL, k
    for k in ("dQ", "dK", "dV", "dbeta", "dW1", "dW2"):
        assert rel_err(g[k], rg[k]) <= BF16_TOL, (k, rel_err(g[k], rg[k]))


def test_mlp_full_size_sampled_head():
    cfg = synth.TTT_MLP_410M
    hidden = synth.TTT_MLP_HIDDEN
    inp = synth.ttt_inputs(cfg, device="cuda")
    w = synth.ttt_mlp_weights(cfg, hidden, device="cuda")
    f, g = run_mlp(cfg, hidden, inp, w)
    b, h = 5, 11
    sub = head_slice(inp, [(b, h)])
    wsub = {k: v[b:b + 1, h:h + 1].contiguous() for k, v in w.items()}
    rf, rg = reference(cfg.replace(B=1, H=1), sub, wsub)
    for k in ("O", "W1_final", "W2_final"):
        assert rel_err(f[k][b:b + 1, h:h + 1], rf[k]) <= BF16_TOL, k
    for k in ("dQ", "dK", "dV", "dbeta", "dW1", "dW2"):
        assert rel_err(g[k][b:b + 1, h:h + 1], rg[k]) <= BF16_TOL, k


def test_mlp_single_chunk_fp32():
    cfg = synth.TTT_MLP_410M.replace(B=1, H=1, T=32, dk=8, dv=8, C=32, dtype="f32", w0_std=0.2)
    hidden = 16
    inp = synth.ttt_inputs(cfg, device="cuda", seed=33)
    w = synth.ttt_mlp_weights(cfg, hidden, device="cuda", seed=33)
    w["dW2_T"].normal_(generator=torch.Generator("cuda").manual_seed(3))
    f, g = run_mlp(cfg, hidden, inp, w)
    rf, rg = reference(cfg, inp, w)
    for k in ("O", "W1_final", "W2_final"):
        assert rel_err(f[k], rf[k]) <= F32_TOL, k
    for k in ("dQ", "dK", "dV", "dbeta", "dW1", "dW2"):
        assert rel_err(g[k], rg[k]) <= F32_TOL, k


TC_CASES = [(256, 128, 128, loss, act, decay) for loss, act in COMBOS for decay in (False, True)]
TC_CASES += [(512, 256, 256, "mse", "silu", True), (512, 256, 256, "ip", "id", False),
             (512, 128, 256, "mse", "silu", True), (512, 256, 128, "ip", "silu", True),
             (256, 256, 256, "mse", "id", True)]  # (one chunk)


@pytest.mark.parametrize("T,C,hidden,loss,act,decay", TC_CASES)
def test_mlp_tensor_core_shapes(T, C, hidden, loss, act, decay):
    cfg = synth.TTT_MLP_410M.replace(B=1, H=2, T=T, C=C, loss=loss, act=act, decay=decay,
                                     w0_std=0.05)
    inp = synth.ttt_inputs(cfg, device="cuda", seed=T + C + hidden)
    w = synth.ttt_mlp_weights(cfg, hidden, device="cuda", seed=T + hidden)
    w["dW1_T"].normal_(generator=torch.Generator("cuda").manual_seed(5))
    w["dW2_T"].normal_(generator=torch.Generator("cuda").manual_seed(6))
    f, g = run_mlp(cfg, hidden, inp, w)
    rf, rg = reference(cfg, inp, w)
    for k in ("O", "W1_final", "W2_final"):
        assert rel_err(f[k], rf[k]) <= BF16_TOL, (k, rel_err(f[k], rf[k]))
    for k in ("dQ", "dK", "dV", "dbeta", "dW1", "dW2"):
        assert rel_err(g[k], rg[k]) <= BF16_TOL, (k, rel_err(g[k], rg[k]))
