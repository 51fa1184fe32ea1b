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


def run(cfg, inp):
    W = inp["W"].clone()
    O = torch.empty((cfg.T, cfg.d_model), device="cuda", dtype=torch.bfloat16)
    n = ttt.inplace_ttt_workspace_bytes(cfg.T, cfg.d_ff, cfg.d_model, cfg.C)
    ws = torch.empty(n, device="cuda", dtype=torch.uint8)
    ttt.inplace_ttt_fwd(cfg.T, cfg.d_ff, cfg.d_model, cfg.C, cfg.lr, inp["Z"], inp["Vhat"], W, O, ws, n)
    torch.cuda.synchronize()
    assert ttt.ttt_get_device_error() == ttt.OK
    return O, W


SMALL = [
    # T, d_ff, d_model, C, lr
    (512, 256, 256, 128, 0.1),
    (384, 320, 384, 128, 0.05),    # ragged N tiles on both GEMMs
    (1024, 512, 128, 256, 0.02),
    (128, 64, 128, 128, 0.1),      # one chunk: a plain GEMM
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
