"""GPU parity of the tcgen05 backward (identity or SiLU activation, MSE or inner-product loss)
against the oracle's reverse-mode of the per-token loop."""
import numpy as np
import pytest
import torch

import synth
from _runners import head_slice, oracle_bwd, oracle_fwd, run_bwd, run_fwd
from _util import rel_err

pytestmark = pytest.mark.gpu

TOL = 2e-2
GRADS = ("dQ", "dK", "dV", "dbeta", "dW0")
SHAPES = [
    # B, H, T, d, C
    (1, 2, 1024, 128, 256),
    (2, 1, 512, 64, 256),
    (1, 2, 640, 128, 128),
    (1, 1, 384, 64, 128),
]


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("loss", ["mse", "ip"])
@pytest.mark.parametrize("decay", [False, True])
@pytest.mark.parametrize("saved_g", [True, False], ids=["g_from_fwd", "g_rebuilt"])
def test_tc_backward_small(shape, loss, decay, saved_g):
    B, H, T, d, C = shape
    cfg = synth.TRAIN_1P45B.replace(B=B, H=H, T=T, dk=d, dv=d, C=C, loss=loss, act="id",
                                    decay=decay, w0_std=1.0 / d)
    inp = synth.ttt_inputs(cfg, device="cuda", seed=5 * T + d)
    inp["dW_T"].normal_(generator=torch.Generator("cuda").manual_seed(9))
    fwd = run_fwd(cfg, inp, save_g=saved_g)
    got = run_bwd(cfg, inp, fwd["W_chunks"], fwd["G_saved"], fwd=fwd)
    ref = oracle_bwd(cfg, inp)
    for k in GRADS + (("dgamma",) if decay else ()):
        assert rel_err(got[k], ref[k]) <= TOL, (k, rel_err(got[k], ref[k]))


def test_tc_backward_full_size_sampled_heads():
    # The whole 16-chunk sequence of the 1.45B workload. The chunk-start states the backward
    # rebuilds Z and G from are stored in bf16 (W_chunks has the storage dtype); the errors
    # below show how much of the 2e-2 budget that and the bf16 operands use after 16 chunks.
    cfg = synth.TRAIN_1P45B
    inp = synth.ttt_inputs(cfg, device="cuda")
    fwd = run_fwd(cfg, inp)
    got = run_bwd(cfg, inp, fwd["W_chunks"], fwd["G_saved"], fwd=fwd)
    rng = np.random.default_rng(44)
    heads = [(int(rng.integers(cfg.B)), int(rng.integers(cfg.H))) for _ in range(2)]
    sub = head_slice(inp, heads)
    ref = oracle_bwd(cfg.replace(B=1, H=len(heads)), sub)
    errs = {}
    for k in GRADS + ("dgamma",):
        g = torch.stack([got[k][b, h] for b, h in heads]).unsqueeze(0)
        errs[k] = rel_err(g, ref[k])
    print("full-length backward errors (max|d| / max|ref|, budget 2e-2):",
          {k: f"{v:.2e}" for k, v in errs.items()})
    for k, v in errs.items():
        assert v <= TOL, (k, v)


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("loss", ["mse", "ip"])
@pytest.mark.parametrize("decay", [False, True])
def test_tc_backward_silu_small(shape, loss, decay):
    # SiLU on the tensor cores reads Zq and G saved by the forward
    B, H, T, d, C = shape
    cfg = synth.SILU_IP_FWD.replace(B=B, H=H, T=T, dk=d, dv=d, C=C, loss=loss, act="silu",
                                    decay=decay, w0_std=1.0 / d)
    inp = synth.ttt_inputs(cfg, device="cuda", seed=3 * T + d)
    inp["dW_T"].normal_(generator=torch.Generator("cuda").manual_seed(10))
    fwd = run_fwd(cfg, inp)
    got = run_bwd(cfg, inp, fwd["W_chunks"], fwd["G_saved"], fwd=fwd)
    ref = oracle_bwd(cfg, inp)
    for k in GRADS + (("dgamma",) if decay else ()):
        assert rel_err(got[k], ref[k]) <= TOL, (k, rel_err(got[k], ref[k]))


def test_tc_backward_silu_full_size_sampled_heads():
    cfg = synth.SILU_IP_FWD
    inp = synth.ttt_inputs(cfg, device="cuda")
    fwd = run_fwd(cfg, inp)
    got = run_bwd(cfg, inp, fwd["W_chunks"], fwd["G_saved"], fwd=fwd)
    rng = np.random.default_rng(45)
    heads = [(int(rng.integers(cfg.B)), int(rng.integers(cfg.H))) for _ in range(2)]
    sub = head_slice(inp, heads)
    ref = oracle_bwd(cfg.replace(B=1, H=len(heads)), sub)
    for k in GRADS + ("dgamma",):
        g = torch.stack([got[k][b, h] for b, h in heads]).unsqueeze(0)
        assert rel_err(g, ref[k]) <= TOL, (k, rel_err(g, ref[k]))


@pytest.mark.parametrize("d,C", [(64, 128), (64, 256), (128, 128), (128, 256)])
@pytest.mark.parametrize("act", ["id", "silu"])
def test_tc_single_chunk(d, C, act):
    # T == C: the chain runs one iteration and the decay gradient's state term comes from
    # W_final and dW_final
    cfg = synth.SILU_IP_FWD.replace(B=1, H=2, T=C, dk=d, dv=d, C=C, loss="mse", act=act,
                                    decay=True, w0_std=1.0 / d)
    inp = synth.ttt_inputs(cfg, device="cuda", seed=d + C)
    inp["dW_T"].normal_(generator=torch.Generator("cuda").manual_seed(12))
    fwd = run_fwd(cfg, inp)
    ref_f = oracle_fwd(cfg, inp)
    for k in ("O", "W_final", "W_chunks"):
        assert rel_err(fwd[k], ref_f[k]) <= TOL, k
    got = run_bwd(cfg, inp, fwd["W_chunks"], fwd["G_saved"], fwd=fwd)
    ref = oracle_bwd(cfg, inp)
    for k in GRADS + ("dgamma",):
        assert rel_err(got[k], ref[k]) <= TOL, (k, rel_err(got[k], ref[k]))


def test_silu_backward_without_saved_zq_is_refused():
    # the SiLU backward on a tensor-core shape reads the forward's Zq from G_saved; called
    # without it on real device tensors it returns TTT_ERR_UNSUPPORTED and touches no output
    import weight_sequence_layers_b200 as ttt
    from _runners import abi_config
    cfg = synth.SILU_IP_FWD.replace(B=1, H=2, T=512, loss="mse")
    inp = synth.ttt_inputs(cfg, device="cuda", seed=71)
    fwd = run_fwd(cfg, inp)
    c = abi_config(cfg)
    n = ttt.ttt_workspace_bytes(c, 2)
    ws = torch.empty(n, device="cuda", dtype=torch.uint8)
    outs = [torch.full_like(inp[k], float("nan")) for k in ("Q", "K", "V", "beta")]
    dW0 = torch.full_like(inp["W0"], float("nan"))
    with pytest.raises(ttt.TTTError) as e:
        ttt.ttt_chunk_bwd(c, inp["Q"], inp["K"], inp["V"], inp["beta"], inp["gamma"], inp["W0"],
                          fwd["W_chunks"], None, inp["dO"], None, None, None, *outs, dW0, None,
                          ws, n)
    assert e.value.status == ttt.ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert all(torch.isnan(t.float()).all() for t in outs + [dW0])
