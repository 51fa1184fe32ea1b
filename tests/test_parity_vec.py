"""GPU parity of the tensor-core forward and backward with a per-feature (vector) decay (bf16,
d = 64, identity activation) against the oracle's per-token loop and its reverse mode."""
import numpy as np
import pytest
import torch

import synth
import weight_sequence_layers_b200 as ttt
from _runners import head_slice, oracle_bwd, oracle_fwd, reference_g, run_bwd, run_fwd
from _util import rel_err

pytestmark = pytest.mark.gpu

TOL = 2e-2


def _cfg(**kw):
    base = dict(decay="vector", w0_std=0.05)
    base.update(kw)
    return synth.FWD_410M.replace(**base)


@pytest.mark.parametrize("B,H,T,C", [(1, 2, 512, 256), (2, 1, 384, 128), (1, 1, 256, 256),
                                     (1, 2, 128, 128)])
@pytest.mark.parametrize("loss", ["mse", "ip"])
def test_vector_decay_forward_small(B, H, T, C, loss):
    cfg = _cfg(B=B, H=H, T=T, C=C, loss=loss)
    inp = synth.ttt_inputs(cfg, device="cuda", seed=T + C + B)
    got = run_fwd(cfg, inp)
    ref = oracle_fwd(cfg, inp)
    ref["G"] = reference_g(cfg, inp, ref["W_chunks"])
    for k in ("O", "W_final", "W_chunks", "G"):
        assert rel_err(got[k], ref[k]) <= TOL, (k, rel_err(got[k], ref[k]))
    # the inference forward (no chunk states or G kept) gives the same O and W_final
    inf = run_fwd(cfg, inp, save_g=False, save_w=False)
    for k in ("O", "W_final"):
        assert rel_err(inf[k], ref[k]) <= TOL, k


def test_vector_decay_forward_full_size_sampled_heads():
    cfg = synth.FWD_410M.replace(decay="vector")
    inp = synth.ttt_inputs(cfg, device="cuda")
    got = run_fwd(cfg, inp)
    rng = np.random.default_rng(46)
    heads = [(int(rng.integers(cfg.B)), int(rng.integers(cfg.H))) for _ in range(3)]
    sub = head_slice(inp, heads)
    ref = oracle_fwd(cfg.replace(B=1, H=len(heads)), sub)
    for k in ("O", "W_final", "W_chunks"):
        g = torch.stack([got[k][b, h] for b, h in heads]).unsqueeze(0)
        assert rel_err(g, ref[k]) <= TOL, (k, rel_err(g, ref[k]))


def test_vector_decay_forward_strong_but_in_range():
    # gamma = 0.5 on every feature: exp(L) over a 256-token chunk underflows, while every scaled
    # operand factor spans 64 tokens (0.5^64 ~ 5e-20, inside the range)
    cfg = _cfg(B=1, H=1, T=512, C=256)
    inp = synth.ttt_inputs(cfg, device="cuda", seed=5)
    inp["gamma"] = torch.full_like(inp["gamma"], 0.5)
    inp["gamma"][..., ::3] = 0.97  # features decaying at different rates
    got = run_fwd(cfg, inp)
    ref = oracle_fwd(cfg, inp)
    assert torch.isfinite(got["O"].float()).all()
    for k in ("O", "W_final"):
        assert rel_err(got[k], ref[k]) <= TOL, (k, rel_err(got[k], ref[k]))


def test_vector_decay_forward_out_of_range_is_reported():
    # a feature decaying by 1e-3 per token: its factor over 64 tokens is far beyond exp(80); the
    # kernel clamps it and reports a range error instead of producing infinities silently
    cfg = _cfg(B=1, H=1, T=256, C=256)
    inp = synth.ttt_inputs(cfg, device="cuda", seed=6)
    inp["gamma"][..., 7] = 1e-3
    c = ttt.make_config(cfg.B, cfg.H, cfg.T, cfg.dk, cfg.dv, cfg.C, cfg.dtype, cfg.loss, cfg.act,
                        cfg.lr_bias, "vector")
    O = torch.empty_like(inp["V"])
    n = ttt.ttt_workspace_bytes(c, 0)
    ws = torch.empty(n, device="cuda", dtype=torch.uint8)
    ttt.ttt_chunk_fwd(c, inp["Q"], inp["K"], inp["V"], inp["beta"], inp["gamma"], inp["W0"], O,
                      None, None, None, ws, n)
    assert ttt.ttt_get_device_error() == ttt.ERR_RANGE
    assert ttt.ttt_get_device_error() == ttt.OK  # reported once, then cleared


GRADS = ("dQ", "dK", "dV", "dbeta", "dW0", "dgamma")


@pytest.mark.parametrize("B,H,T,C", [(1, 2, 512, 256), (2, 1, 384, 128), (1, 1, 256, 256),
                                     (1, 2, 128, 128)])
@pytest.mark.parametrize("loss", ["mse", "ip"])
def test_vector_decay_backward_small(B, H, T, C, loss):
    cfg = _cfg(B=B, H=H, T=T, C=C, loss=loss)
    inp = synth.ttt_inputs(cfg, device="cuda", seed=T + C + B + 1)
    inp["dW_T"].normal_(generator=torch.Generator("cuda").manual_seed(9))
    got = run_fwd(cfg, inp)
    g = run_bwd(cfg, inp, got["W_chunks"], fwd=got)
    r = oracle_bwd(cfg, inp)
    for k in GRADS:
        assert rel_err(g[k], r[k]) <= TOL, (k, rel_err(g[k], r[k]))
    # without the decay gradient the other gradients are the same
    g2 = run_bwd(cfg, inp, got["W_chunks"])
    for k in GRADS[:-1]:
        assert rel_err(g2[k], g[k]) <= 1e-6, k
    # given the forward's saved buffer (G, the decayed operands, R) instead of forming them
    g3 = run_bwd(cfg, inp, got["W_chunks"], got["G_saved"], fwd=got)
    for k in GRADS:
        assert rel_err(g3[k], r[k]) <= TOL, ("saved", k, rel_err(g3[k], r[k]))


def test_vector_decay_backward_without_final_state_gradient():
    cfg = _cfg(B=1, H=2, T=512, C=256)
    inp = synth.ttt_inputs(cfg, device="cuda", seed=12)
    inp["dW_T"] = None
    got = run_fwd(cfg, inp)
    g = run_bwd(cfg, inp, got["W_chunks"], fwd=got)
    r = oracle_bwd(cfg, inp)
    for k in GRADS:
        assert rel_err(g[k], r[k]) <= TOL, (k, rel_err(g[k], r[k]))


@pytest.mark.parametrize("loss", ["mse", "ip"])
def test_vector_decay_backward_full_size_sampled_heads(loss):
    cfg = synth.FWD_410M.replace(decay="vector", loss=loss)
    inp = synth.ttt_inputs(cfg, device="cuda", seed=47)
    inp["dW_T"].normal_(generator=torch.Generator("cuda").manual_seed(48))
    got = run_fwd(cfg, inp)
    g = run_bwd(cfg, inp, got["W_chunks"], got["G_saved"], fwd=got)
    rng = np.random.default_rng(49)
    heads = [(int(rng.integers(cfg.B)), int(rng.integers(cfg.H))) for _ in range(2)]
    sub = head_slice(inp, heads)
    r = oracle_bwd(cfg.replace(B=1, H=len(heads)), sub)
    for k in GRADS:
        got_k = torch.stack([g[k][b, h] for b, h in heads]).unsqueeze(0)
        err = rel_err(got_k, r[k])
        print(f"{loss} {k}: rel err {err:.2e} (bound {TOL:.0e}, margin {TOL / max(err, 1e-30):.1f}x)")
        assert err <= TOL, (k, err)


@pytest.mark.parametrize("loss", ["mse", "ip"])
def test_vector_decay_of_ones_equals_no_decay(loss):
    # gamma = 1 on every feature: the per-feature path (scaled operands, its own kernels) must
    # give what the scalar-decay kernels give without a decay
    cfg = _cfg(B=1, H=2, T=512, C=256, loss=loss)
    inp = synth.ttt_inputs(cfg, device="cuda", seed=14)
    inp["gamma"] = torch.ones_like(inp["gamma"])
    inp["dW_T"].normal_(generator=torch.Generator("cuda").manual_seed(15))
    vec = run_fwd(cfg, inp)
    gv = run_bwd(cfg, inp, vec["W_chunks"], vec["G_saved"], fwd=vec)
    sc_cfg = cfg.replace(decay=False)
    sc_inp = dict(inp, gamma=None)
    sc = run_fwd(sc_cfg, sc_inp)
    gs = run_bwd(sc_cfg, sc_inp, sc["W_chunks"], sc["G_saved"])
    assert rel_err(vec["O"], sc["O"]) <= 1e-2
    assert rel_err(vec["W_final"], sc["W_final"]) <= 1e-2
    for k in GRADS[:-1]:
        assert rel_err(gv[k], gs[k]) <= 1e-2, (k, rel_err(gv[k], gs[k]))
