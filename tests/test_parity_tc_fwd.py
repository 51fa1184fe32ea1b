"""GPU parity of the tcgen05 forward (bf16 storage, fp32 state) against the oracle."""
import numpy as np
import pytest
import torch

import synth
from _runners import head_slice, oracle_fwd, reference_g, run_fwd
from _util import rel_err

pytestmark = pytest.mark.gpu

TOL = 2e-2
COMBOS = [("mse", "id"), ("mse", "silu"), ("ip", "id"), ("ip", "silu")]
SHAPES = [
    # B, H, T, d, C
    (1, 2, 1024, 128, 256),
    (2, 1, 512, 64, 256),
    (1, 2, 640, 128, 128),
    (1, 1, 384, 64, 128),
]


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("loss,act", COMBOS)
@pytest.mark.parametrize("decay", [False, True])
def test_tc_forward_small(shape, loss, act, decay):
    B, H, T, d, C = shape
    cfg = synth.SILU_IP_FWD.replace(B=B, H=H, T=T, dk=d, dv=d, C=C, loss=loss, act=act,
                                    decay=decay, w0_std=1.0 / d)
    inp = synth.ttt_inputs(cfg, device="cuda", seed=7 * T + d)
    got = run_fwd(cfg, inp)
    ref = oracle_fwd(cfg, inp)
    ref["G"] = reference_g(cfg, inp, ref["W_chunks"])
    for k in ("O", "W_final", "W_chunks", "G"):
        assert rel_err(got[k], ref[k]) <= TOL, (k, rel_err(got[k], ref[k]))


def test_tc_forward_strong_decay_is_finite_and_matches():
    """Decay strong enough that Gamma over a chunk underflows: no 1/Gamma is ever formed."""
    cfg = synth.SILU_IP_FWD.replace(B=1, H=1, T=512, loss="mse", act="id")
    inp = synth.ttt_inputs(cfg, device="cuda", seed=11)
    inp["gamma"] = torch.full_like(inp["gamma"], 0.5)
    got = run_fwd(cfg, inp)
    ref = oracle_fwd(cfg, inp)
    assert torch.isfinite(got["O"].float()).all()
    for k in ("O", "W_final"):
        assert rel_err(got[k], ref[k]) <= TOL, k


@pytest.mark.parametrize("cfg", [synth.FWD_410M, synth.SILU_IP_FWD, synth.TRAIN_1P45B],
                         ids=lambda c: c.name)
def test_tc_forward_full_size_sampled_heads(cfg):
    inp = synth.ttt_inputs(cfg, device="cuda")
    got = run_fwd(cfg, inp)
    rng = np.random.default_rng(cfg.seed)
    heads = [(int(rng.integers(cfg.B)), int(rng.integers(cfg.H))) for _ in range(3)]
    sub = head_slice(inp, heads)
    sub_cfg = cfg.replace(B=1, H=len(heads))
    ref = oracle_fwd(sub_cfg, sub)
    ref["G"] = reference_g(sub_cfg, sub, ref["W_chunks"])
    for k in ("O", "W_final", "W_chunks", "G"):
        g = torch.stack([got[k][b, h] for b, h in heads]).unsqueeze(0)
        assert rel_err(g, ref[k]) <= TOL, (k, rel_err(g, ref[k]))


@pytest.mark.parametrize("d,C,loss,act", [(64, 256, "mse", "id"), (128, 256, "ip", "silu"),
                                          (128, 128, "mse", "silu"), (64, 128, "ip", "id")])
def test_tc_inference_forward_without_saved_tensors(d, C, loss, act):
    # the forward with no W_chunks and no G_saved (nothing kept for a backward) gives the same
    # O and W_final as the oracle
    cfg = synth.SILU_IP_FWD.replace(B=1, H=2, T=4 * C, dk=d, dv=d, C=C, loss=loss, act=act)
    inp = synth.ttt_inputs(cfg, device="cuda", seed=d + C)
    got = run_fwd(cfg, inp, save_g=False, save_w=False)
    ref = oracle_fwd(cfg, inp)
    for k in ("O", "W_final"):
        assert rel_err(got[k], ref[k]) <= TOL, k
