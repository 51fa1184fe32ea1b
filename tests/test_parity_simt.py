"""GPU parity of the SIMT kernels (float32 workloads, and bf16 shapes outside the tensor-core
envelope) against the oracle, element by element."""
import pytest
import torch

import synth
from _runners import oracle_bwd, oracle_fwd, reference_g, run_bwd, run_fwd
from _util import rel_err

pytestmark = pytest.mark.gpu

F32_TOL = 1e-4
BF16_TOL = 2e-2


def test_tiny_fp32_workload_forward():
    cfg = synth.TINY_FP32
    inp = synth.ttt_inputs(cfg, device="cuda")
    got = run_fwd(cfg, inp)
    ref = oracle_fwd(cfg, inp)
    for k in ("O", "W_final", "W_chunks"):
        assert rel_err(got[k], ref[k]) <= F32_TOL, k
    # the inference forward (no chunk states, no G kept for a backward)
    got = run_fwd(cfg, inp, save_g=False, save_w=False)
    for k in ("O", "W_final"):
        assert rel_err(got[k], ref[k]) <= F32_TOL, k


SHAPES = [
    # B, H, T, dk, dv, C
    (1, 2, 96, 16, 24, 32),
    (2, 1, 192, 64, 40, 64),
    (1, 1, 60, 8, 8, 20),      # C not a multiple of the 32-row query tile
    (1, 1, 512, 128, 128, 256),  # the backward's scratch only partly in shared memory
    (4, 8, 128, 32, 64, 32),     # enough heads for the forward's 32-column value slices
]
COMBOS = [("mse", "id"), ("mse", "silu"), ("ip", "id"), ("ip", "silu")]


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("loss,act", COMBOS)
@pytest.mark.parametrize("decay", [False, True, "vector"])
def test_fp32_forward_backward(shape, loss, act, decay):
    B, H, T, dk, dv, C = shape
    cfg = synth.TINY_FP32.replace(B=B, H=H, T=T, dk=dk, dv=dv, C=C, loss=loss, act=act,
                                  decay=decay, w0_std=0.05, normalize="qk")
    inp = synth.ttt_inputs(cfg, device="cuda", seed=T + dk)
    inp["dW_T"].normal_(generator=torch.Generator("cuda").manual_seed(3))
    got = run_fwd(cfg, inp)
    ref = oracle_fwd(cfg, inp)
    ref["G"] = reference_g(cfg, inp, ref["W_chunks"])
    for k in ("O", "W_final", "W_chunks", "G"):
        assert rel_err(got[k], ref[k]) <= F32_TOL, k
    g = run_bwd(cfg, inp, got["W_chunks"], got["G_saved"] if decay else None, fwd=got)
    r = oracle_bwd(cfg, inp)
    for k in ("dQ", "dK", "dV", "dbeta", "dW0") + (("dgamma",) if decay else ()):
        assert rel_err(g[k], r[k]) <= F32_TOL, k


@pytest.mark.parametrize("loss,act", COMBOS)
def test_bf16_shapes_outside_the_tensor_core_envelope(loss, act):
    cfg = synth.FWD_410M.replace(B=1, H=2, T=256, dk=32, dv=48, C=64, loss=loss, act=act,
                                 w0_std=0.05)
    inp = synth.ttt_inputs(cfg, device="cuda")
    got = run_fwd(cfg, inp)
    ref = oracle_fwd(cfg, inp)
    for k in ("O", "W_final"):
        assert rel_err(got[k], ref[k]) <= BF16_TOL, k
    g = run_bwd(cfg, inp, got["W_chunks"], fwd=got)
    r = oracle_bwd(cfg, inp)
    for k in ("dQ", "dK", "dV", "dbeta", "dW0") + (("dgamma",) if inp["gamma"] is not None else ()):
        assert rel_err(g[k], r[k]) <= BF16_TOL, k


@pytest.mark.parametrize("loss,act", COMBOS)
def test_vector_decay_on_tensor_core_shapes(loss, act):
    # bf16, d = 64, C = 256 with a per-feature decay: the forward runs on the tensor cores with
    # the identity activation and on the SIMT kernels with SiLU; the backward (decay gradient
    # included) runs on the SIMT kernels
    cfg = synth.FWD_410M.replace(B=1, H=2, T=512, loss=loss, act=act, decay="vector", w0_std=0.05)
    inp = synth.ttt_inputs(cfg, device="cuda", seed=77)
    inp["dW_T"].normal_(generator=torch.Generator("cuda").manual_seed(4))
    got = run_fwd(cfg, inp)
    ref = oracle_fwd(cfg, inp)
    for k in ("O", "W_final", "W_chunks"):
        assert rel_err(got[k], ref[k]) <= BF16_TOL, k
    g = run_bwd(cfg, inp, got["W_chunks"], got["G_saved"], fwd=got)
    r = oracle_bwd(cfg, inp)
    for k in ("dQ", "dK", "dV", "dbeta", "dW0", "dgamma"):
        assert rel_err(g[k], r[k]) <= BF16_TOL, k
