"""The seeded input generators draw what the workloads state: shapes, storage types and value
distributions (Q, K, V rows, beta, the decay gamma = sigmoid(N(3, 0.5)), the fast-weight init,
the In-Place Z = SiLU(N(0,1)) * N(0,1), Vhat and W_down ~ N(0, 0.02), the NTP-target inputs and
the TTT-MLP weights), and the same seed gives the same tensors. N(mu, s) takes s as the standard
deviation. Statistics are taken over enough entries for a few-percent tolerance."""
import math

import numpy as np
import pytest
import torch

import synth


def _f64(x):
    return x.double().numpy()


def _logit(g):
    return np.log(g / (1.0 - g))


def test_lr_bias_gives_eta0_of_one_tenth():
    assert 2.0 / (1.0 + math.exp(-synth.LR_BIAS_ETA0_0P1)) == pytest.approx(0.1, rel=1e-12)


@pytest.mark.parametrize("cfg", [synth.TINY_FP32, synth.FWD_410M, synth.SILU_IP_FWD,
                                 synth.TRAIN_1P45B], ids=lambda c: c.name)
def test_layer_workload_recipe(cfg):
    small = cfg.replace(B=min(cfg.B, 2), H=min(cfg.H, 4), T=min(cfg.T, 1024))
    inp = synth.ttt_inputs(small)
    B, H, T, dk, dv = small.B, small.H, small.T, small.dk, small.dv
    sd = torch.float32 if cfg.dtype == "f32" else torch.bfloat16
    shapes = dict(Q=(B, H, T, dk), K=(B, H, T, dk), V=(B, H, T, dv), dO=(B, H, T, dv),
                  beta=(B, H, T), W0=(B, H, dk, dv), dW_T=(B, H, dk, dv))
    for k, s in shapes.items():
        assert tuple(inp[k].shape) == s, k
        assert inp[k].is_contiguous(), k
    for k in ("Q", "K", "V", "dO"):
        assert inp[k].dtype == sd, k
    for k in ("beta", "W0", "dW_T"):
        assert inp[k].dtype == torch.float32, k
    # rows of Q and K (and of V for the tiny workload) have unit L2 norm, up to storage rounding
    tol = 1e-5 if cfg.dtype == "f32" else 1e-2
    norm = lambda x: np.linalg.norm(_f64(x), axis=-1)
    for k in ("Q", "K") + (("V",) if cfg.normalize == "qkv" else ()):
        np.testing.assert_allclose(norm(inp[k]), 1.0, atol=tol, err_msg=k)
    if cfg.normalize == "qk":
        assert _f64(inp["V"]).std() == pytest.approx(1.0, rel=0.03)
    assert _f64(inp["beta"]).mean() == pytest.approx(0.0, abs=0.03)
    assert _f64(inp["beta"]).std() == pytest.approx(1.0, rel=0.03)
    assert _f64(inp["dO"]).std() == pytest.approx(1.0, rel=0.03)
    assert not inp["dW_T"].any()
    if cfg.decay:
        z = _logit(_f64(inp["gamma"]))
        assert tuple(inp["gamma"].shape) == (B, H, T)
        assert z.mean() == pytest.approx(3.0, abs=0.03)
        assert z.std() == pytest.approx(0.5, rel=0.05)
    else:
        assert inp["gamma"] is None
    if cfg.w0_std == 0:
        assert not inp["W0"].any()
    else:
        assert _f64(inp["W0"]).std() == pytest.approx(cfg.w0_std, rel=0.05)


def test_workload_constants():
    # sizes and settings of the five workloads
    t = synth.TINY_FP32
    assert (t.B, t.H, t.T, t.dk, t.dv, t.C, t.dtype, t.loss, t.act, t.decay) == \
        (1, 2, 512, 64, 64, 64, "f32", "mse", "id", False)
    assert t.w0_std == pytest.approx(1 / 64)
    f = synth.FWD_410M
    assert (f.B, f.H, f.T, f.dk, f.dv, f.C, f.dtype, f.loss, f.decay, f.w0_std) == \
        (8, 16, 2048, 64, 64, 256, "bf16", "mse", True, 0.0)
    s = synth.SILU_IP_FWD
    assert (s.B, s.H, s.T, s.dk, s.dv, s.C, s.loss, s.act, s.decay) == \
        (4, 16, 4096, 128, 128, 256, "ip", "silu", True)
    assert s.w0_std == pytest.approx(1 / 128)
    r = synth.TRAIN_1P45B
    assert (r.B, r.H, r.T, r.dk, r.dv, r.C, r.loss, r.act, r.decay, r.backward) == \
        (4, 16, 4096, 128, 128, 256, "mse", "id", True, True)
    i = synth.INPLACE_QWEN4B
    assert (i.T, i.d_ff, i.d_model, i.C) == (32768, 9728, 2560, 1024)
    assert i.lr == pytest.approx(1e-3)


def test_vector_decay_has_one_factor_per_key_feature():
    cfg = synth.FWD_410M.replace(B=1, H=2, T=512, decay="vector")
    g = synth.ttt_inputs(cfg)["gamma"]
    assert tuple(g.shape) == (1, 2, 512, cfg.dk) and g.dtype == torch.float32
    z = _logit(_f64(g))
    assert z.mean() == pytest.approx(3.0, abs=0.03) and z.std() == pytest.approx(0.5, rel=0.05)


def test_same_seed_same_tensors_other_seed_differs():
    cfg = synth.FWD_410M.replace(B=1, H=2, T=256)
    a, b, c = synth.ttt_inputs(cfg), synth.ttt_inputs(cfg), synth.ttt_inputs(cfg, seed=99)
    for k in ("Q", "K", "V", "beta", "gamma", "dO"):
        assert torch.equal(a[k], b[k]), k
        assert not torch.equal(a[k], c[k]), k
    icfg = synth.INPLACE_QWEN4B.replace(T=256, d_ff=256, d_model=128)
    x, y = synth.inplace_inputs(icfg), synth.inplace_inputs(icfg)
    for k in x:
        assert torch.equal(x[k], y[k]), k


def _silu_times_normal_moments():
    """E[SiLU(a)^2] for a ~ N(0, 1), by quadrature: the variance of SiLU(a) * b, b ~ N(0, 1)
    independent (the product has mean 0)."""
    a = np.linspace(-12, 12, 200001)
    pdf = np.exp(-a * a / 2) / math.sqrt(2 * math.pi)
    silu = a / (1 + np.exp(-a))
    return np.trapezoid(silu ** 2 * pdf, a)


def test_inplace_workload_recipe():
    icfg = synth.INPLACE_QWEN4B.replace(T=512, d_ff=1024, d_model=256)
    inp = synth.inplace_inputs(icfg)
    T, F, M = icfg.T, icfg.d_ff, icfg.d_model
    assert tuple(inp["Z"].shape) == (T, F) and inp["Z"].dtype == torch.bfloat16
    assert tuple(inp["Vhat"].shape) == (T, M) and inp["Vhat"].dtype == torch.bfloat16
    assert tuple(inp["W"].shape) == (M, F) and inp["W"].dtype == torch.float32
    assert tuple(inp["dO"].shape) == (T, M) and inp["dO"].dtype == torch.bfloat16
    z = _f64(inp["Z"])
    assert z.mean() == pytest.approx(0.0, abs=0.01)
    assert z.var() == pytest.approx(_silu_times_normal_moments(), rel=0.03)
    assert _f64(inp["Vhat"]).std() == pytest.approx(0.02, rel=0.03)
    assert _f64(inp["W"]).std() == pytest.approx(0.02, rel=0.03)
    assert _f64(inp["dO"]).std() == pytest.approx(1.0, rel=0.03)


def test_ntp_target_and_mlp_recipe():
    icfg = synth.INPLACE_QWEN4B.replace(T=1024, d_model=512)
    k = 4
    tin = synth.inplace_target_inputs(icfg, k=k)
    d = icfg.d_model
    assert tuple(tin["X0"].shape) == (1024, d) and tin["X0"].dtype == torch.bfloat16
    assert tuple(tin["conv_w"].shape) == (k, d) and tin["conv_w"].dtype == torch.float32
    assert tuple(tin["W_target"].shape) == (d, d) and tin["W_target"].dtype == torch.bfloat16
    assert _f64(tin["X0"]).std() == pytest.approx(0.02, rel=0.03)
    assert _f64(tin["conv_w"]).std() == pytest.approx(1 / math.sqrt(k), rel=0.05)
    assert _f64(tin["W_target"]).std() == pytest.approx(1 / math.sqrt(d), rel=0.03)
    assert _f64(tin["dVhat"]).std() == pytest.approx(1.0, rel=0.03)
    cfg = synth.TTT_MLP_410M.replace(B=2, H=4)
    w = synth.ttt_mlp_weights(cfg, synth.TTT_MLP_HIDDEN)
    assert tuple(w["W1"].shape) == (2, 4, cfg.dk, synth.TTT_MLP_HIDDEN)
    assert tuple(w["W2"].shape) == (2, 4, synth.TTT_MLP_HIDDEN, cfg.dv)
    assert synth.TTT_MLP_HIDDEN == 4 * cfg.dk
    for key in ("W1", "W2"):
        assert _f64(w[key]).std() == pytest.approx(0.02, rel=0.03), key
    assert not w["dW1_T"].any() and not w["dW2_T"].any()
