"""The host-side arithmetic behind every roofline fraction bench.py prints, checked on the CPU.

bench.py divides algorithmic flops and bytes by measured time. Here the flop formulas are
checked against a count of the multiply-adds of a chunk dual form evaluated step by step in
numpy. The forward is the one of page "Modular TTT: Rethinking Test-Time Training as
Composable Modules", section "方法步骤详情" (Algorithm 1). The backward is the reverse
mode of that forward. Both evaluations are checked against the oracle first, so the count
covers a computation that really produces the layer's outputs and gradients. The byte
formulas are checked against the sizes of the tensors that a call reads and writes.
"""
import numpy as np
import pytest
import torch

import bench
import oracle
import synth


class _Counter:
    """Counts the multiply-adds of contractions; elementwise work is not counted (the
    algorithmic figures count only the contractions)."""

    def __init__(self):
        self.macs = 0

    def mm(self, a, b):
        """Dense a @ b."""
        self.macs += a.shape[0] * a.shape[1] * b.shape[1]
        return a @ b

    def masked_out(self, a, b, mask):
        """a @ b evaluated only at the output entries under `mask` (each costs the inner
        size); the others are zero."""
        self.macs += int(mask.sum()) * a.shape[1]
        return np.where(mask, a @ b, 0.0)

    def tri(self, A, b, mask):
        """A @ b where A is zero outside `mask`: only the terms under the mask are summed."""
        self.macs += int(mask.sum()) * b.shape[1]
        return np.where(mask, A, 0.0) @ b


def _chunk_fwd(cnt, q, k, v, beta, gamma, W, b):
    """One chunk of the dual form for MSE loss and identity activation: O, W_end and what the
    backward reads. Every gradient of the chunk is taken at its start weight W."""
    C = q.shape[0]
    eta = 2.0 / (1.0 + np.exp(-(beta + b)))
    L = np.cumsum(np.log(gamma))
    low = np.tril(np.ones((C, C), dtype=bool))
    G = cnt.mm(k, W) - v
    P = cnt.masked_out(q, k.T, low)
    Mw = np.where(low, eta[None, :] * np.exp(L[:, None] - L[None, :]), 0.0)
    S = P * Mw
    O = np.exp(L)[:, None] * cnt.mm(q, W) - cnt.tri(S, G, low)
    u = eta * np.exp(L[-1] - L)
    W_end = np.exp(L[-1]) * W - cnt.mm(k.T, u[:, None] * G)
    return O, W_end, dict(eta=eta, L=L, low=low, G=G, P=P, Mw=Mw, S=S, u=u, W=W)


def _chunk_bwd(cnt, q, k, dO, dW_end, sv):
    """Reverse mode of _chunk_fwd from its saved quantities (nothing recomputed): dQ, dK, dV,
    dbeta of the chunk and the adjoint of its start weight."""
    eta, L, low, G, P, Mw, S, u, W = (sv[n] for n in ("eta", "L", "low", "G", "P", "Mw", "S",
                                                        "u", "W"))
    Gam = np.exp(L)[:, None]
    dQ = Gam * cnt.mm(dO, W.T)
    dW = cnt.mm(q.T, Gam * dO) + np.exp(L[-1]) * dW_end
    dS = -cnt.masked_out(dO, G.T, low)
    KdW = cnt.mm(k, dW_end)
    dG = -cnt.tri(S.T, dO, low.T) - u[:, None] * KdW
    dK = -cnt.mm(u[:, None] * G, dW_end.T)
    du = -(G * KdW).sum(1)
    dP = dS * Mw
    dQ = dQ + cnt.tri(dP, k, low)
    dK = dK + cnt.tri(dP.T, q, low.T)
    dK = dK + cnt.mm(dG, W.T)
    dW = dW + cnt.mm(k.T, dG)
    deta = (dS * P * np.where(low, np.exp(L[:, None] - L[None, :]), 0.0)).sum(0) + \
        du * np.exp(L[-1] - L)
    return dQ, dK, -dG, deta * eta * (1.0 - eta / 2.0), dW


def _counted_layer(cfg, inp):
    """Forward then backward of every head through the counted chunk evaluations."""
    f = lambda x: None if x is None else np.asarray(x, dtype=np.float64)
    Q, K, V, beta, W0, dO, dWT = (f(inp[n]) for n in ("Q", "K", "V", "beta", "W0", "dO", "dW_T"))
    gamma = f(inp["gamma"]) if inp["gamma"] is not None else np.ones_like(beta)
    B, H, T, dk = Q.shape
    C, b = cfg.C, float(np.float32(cfg.lr_bias))
    fcnt, bcnt = _Counter(), _Counter()
    out = {n: np.zeros_like(x) for n, x in (("O", V), ("dQ", Q), ("dK", K), ("dV", V),
                                           ("dbeta", beta))}
    out["W_final"], out["dW0"] = np.zeros_like(W0), np.zeros_like(W0)
    for bi in range(B):
        for h in range(H):
            W, saved = W0[bi, h], []
            for c in range(T // C):
                t = slice(c * C, (c + 1) * C)
                O, W, sv = _chunk_fwd(fcnt, Q[bi, h, t], K[bi, h, t], V[bi, h, t],
                                      beta[bi, h, t], gamma[bi, h, t], W, b)
                out["O"][bi, h, t] = O
                saved.append(sv)
            out["W_final"][bi, h] = W
            dW = dWT[bi, h]
            for c in reversed(range(T // C)):
                t = slice(c * C, (c + 1) * C)
                dq, dk_, dv, db, dW = _chunk_bwd(bcnt, Q[bi, h, t], K[bi, h, t], dO[bi, h, t], dW,
                                                 saved[c])
                out["dQ"][bi, h, t], out["dK"][bi, h, t], out["dV"][bi, h, t] = dq, dk_, dv
                out["dbeta"][bi, h, t] = db
            out["dW0"][bi, h] = dW
    return out, 2 * fcnt.macs, 2 * bcnt.macs


SMALL = [  # B, H, T, dk, dv, C
    (1, 2, 32, 8, 6, 8),
    (2, 1, 48, 5, 7, 16),
    (1, 1, 24, 4, 4, 24),
]


@pytest.mark.parametrize("shape", SMALL)
@pytest.mark.parametrize("decay", [True, False])
def test_flop_formulas_count_the_multiply_adds_of_the_layer(shape, decay):
    B, H, T, dk, dv, C = shape
    cfg = synth.TINY_FP32.replace(B=B, H=H, T=T, dk=dk, dv=dv, C=C, decay=decay, w0_std=0.1,
                                  normalize="qk")
    inp = synth.ttt_inputs(cfg, seed=T + dk)
    inp["dW_T"].normal_(generator=torch.Generator().manual_seed(7))
    got, fwd_flops, bwd_flops = _counted_layer(cfg, inp)
    # the counted evaluations compute the layer: they agree with the oracle's per-token loop
    b32 = float(np.float32(cfg.lr_bias))
    O, Wf, _, _ = oracle.ttt_fwd(inp["Q"], inp["K"], inp["V"], inp["beta"], inp["gamma"],
                                 inp["W0"], C=C, lr_bias=b32)
    ref = oracle.ttt_bwd(inp["Q"], inp["K"], inp["V"], inp["beta"], inp["gamma"], inp["W0"],
                         inp["dO"], inp["dW_T"], C=C, lr_bias=b32)
    ref.update(O=O, W_final=Wf)
    for n in ("O", "W_final", "dQ", "dK", "dV", "dbeta", "dW0"):
        np.testing.assert_allclose(got[n], ref[n], rtol=1e-9, atol=1e-11, err_msg=n)
    w = bench.layer_work(cfg)
    assert w["fwd_flops"] == fwd_flops
    assert w["bwd_flops"] == bwd_flops


@pytest.mark.parametrize("decay", [True, False, "vector"])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_byte_formulas_are_the_sizes_of_the_tensors_a_call_touches(decay, dtype):
    cfg = synth.FWD_410M.replace(B=2, H=3, T=64, dk=16, dv=24, C=32, decay=decay, dtype=dtype)
    inp = synth.ttt_inputs(cfg)
    nb = lambda *names: sum(inp[n].numel() * inp[n].element_size() for n in names
                            if inp[n] is not None)
    sizes = {"O": nb("V"), "W_final": nb("W0"), "dQ": nb("Q"), "dK": nb("K"), "dV": nb("V"),
             "dbeta": nb("beta"), "dW0": nb("W0")}
    fwd = nb("Q", "K", "V", "beta", "gamma", "W0") + sizes["O"] + sizes["W_final"]
    bwd = nb("Q", "K", "V", "dO", "beta", "gamma", "W0") + sum(
        sizes[n] for n in ("dQ", "dK", "dV", "dbeta", "dW0"))
    w = bench.layer_work(cfg)
    assert w["fwd_bytes"] == fwd
    assert w["bwd_bytes"] == bwd


def test_figures_of_the_timed_workloads():
    # the per-call figures quoted beside the measured times (1.45B-shaped training step,
    # 410M-shaped forward, In-Place forward at T=32768, d_ff=9728, d_model=2560)
    w = bench.layer_work(synth.TRAIN_1P45B)
    assert round(w["fwd_flops"] / 1e9, 1) == 43.0 and round(w["bwd_flops"] / 1e9, 1) == 86.0
    assert round(w["fwd_bytes"] / 1e6, 1) == 278.9 and round(w["bwd_bytes"] / 1e6, 1) == 481.3
    w = bench.layer_work(synth.FWD_410M)
    assert round(w["fwd_flops"] / 1e9, 2) == 15.07 and round(w["fwd_bytes"] / 1e6, 1) == 140.5
    fl, by = bench.inplace_work(synth.INPLACE_QWEN4B)
    # two GEMMs per chunk, (C x d_ff) x (d_ff x d_model) and (d_model x C) x (C x d_ff), over
    # every chunk: 2 (T d_ff d_model) multiply-adds each
    icfg = synth.INPLACE_QWEN4B
    assert fl == 2 * 2 * icfg.T * icfg.d_ff * icfg.d_model
    # Z and Vhat read (bf16), W read and written (fp32), O written (bf16)
    assert by == 2 * icfg.T * (icfg.d_ff + icfg.d_model) + 8 * icfg.d_model * icfg.d_ff + \
        2 * icfg.T * icfg.d_model
    assert round(fl / 1e12, 3) == 3.264 and round(by / 1e9, 3) == 1.172


def test_replica_throughput_and_peak_sources(tmp_path, monkeypatch):
    # one replica: ms per step and tokens per second from the device time of `steps` steps
    ms, value = bench.replica_throughput(200.0, steps=4, tokens_per_rank=1000, world=1)
    assert ms == 50.0 and value == pytest.approx(1000 / 0.05)
    # the measured peaks when the file is there, else the fallback, named as such
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    peaks, src = bench.load_peaks()
    assert src == "fallback" and peaks == bench.FALLBACK_PEAKS
    (tmp_path / "MEASURED_PEAKS.json").write_text(
        '{"hbm_gbs": 6000, "bf16_tflops": 1600, "bf16_tflops_sustained": 1300}')
    peaks, src = bench.load_peaks()
    assert src == "measured" and peaks == {"hbm_gbs": 6000.0, "bf16_tflops": 1600.0,
                                           "bf16_tflops_sustained": 1300.0}


def test_traffic_counters_are_dropped_once_a_source_changes(tmp_path, monkeypatch):
    import hashlib
    import json
    (tmp_path / "profiles").mkdir()
    src = tmp_path / "k.cu"
    src.write_bytes(b"kernel v1")
    sha = hashlib.sha256(b"k.cu" + b"kernel v1").hexdigest()[:16]
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(
        {"call": {"workload": "w", "bytes": 123, "sources": ["k.cu"], "sha": sha}}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.measured_traffic("call", "w") == 123
    assert bench.measured_traffic("call", "other workload") is None
    assert bench.measured_traffic("missing", "w") is None
    src.write_bytes(b"kernel v2")
    assert bench.measured_traffic("call", "w") is None


def test_reference_arm_line():
    # `bench.py --impl reference` times the oracle on the host cores; it needs no GPU
    import json
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    cmd = [sys.executable, os.path.join(root, "bench.py"), "--impl", "reference", "--steps", "1",
           "--warmup", "0"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=root)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC
    assert line["unit"] == "tokens/s" and line["higher_is_better"] is True
    assert line["steps"] == 1 and line["warmup"] >= 3  # at least three warm-up steps, always
    assert line["config"]["workload"] == synth.TRAIN_1P45B.name
    assert line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"] == {"value": line["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
    # under torchrun only rank 0 runs it; the other ranks exit at once without output
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=120, cwd=root,
                       env=dict(os.environ, RANK="1", WORLD_SIZE="2"))
    assert r.returncode == 0 and r.stdout.strip() == ""
