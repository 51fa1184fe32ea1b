"""Seeded synthetic workloads for the chunkwise TTT layer and In-Place TTT.

This module only draws random tensors with the shapes and value
distributions of the workloads described for Modular TTT (page
"Modular TTT: Rethinking Test-Time Training as Composable Modules",
section "复现评估": chunk 256, fast-weight init std 0.02, small-lr init)
and In-Place TTT (page "In-Place Test-Time Training", section
"核心方法和技术细节"). It holds none of the method's arithmetic: both
the CUDA path and the CPU oracle receive the tensors produced here.

Layouts
    Q, K, V, O, dO : [B, H, T, d]   (d = d_k for Q/K, d_v for V/O/dO)
    beta           : [B, H, T]      float32
    gamma          : [B, H, T] (scalar decay) or [B, H, T, d_k] (vector decay) float32
    W0, dW_T       : [B, H, d_k, d_v] float32
    In-Place: Z [T, d_ff] bf16, Vhat [T, d_model] bf16, W [d_model, d_ff] f32, dO [T, d_model] bf16

Distribution notation: N(mu, s) takes s as the standard deviation.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, asdict

import torch

# b such that eta_0 = 2*sigmoid(b) = 0.1  ->  sigmoid(b) = 0.05
LR_BIAS_ETA0_0P1 = math.log(0.05 / 0.95)


@dataclass(frozen=True)
class TTTConfig:
    name: str
    B: int
    H: int
    T: int
    dk: int
    dv: int
    C: int
    dtype: str          # "f32" or "bf16": storage type of Q, K, V, O, dO, dQ, dK, dV
    loss: str           # "mse" or "ip"
    act: str            # "id" or "silu"
    decay: bool | str   # True: scalar decay gamma_t [B,H,T]; "vector": one decay per key feature
                        # [B,H,T,dk]; False: gamma == 1, passed as NULL
    w0_std: float       # std of the initial fast weight (0 -> zeros)
    normalize: str      # "qkv": L2-normalise rows of Q, K and V; "qk": of Q and K only
    lr_bias: float = LR_BIAS_ETA0_0P1
    backward: bool = False
    seed: int = 0

    @property
    def tokens(self) -> int:
        return self.B * self.T

    def replace(self, **kw) -> "TTTConfig":
        d = asdict(self)
        d.update(kw)
        return TTTConfig(**d)


@dataclass(frozen=True)
class InPlaceConfig:
    name: str
    T: int
    d_ff: int
    d_model: int
    C: int
    lr: float
    seed: int = 0

    def replace(self, **kw) -> "InPlaceConfig":
        d = asdict(self)
        d.update(kw)
        return InPlaceConfig(**d)


# The five workloads (seeds 1..5).
TINY_FP32 = TTTConfig("tiny-ttt-linear-fp32-fwd", B=1, H=2, T=512, dk=64, dv=64, C=64,
                      dtype="f32", loss="mse", act="id", decay=False, w0_std=1 / 64,
                      normalize="qkv", seed=1)
FWD_410M = TTTConfig("410m-ttt-linear-fwd", B=8, H=16, T=2048, dk=64, dv=64, C=256,
                     dtype="bf16", loss="mse", act="id", decay=True, w0_std=0.0,
                     normalize="qk", seed=2)
SILU_IP_FWD = TTTConfig("silu-ip-fwd", B=4, H=16, T=4096, dk=128, dv=128, C=256,
                        dtype="bf16", loss="ip", act="silu", decay=True, w0_std=1 / 128,
                        normalize="qk", seed=3)
TRAIN_1P45B = TTTConfig("1.45b-ttt-linear-fwd-bwd", B=4, H=16, T=4096, dk=128, dv=128, C=256,
                        dtype="bf16", loss="mse", act="id", decay=True, w0_std=1 / 128,
                        normalize="qk", backward=True, seed=4)
INPLACE_QWEN4B = InPlaceConfig("inplace-ttt-wdown-fwd", T=32768, d_ff=9728, d_model=2560,
                               C=1024, lr=1e-3, seed=5)

TTT_CONFIGS = {c.name: c for c in (TINY_FP32, FWD_410M, SILU_IP_FWD, TRAIN_1P45B)}


def storage_dtype(cfg: TTTConfig) -> torch.dtype:
    return torch.float32 if cfg.dtype == "f32" else torch.bfloat16


def _randn(shape, gen, device):
    return torch.randn(*shape, generator=gen, device=device, dtype=torch.float32)


def _l2_rows(x):
    return x / x.norm(dim=-1, keepdim=True)


def make_generator(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def ttt_inputs(cfg: TTTConfig, device="cpu", seed: int | None = None) -> dict:
    """Draw one seeded batch for a TTT layer workload.

    Returns a dict of tensors on `device`: Q, K, V (storage dtype), beta,
    gamma (float32, gamma is None when cfg.decay is False), W0 (float32) and,
    for every config, an upstream gradient dO (storage dtype) and dW_T
    (float32 zeros) so that the backward can be exercised on any workload.
    """
    seed = cfg.seed if seed is None else seed
    g = make_generator(seed, device)
    B, H, T, dk, dv = cfg.B, cfg.H, cfg.T, cfg.dk, cfg.dv
    sd = storage_dtype(cfg)
    q = _randn((B, H, T, dk), g, device)
    k = _randn((B, H, T, dk), g, device)
    v = _randn((B, H, T, dv), g, device)
    if cfg.normalize in ("qk", "qkv"):
        q = _l2_rows(q)
        k = _l2_rows(k)
    if cfg.normalize == "qkv":
        v = _l2_rows(v)
    beta = _randn((B, H, T), g, device)
    if cfg.decay == "vector":
        gamma = torch.sigmoid(3.0 + 0.5 * _randn((B, H, T, dk), g, device))
    elif cfg.decay:
        gamma = torch.sigmoid(3.0 + 0.5 * _randn((B, H, T), g, device))
    else:
        gamma = None
    if cfg.w0_std > 0:
        w0 = cfg.w0_std * _randn((B, H, dk, dv), g, device)
    else:
        w0 = torch.zeros((B, H, dk, dv), device=device, dtype=torch.float32)
    do = _randn((B, H, T, dv), g, device)
    return dict(
        Q=q.to(sd).contiguous(), K=k.to(sd).contiguous(), V=v.to(sd).contiguous(),
        beta=beta.contiguous(), gamma=None if gamma is None else gamma.contiguous(),
        W0=w0.contiguous(), dO=do.to(sd).contiguous(),
        dW_T=torch.zeros((B, H, dk, dv), device=device, dtype=torch.float32),
    )


def inplace_inputs(cfg: InPlaceConfig, device="cpu", seed: int | None = None) -> dict:
    """Draw one seeded In-Place TTT workload: Z = SiLU(N(0,1)) * N(0,1) [T, d_ff] bf16,
    Vhat ~ N(0, 0.02) [T, d_model] bf16, W_down ~ N(0, 0.02) [d_model, d_ff] float32 and, for
    the backward, an upstream gradient dO ~ N(0, 1) [T, d_model] bf16 (drawn last, so the
    forward's tensors do not depend on it)."""
    seed = cfg.seed if seed is None else seed
    g = make_generator(seed, device)
    a = _randn((cfg.T, cfg.d_ff), g, device)
    z = torch.nn.functional.silu(a)
    z.mul_(_randn((cfg.T, cfg.d_ff), g, device))
    z = z.to(torch.bfloat16)
    vhat = (0.02 * _randn((cfg.T, cfg.d_model), g, device)).to(torch.bfloat16)
    w = 0.02 * _randn((cfg.d_model, cfg.d_ff), g, device)
    do = _randn((cfg.T, cfg.d_model), g, device).to(torch.bfloat16)
    return dict(Z=z.contiguous(), Vhat=vhat.contiguous(), W=w.contiguous(), dO=do.contiguous())


def inplace_target_inputs(cfg: InPlaceConfig, k: int = 4, device="cpu", seed: int | None = None) -> dict:
    """Draw the inputs of the NTP-aligned target Vhat = Conv1D(X0) W_target (page "In-Place
    Test-Time Training", section "核心方法和技术细节"): token embeddings X0 ~ N(0, 0.02)
    [T, d_model] bf16, depthwise taps conv_w ~ N(0, 1/k) [k, d_model] float32 over the current
    and the next k - 1 tokens, W_target ~ N(0, 1/sqrt(d_model)) [d_model, d_model] bf16 (input
    rows, output columns), and an upstream gradient dVhat ~ N(0, 1) [T, d_model] bf16. The
    page gives no window size; k = 4 is this workload's choice. Seeded apart from
    inplace_inputs (seed + 1000)."""
    seed = (cfg.seed if seed is None else seed) + 1000
    g = make_generator(seed, device)
    d = cfg.d_model
    x0 = (0.02 * _randn((cfg.T, d), g, device)).to(torch.bfloat16)
    w = _randn((k, d), g, device) / math.sqrt(k)
    wt = (_randn((d, d), g, device) / math.sqrt(d)).to(torch.bfloat16)
    dv = _randn((cfg.T, d), g, device).to(torch.bfloat16)
    return dict(X0=x0.contiguous(), conv_w=w.contiguous(), W_target=wt.contiguous(),
                dVhat=dv.contiguous())


# TTT-MLP workload: the 410M layer shape with a two-layer fast weight of hidden width 4 d,
# SiLU between the layers, both layers initialised with std 0.02 (section "复现评估").
TTT_MLP_410M = TTTConfig("410m-ttt-mlp-fwd-bwd", B=8, H=16, T=2048, dk=64, dv=64, C=256,
                         dtype="bf16", loss="mse", act="silu", decay=True, w0_std=0.02,
                         normalize="qk", backward=True, seed=6)
TTT_MLP_HIDDEN = 256


def ttt_mlp_weights(cfg: TTTConfig, hidden: int, device="cpu", seed: int | None = None) -> dict:
    """Initial weights of the two-layer fast weight: W1 [B,H,dk,hidden] and W2 [B,H,hidden,dv]
    ~ N(0, cfg.w0_std) float32, and upstream gradients of the final weights dW1_T, dW2_T
    (zeros). Seeded apart from ttt_inputs (seed + 2000)."""
    seed = (cfg.seed if seed is None else seed) + 2000
    g = make_generator(seed, device)
    B, H = cfg.B, cfg.H
    w1 = cfg.w0_std * _randn((B, H, cfg.dk, hidden), g, device)
    w2 = cfg.w0_std * _randn((B, H, hidden, cfg.dv), g, device)
    z1 = torch.zeros_like(w1)
    z2 = torch.zeros_like(w2)
    return dict(W1=w1.contiguous(), W2=w2.contiguous(), dW1_T=z1, dW2_T=z2)
