"""Runs one workload through the C ABI (via the binding) and through the oracle."""
import numpy as np
import torch

import oracle
import synth
import weight_sequence_layers_b200 as ttt


def lr_bias32(cfg):
    # the ABI takes b as float32: hand the oracle the same value
    return float(np.float32(cfg.lr_bias))


def abi_config(cfg):
    return ttt.make_config(cfg.B, cfg.H, cfg.T, cfg.dk, cfg.dv, cfg.C, cfg.dtype, cfg.loss, cfg.act,
                           cfg.lr_bias, "vector" if cfg.decay == "vector" else "scalar")


def gpu_inputs(cfg, seed=None):
    return synth.ttt_inputs(cfg, device="cuda", seed=seed)


def run_fwd(cfg, inp, save_g=True, save_w=True):
    """The forward through the C ABI; save_w / save_g request the chunk-start states and G (with
    SiLU also Zq) that a backward reads. With both off it is the inference forward."""
    c = abi_config(cfg)
    sd = synth.storage_dtype(cfg)
    B, H, T, dk, dv, C = cfg.B, cfg.H, cfg.T, cfg.dk, cfg.dv, cfg.C
    O = torch.empty((B, H, T, dv), device="cuda", dtype=sd)
    Wf = torch.empty((B, H, dk, dv), device="cuda", dtype=torch.float32)
    Wc = torch.empty((B, H, T // C, dk, dv), device="cuda", dtype=sd) if save_w else None
    # the saved buffer holds G, then with SiLU Zq (the readout before the activation); with a
    # vector decay on the tensor cores more follows (whole [B, H, T, dv] planes, rounded up)
    planes = -(-ttt.ttt_saved_bytes(c) // (B * H * T * dv * sd.itemsize))
    Gs = torch.empty((planes, B, H, T, dv), device="cuda", dtype=sd) if save_g else None
    n = ttt.ttt_workspace_bytes(c, 0)
    ws = torch.empty(max(n, 16), device="cuda", dtype=torch.uint8)
    ttt.ttt_chunk_fwd(c, inp["Q"], inp["K"], inp["V"], inp["beta"], inp["gamma"], inp["W0"], O, Wf,
                      Wc, Gs, ws, n)
    torch.cuda.synchronize()
    assert ttt.ttt_get_device_error() == ttt.OK
    return dict(O=O, W_final=Wf, W_chunks=Wc, G=None if Gs is None else Gs[0], G_saved=Gs,
                Zq=Gs[1] if Gs is not None and cfg.act == "silu" else None)


def run_bwd(cfg, inp, W_chunks, G=None, fwd=None):
    """The backward; G (run_fwd's "G_saved") is passed as G_saved, else the library rebuilds it.
    With `fwd` (run_fwd's outputs) and a decay, the decay gradient is asked for too."""
    c = abi_config(cfg)
    sd = synth.storage_dtype(cfg)
    B, H, T, dk, dv = cfg.B, cfg.H, cfg.T, cfg.dk, cfg.dv
    out = dict(dQ=torch.empty((B, H, T, dk), device="cuda", dtype=sd),
               dK=torch.empty((B, H, T, dk), device="cuda", dtype=sd),
               dV=torch.empty((B, H, T, dv), device="cuda", dtype=sd),
               dbeta=torch.empty((B, H, T), device="cuda", dtype=torch.float32),
               dW0=torch.empty((B, H, dk, dv), device="cuda", dtype=torch.float32))
    want_dg = fwd is not None and inp["gamma"] is not None
    if want_dg:
        out["dgamma"] = torch.empty(inp["gamma"].shape, device="cuda", dtype=torch.float32)
    n = ttt.ttt_workspace_bytes(c, 2 if G is not None else 1)
    ws = torch.empty(max(n, 16), device="cuda", dtype=torch.uint8)
    ttt.ttt_chunk_bwd(c, inp["Q"], inp["K"], inp["V"], inp["beta"], inp["gamma"], inp["W0"],
                      W_chunks, G, inp["dO"], inp["dW_T"], fwd["O"] if want_dg else None,
                      fwd["W_final"] if want_dg else None, out["dQ"], out["dK"], out["dV"],
                      out["dbeta"], out["dW0"], out.get("dgamma"), ws, n)
    torch.cuda.synchronize()
    assert ttt.ttt_get_device_error() == ttt.OK
    return out


def reference_g(cfg, inp, W_chunks):
    """G of every token written out from its definition, g_t = a(z_t) act'(z_t) with z_t = k_t W0
    of the token's chunk (a = act(z) - v for MSE, -v for IP), in fp64 from the oracle's states."""
    K = inp["K"].double().cpu().numpy()
    V = inp["V"].double().cpu().numpy()
    Wc = np.asarray(W_chunks, dtype=np.float64)
    B, H, T, dk = K.shape
    C = cfg.C
    z = np.einsum("bhcsi,bhcij->bhcsj", K.reshape(B, H, T // C, C, dk), Wc).reshape(B, H, T, -1)
    if cfg.act == "silu":
        sg = 1.0 / (1.0 + np.exp(-z))
        act, d1 = z * sg, sg * (1.0 + z * (1.0 - sg))
    else:
        act, d1 = z, np.ones_like(z)
    a = act - V if cfg.loss == "mse" else -V
    return a * d1


def oracle_fwd(cfg, inp):
    O, Wf, Wc, _ = oracle.ttt_fwd(inp["Q"], inp["K"], inp["V"], inp["beta"], inp["gamma"], inp["W0"],
                                  C=cfg.C, loss=cfg.loss, act=cfg.act, lr_bias=lr_bias32(cfg))
    return dict(O=O, W_final=Wf, W_chunks=Wc)


def oracle_bwd(cfg, inp):
    return oracle.ttt_bwd(inp["Q"], inp["K"], inp["V"], inp["beta"], inp["gamma"], inp["W0"],
                          inp["dO"], inp["dW_T"], C=cfg.C, loss=cfg.loss, act=cfg.act,
                          lr_bias=lr_bias32(cfg))


def head_slice(inp, heads):
    """The per-head tensors of the listed (b, h) pairs, stacked as B = 1, H = len(heads).
    Heads evolve independently, so the oracle on this slice is exact for those heads."""
    out = {}
    for k, v in inp.items():
        out[k] = None if v is None else torch.stack([v[b, h] for b, h in heads]).unsqueeze(0)
    return out
