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
                           cfg.lr_bias)


def gpu_inputs(cfg, seed=None):
    return synth.ttt_inputs(cfg, device="cuda", seed=seed)


def run_fwd(cfg, inp):
    c = abi_config(cfg)
    sd = synth.storage_dtype(cfg)
    B, H, T, dk, dv, C = cfg.B, cfg.H, cfg.T, cfg.dk, cfg.dv, cfg.C
    O = torch.empty((B, H, T, dv), device="cuda", dtype=sd)
    Wf = torch.empty((B, H, dk, dv), device="cuda", dtype=torch.float32)
    Wc = torch.empty((B, H, T // C, dk, dv), device="cuda", dtype=sd)
    n = ttt.ttt_workspace_bytes(c, False)
    ws = torch.empty(max(n, 16), device="cuda", dtype=torch.uint8)
    ttt.ttt_chunk_fwd(c, inp["Q"], inp["K"], inp["V"], inp["beta"], inp["gamma"], inp["W0"], O, Wf,
                      Wc, ws, n)
    torch.cuda.synchronize()
    assert ttt.ttt_get_device_error() == ttt.OK
    return dict(O=O, W_final=Wf, W_chunks=Wc)


def run_bwd(cfg, inp, W_chunks):
    c = abi_config(cfg)
    sd = synth.storage_dtype(cfg)
    B, H, T, dk, dv = cfg.B, cfg.H, cfg.T, cfg.dk, cfg.dv
    out = dict(dQ=torch.empty((B, H, T, dk), device="cuda", dtype=sd),
               dK=torch.empty((B, H, T, dk), device="cuda", dtype=sd),
               dV=torch.empty((B, H, T, dv), device="cuda", dtype=sd),
               dbeta=torch.empty((B, H, T), device="cuda", dtype=torch.float32),
               dW0=torch.empty((B, H, dk, dv), device="cuda", dtype=torch.float32))
    n = ttt.ttt_workspace_bytes(c, True)
    ws = torch.empty(max(n, 16), device="cuda", dtype=torch.uint8)
    ttt.ttt_chunk_bwd(c, inp["Q"], inp["K"], inp["V"], inp["beta"], inp["gamma"], inp["W0"],
                      W_chunks, inp["dO"], inp["dW_T"], out["dQ"], out["dK"], out["dV"],
                      out["dbeta"], out["dW0"], ws, n)
    torch.cuda.synchronize()
    assert ttt.ttt_get_device_error() == ttt.OK
    return out


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
