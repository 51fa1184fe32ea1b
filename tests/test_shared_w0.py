"""GPU checks of a W0 shared across the batch (ttt_config.w0_shared): a call that passes one
initial state per head, [H, dk, dv], gives bit for bit what the same call gives with that state
repeated for every sequence, [B, H, dk, dv], on every kernel family (the only difference is the
address each (batch, head) reads its initial state from)."""
import pytest
import torch

import synth
import weight_sequence_layers_b200 as ttt

pytestmark = pytest.mark.gpu


def _config(cfg, shared):
    return ttt.make_config(cfg.B, cfg.H, cfg.T, cfg.dk, cfg.dv, cfg.C, cfg.dtype, cfg.loss,
                           cfg.act, cfg.lr_bias, "vector" if cfg.decay == "vector" else "scalar",
                           w0_shared=shared)


def _layer(cfg, inp, W0, shared):
    c = _config(cfg, shared)
    sd = synth.storage_dtype(cfg)
    B, H, T, dk, dv, C = cfg.B, cfg.H, cfg.T, cfg.dk, cfg.dv, cfg.C
    O = torch.empty((B, H, T, dv), device="cuda", dtype=sd)
    Wf = torch.empty((B, H, dk, dv), device="cuda")
    Wc = torch.empty((B, H, T // C, dk, dv), device="cuda", dtype=sd)
    nG = ttt.ttt_saved_bytes(c)
    G = torch.empty(-(-nG // 2), device="cuda", dtype=torch.bfloat16) if sd == torch.bfloat16 \
        else torch.empty(-(-nG // 4), device="cuda")
    n = max(ttt.ttt_workspace_bytes(c, 0), ttt.ttt_workspace_bytes(c, 2), 16)
    ws = torch.empty(n, device="cuda", dtype=torch.uint8)
    ttt.ttt_chunk_fwd(c, inp["Q"], inp["K"], inp["V"], inp["beta"], inp["gamma"], W0, O, Wf, Wc,
                      G, ws, n)
    g = {k: torch.empty_like(inp[k]) for k in ("Q", "K", "V", "beta")}
    dW0 = torch.empty((B, H, dk, dv), device="cuda")
    ttt.ttt_chunk_bwd(c, inp["Q"], inp["K"], inp["V"], inp["beta"], inp["gamma"], W0, Wc, G,
                      inp["dO"], inp["dW_T"], None, None, g["Q"], g["K"], g["V"], g["beta"], dW0,
                      None, ws, n)
    torch.cuda.synchronize()
    assert ttt.ttt_get_device_error() == ttt.OK
    return dict(O=O, W_final=Wf, W_chunks=Wc, dQ=g["Q"], dK=g["K"], dV=g["V"], dbeta=g["beta"],
                dW0=dW0)


CASES = [
    (synth.TRAIN_1P45B, dict(B=2, H=2, T=512)),                         # tensor cores, d = 128
    (synth.FWD_410M, dict(B=2, H=2, T=512, decay="vector")),            # vector decay
    (synth.TINY_FP32, dict(B=2, H=2, T=128)),                           # SIMT, float32
]


@pytest.mark.parametrize("base,kw", CASES, ids=["tc", "tc-vector", "simt-f32"])
def test_shared_initial_state_equals_repeated(base, kw):
    cfg = base.replace(**kw)
    inp = synth.ttt_inputs(cfg, device="cuda", seed=211)
    inp["dW_T"].normal_(generator=torch.Generator("cuda").manual_seed(212))
    W0h = torch.randn((cfg.H, cfg.dk, cfg.dv), device="cuda") * 0.05
    W0b = W0h.unsqueeze(0).expand(cfg.B, -1, -1, -1).contiguous()
    a = _layer(cfg, inp, W0h, True)
    b = _layer(cfg, inp, W0b, False)
    for k in a:
        assert torch.equal(a[k], b[k]), k


def test_shared_initial_weights_of_ttt_mlp():
    cfg, hid = synth.TTT_MLP_410M.replace(B=2, H=2, T=512), synth.TTT_MLP_HIDDEN
    inp = synth.ttt_inputs(cfg, device="cuda", seed=213)
    w = synth.ttt_mlp_weights(cfg, hid, device="cuda", seed=214)
    W1h, W2h = w["W1"][0].contiguous(), w["W2"][0].contiguous()
    W1b = W1h.unsqueeze(0).expand(cfg.B, -1, -1, -1).contiguous()
    W2b = W2h.unsqueeze(0).expand(cfg.B, -1, -1, -1).contiguous()
    outs = []
    for shared, W1, W2 in ((True, W1h, W2h), (False, W1b, W2b)):
        c = _config(cfg, shared)
        O = torch.empty_like(inp["V"])
        W1f, W2f = torch.empty_like(w["W1"]), torch.empty_like(w["W2"])
        n = ttt.ttt_mlp_workspace_bytes(c, hid)
        ws = torch.empty(n, device="cuda", dtype=torch.uint8)
        ttt.ttt_mlp_fwd(c, hid, inp["Q"], inp["K"], inp["V"], inp["beta"], inp["gamma"], W1, W2,
                        O, W1f, W2f, None, None, ws, n)
        torch.cuda.synchronize()
        outs.append((O, W1f, W2f))
    for x, y in zip(*outs):
        assert torch.equal(x, y)
