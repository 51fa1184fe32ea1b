"""Failure detection without faulting the GPU: a bounded in-kernel wait on a barrier that
nothing completes must give up, report TTT_ERR_TIMEOUT through the error word, and leave
the context usable."""
import pytest
import torch

import synth
import weight_sequence_layers_b200 as ttt
from _runners import run_fwd

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives():
    assert ttt.ttt_get_device_error() == ttt.OK
    ttt.ttt_selftest_bounded_wait(2000)
    assert ttt.ttt_get_device_error() == ttt.ERR_TIMEOUT
    assert ttt.ttt_get_device_error() == ttt.OK  # the word was cleared
    cfg = synth.TINY_FP32.replace(B=1, H=1, T=128)
    out = run_fwd(cfg, synth.ttt_inputs(cfg, device="cuda"))
    assert torch.isfinite(out["O"]).all()
