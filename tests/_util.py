"""Shared helpers of the test suite (no method arithmetic)."""
import numpy as np
import torch


def to_np(x):
    return x.detach().to("cpu").double().numpy() if isinstance(x, torch.Tensor) else np.asarray(x, np.float64)


def rel_err(got, ref):
    """max|got - ref| / max|ref| over the whole tensor (the tolerance metric of the workloads)."""
    g, r = to_np(got), to_np(ref)
    assert g.shape == r.shape, (g.shape, r.shape)
    denom = np.abs(r).max()
    return float(np.abs(g - r).max() / (denom if denom > 0 else 1.0))


def gpu_available():
    return torch.cuda.is_available()
