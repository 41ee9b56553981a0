"""Shared helpers of the parity tests (GPU result vs fp64 oracle)."""
import numpy as np
import torch


def rel_max_err(got, ref):
    """max |got - ref| / max |ref| over the whole tensor (the layer's tolerance metric)."""
    g = got.detach().double().cpu().numpy() if isinstance(got, torch.Tensor) else np.asarray(got, np.float64)
    r = np.asarray(ref, np.float64)
    assert g.shape == r.shape, (g.shape, r.shape)
    denom = np.max(np.abs(r))
    return float(np.max(np.abs(g - r)) / (denom if denom > 0 else 1.0))


def rel_update_err(W1_got, W1_ref, W0):
    """Error of the update itself: max |dW_got - dW_ref| / max |dW_ref|, dW = W1 - W0."""
    g = W1_got.detach().double().cpu().numpy() - np.asarray(W0, np.float64)
    r = np.asarray(W1_ref, np.float64) - np.asarray(W0, np.float64)
    return float(np.max(np.abs(g - r)) / max(np.max(np.abs(r)), 1e-300))


TOL = {"fp32": 1e-5, "bf16": 1e-2}
