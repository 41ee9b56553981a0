"""Parity of the linear head (ttt_forward_linear through the C ABI) against the fp64 oracle.

Tolerance (max|dZ| / max|Z_ref| over the whole output): 1e-5 for fp32 inputs, 1e-2 for bf16
inputs with fp32 accumulation.  The updated weights (W1_out) are checked on the update itself,
dW = W1 - W0, with the same tolerances, so that a dropped or mis-scaled update cannot hide inside
the output tolerance.
"""
import numpy as np
import pytest
import torch

import oracle
from tests.parity import TOL, rel_max_err, rel_update_err
from vision_test_token_b200 import WORKLOADS, forward_layer, forward_linear, make_inputs
from vision_test_token_b200.inputs import random_unit

pytestmark = pytest.mark.gpu


def _run(x, eta, H, W, dev, with_w1=True, max_sms=0):
    Q, K, V = (x[k].to(dev) for k in ("Q", "K", "V"))
    W0 = x["W0_lin"].to(dev)
    B, h = Q.shape[:2]
    W1 = torch.full((B, h, 64, 64), float("nan"), device=dev) if with_w1 else None
    Z = forward_linear(Q, K, V, W0, eta, H, W, W1_out=W1, max_sms=max_sms)
    torch.cuda.synchronize()
    return Z, W1


def _check(x, eta, H, W, dev, dtype, max_sms=0):
    Z, W1 = _run(x, eta, H, W, dev, max_sms=max_sms)
    Zr, W1r = oracle.linear(x["Q"], x["K"], x["V"], x["W0_lin"], eta)
    W0 = x["W0_lin"].double().numpy()[None]
    ez, ew = rel_max_err(Z, Zr), rel_update_err(W1, W1r, W0)
    assert ez <= TOL[dtype], f"Z rel err {ez:.3g}"
    assert ew <= TOL[dtype], f"dW rel err {ew:.3g}"
    return ez, ew


def test_lin196_fp32_workload(cuda_dev):
    w = WORKLOADS["lin196_fp32"]
    _check(make_inputs(w), w.eta, w.H, w.W, cuda_dev, "fp32")


def test_lin196_bf16_workload(cuda_dev):
    w = WORKLOADS["lin196_bf16"]
    _check(make_inputs(w), w.eta, w.H, w.W, cuda_dev, "bf16")


def test_lin6400_bf16_workload_full(cuda_dev):
    w = WORKLOADS["lin6400_bf16"]
    _check(make_inputs(w), w.eta, w.H, w.W, cuda_dev, "bf16")


@pytest.mark.parametrize("max_sms", [1, 7, 50, 123])
@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_sm_budget(cuda_dev, max_sms, dtype):
    """A bounded SM budget (fewer clusters or CTAs than units, smaller clusters) stays in tolerance."""
    _, x = random_unit(8, 5, 30, 40, dtype=dtype, seed=max_sms)
    _check(x, 0.5, 30, 40, cuda_dev, dtype, max_sms=max_sms)


@pytest.mark.parametrize("B,h,H,W", [
    (1, 1, 1, 1),        # a single token
    (1, 1, 1, 127),      # one ragged tile
    (2, 1, 8, 16),       # exactly one tile
    (1, 2, 3, 43),       # one full tile + 1 token
    (3, 5, 10, 20),      # H != W, 2 tiles per unit
    (37, 1, 15, 20),     # 3 tiles per unit, units spread over several CTAs
    (200, 1, 10, 13),    # many small units: CTAs span several units
    (2, 3, 77, 79),      # ragged large units
    (1, 2, 16, 24),      # 384 tokens: the largest unit of the fp32 cluster kernel
    (1, 1, 5, 77),       # 385 tokens: the fp32 tile kernels again
])
@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_odd_shapes(cuda_dev, B, h, H, W, dtype):
    _, x = random_unit(B, h, H, W, dtype=dtype, seed=B * 1000 + H * 10 + W)
    _check(x, 0.8, H, W, cuda_dev, dtype)


def test_adversarial_update_dominates(cuda_dev):
    """Large eta, un-normalised keys, small W0: the update is most of W1."""
    _, x = random_unit(2, 2, 20, 30, dtype="bf16", seed=5)
    g = torch.Generator().manual_seed(11)
    x["K"] = (torch.randn(x["K"].shape, generator=g) * 0.7).to(torch.bfloat16)
    x["W0_lin"] = x["W0_lin"] * 0.01
    _check(x, 3.0, 20, 30, cuda_dev, "bf16")


def test_eta_zero_is_plain_readout(cuda_dev):
    _, x = random_unit(2, 3, 9, 9, dtype="fp32", seed=3)
    Z, W1 = _run(x, 0.0, 9, 9, cuda_dev)
    ref = np.einsum("bhnj,hij->bhni", x["Q"].double().numpy(), x["W0_lin"].double().numpy())
    assert rel_max_err(Z, ref) <= 1e-5
    assert torch.equal(W1.cpu(), x["W0_lin"][None].expand_as(W1.cpu()))


def test_bitwise_deterministic(cuda_dev):
    w = WORKLOADS["lin196_bf16"]
    x = make_inputs(w)
    Z1, W1a = _run(x, w.eta, w.H, w.W, cuda_dev)
    Z2, W1b = _run(x, w.eta, w.H, w.W, cuda_dev)
    assert torch.equal(Z1, Z2) and torch.equal(W1a, W1b)


def test_mixed_layer_linear_heads(cuda_dev):
    """The 6084-token layer's five linear heads, run as head slices of the shared buffers."""
    w = WORKLOADS["mixed6084_bf16"]
    x = make_inputs(w)
    dev = cuda_dev
    Q, K, V = (x[k].to(dev) for k in ("Q", "K", "V"))
    Z = torch.full_like(Q, float("nan"))
    nl = w.lin_heads
    W1 = torch.empty((w.batch, nl, 64, 64), device=dev)
    forward_linear(Q[:, :nl], K[:, :nl], V[:, :nl], x["W0_lin"].to(dev), w.eta, w.H, w.W, Z=Z[:, :nl], W1_out=W1)
    torch.cuda.synchronize()
    Zr, W1r = oracle.linear(x["Q"][:, :nl], x["K"][:, :nl], x["V"][:, :nl], x["W0_lin"], w.eta)
    assert rel_max_err(Z[:, :nl], Zr) <= TOL["bf16"]
    assert rel_update_err(W1, W1r, x["W0_lin"].double().numpy()[None]) <= TOL["bf16"]
    assert torch.isnan(Z[:, nl:].float()).all(), "the call wrote outside its heads"


def test_workspace_reports_no_timeout(cuda_dev):
    from vision_test_token_b200 import capi, workspace, workspace_status
    _, x = random_unit(2, 2, 16, 16, dtype="bf16", seed=1)
    _run(x, 1.0, 16, 16, cuda_dev)
    shape = capi.make_shape(2, 2, 16, 16, 64, 2 * 256 * 64, 256 * 64, capi.TTT_BF16)
    ws = workspace(capi.TTT_HEAD_LINEAR, shape, cuda_dev)
    assert workspace_status(ws) == capi.TTT_OK
