"""Parity of the mini-batch linear head (ttt_forward_linear_minibatch through the C ABI) against the
fp64 oracle, in both modes:
  prefix ("Vision-TTT" paper notes, section 关键设计 4): causal prefix sums inside consecutive
    mini-batches of b tokens, z_t = W_t q_t;
  epoch (press article, Observation 2 and Fig. 3): one mean-gradient step per consecutive
    mini-batch, every query read out with the final weights.

Tolerance, as for the full-batch heads: max|dZ| / max|Z_ref| and max|dW - dW_ref| / max|dW_ref|
(dW = W1 - W0, the weights after the last mini-batch) at most 1e-2 for bf16 inputs (the kernel
computes in fp32 from the bf16 inputs; Z is rounded to bf16) and 1e-5 for fp32 inputs.  The
recurrence contracts for unit-norm keys at these eta, so fp32 rounding does not grow along the
chain of mini-batches.
"""
import numpy as np
import pytest
import torch

import oracle
from tests.parity import TOL, rel_max_err, rel_update_err
from vision_test_token_b200 import WORKLOADS, forward_linear_minibatch, make_inputs
from vision_test_token_b200.inputs import random_unit

pytestmark = pytest.mark.gpu


def _run(x, eta, H, W, b, mode, dev, max_sms=0):
    Q, K, V = (x[k].to(dev) for k in ("Q", "K", "V"))
    B, h = Q.shape[:2]
    Z = torch.full_like(Q, float("nan"))
    W1 = torch.full((B, h, 64, 64), float("nan"), device=dev)
    forward_linear_minibatch(Q, K, V, x["W0_lin"].to(dev), eta, H, W, b, mode, Z=Z, W1_out=W1, max_sms=max_sms)
    torch.cuda.synchronize()
    return Z, W1


def _check(x, eta, H, W, b, mode, dev, dtype, max_sms=0):
    Z, W1 = _run(x, eta, H, W, b, mode, dev, max_sms)
    Zr, W1r = oracle.linear_minibatch(x["Q"], x["K"], x["V"], x["W0_lin"], eta, b, mode)
    ez = rel_max_err(Z, Zr)
    ew = rel_update_err(W1, W1r, x["W0_lin"].double().numpy()[None])
    assert ez <= TOL[dtype], f"Z rel err {ez:.3g}"
    assert ew <= TOL[dtype], f"dW rel err {ew:.3g}"
    return Z, W1


@pytest.mark.parametrize("B,h,H,W,b", [
    (1, 1, 1, 1, 1),        # one token
    (2, 1, 5, 7, 1),        # per-token sequential TTT
    (1, 2, 6, 6, 16),       # whole sub-blocks
    (3, 1, 7, 9, 16),       # a ragged last mini-batch
    (2, 2, 10, 13, 5),      # mini-batches shorter than a sub-block
    (1, 1, 9, 11, 40),      # mini-batches of several sub-blocks, ragged
    (2, 1, 14, 14, 196),    # one mini-batch (b = N)
    (1, 3, 8, 8, 1000),     # b > N
    (40, 1, 4, 4, 16),      # many units: CTAs loop over several units
])
@pytest.mark.parametrize("mode", ["prefix", "epoch"])
@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_minibatch_shapes(cuda_dev, B, h, H, W, b, mode, dtype):
    _, x = random_unit(B, h, H, W, dtype=dtype, seed=B * 100 + H * 10 + b)
    _check(x, 0.25, H, W, b, mode, cuda_dev, dtype)


@pytest.mark.parametrize("max_sms", [1, 7])
def test_minibatch_sm_budget(cuda_dev, max_sms):
    _, x = random_unit(4, 3, 12, 12, dtype="bf16", seed=max_sms)
    _check(x, 0.25, 12, 12, 16, "prefix", cuda_dev, "bf16", max_sms=max_sms)


def test_minibatch_epoch_single_batch_is_the_full_batch_layer(cuda_dev):
    """Epoch mode with b >= N is the full-batch step: it must match the full-batch oracle."""
    _, x = random_unit(2, 2, 10, 10, dtype="fp32", seed=5)
    Z, W1 = _run(x, 0.5, 10, 10, 100, "epoch", cuda_dev)
    Zr, W1r = oracle.linear(x["Q"], x["K"], x["V"], x["W0_lin"], 0.5)
    assert rel_max_err(Z, Zr) <= TOL["fp32"]
    assert rel_update_err(W1, W1r, x["W0_lin"].double().numpy()[None]) <= TOL["fp32"]


def test_minibatch_eta_zero_is_plain_readout(cuda_dev):
    _, x = random_unit(2, 1, 9, 9, dtype="fp32", seed=8)
    for mode in ("prefix", "epoch"):
        Z, W1 = _run(x, 0.0, 9, 9, 16, mode, cuda_dev)
        ref = np.einsum("hij,bhnj->bhni", x["W0_lin"].double().numpy(), x["Q"].double().numpy())
        assert rel_max_err(Z, ref) <= 1e-6
        assert torch.equal(W1.cpu(), x["W0_lin"][None].expand_as(W1.cpu()))


def test_minibatch_bitwise_repeatable(cuda_dev):
    _, x = random_unit(3, 2, 20, 20, dtype="bf16", seed=9)
    Za, Wa = _run(x, 0.25, 20, 20, 16, "prefix", cuda_dev)
    Zb, Wb = _run(x, 0.25, 20, 20, 16, "prefix", cuda_dev)
    assert torch.equal(Za, Zb) and torch.equal(Wa, Wb)


def test_minibatch_workload_full(cuda_dev):
    """The bench workload at full size (8 images x 6 heads x 78 x 78 tokens, b = 16, prefix), every
    unit against the oracle."""
    w = WORKLOADS["mb16_6084_bf16"]
    x = make_inputs(w)
    _check(x, w.eta, w.H, w.W, w.mb_tokens, w.mb_mode, cuda_dev, "bf16")
