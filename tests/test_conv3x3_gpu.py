"""Parity of the full 3x3 conv head (ttt_forward_conv3x3 through the C ABI) against the fp64 oracle:
max|dZ| / max|Z_ref| <= 1e-2 (bf16 with fp32 accumulation) and the same bound on the update W1 - W0
of the d x d x 3 x 3 kernel.  Shapes span several 8 x 16 position tiles with ragged edges in both
directions, single-row, single-column and single-token grids, units that share a CTA, and SM
budgets from one CTA to the whole device."""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from tests.parity import TOL, rel_max_err, rel_update_err
from vision_test_token_b200 import WORKLOADS, capi, forward_conv3x3, make_inputs
from vision_test_token_b200.inputs import Workload

pytestmark = pytest.mark.gpu


def _inputs(B, h, H, W, seed):
    return make_inputs(Workload("c3", B, h, H, W, "bf16", 0.5, "conv3x3"), seed)


def _run(x, eta, H, W, dev, max_sms=0):
    Q, K, V = (x[k].to(dev) for k in ("Q", "K", "V"))
    B, h = Q.shape[:2]
    W1 = torch.full((B, h, 64, 64, 3, 3), float("nan"), device=dev)
    Z = forward_conv3x3(Q, K, V, x["W0_c3"].to(dev), eta, H, W, W1_out=W1, max_sms=max_sms)
    torch.cuda.synchronize()
    return Z, W1


def _check(x, eta, H, W, dev, max_sms=0):
    Z, W1 = _run(x, eta, H, W, dev, max_sms)
    Zr, W1r = oracle.conv3x3(x["Q"], x["K"], x["V"], x["W0_c3"], eta, H, W)
    W0 = x["W0_c3"].double().numpy()[None]
    ez, ew = rel_max_err(Z, Zr), rel_update_err(W1, W1r, W0)
    assert ez <= TOL["bf16"], f"Z rel err {ez:.3g}"
    assert ew <= TOL["bf16"], f"dW rel err {ew:.3g}"
    return Z, W1


@pytest.mark.parametrize("B,h,H,W", [
    (1, 1, 1, 1), (1, 1, 1, 21), (1, 1, 19, 1), (2, 1, 9, 20), (1, 2, 16, 16), (3, 1, 17, 33), (2, 3, 8, 16),
    (1, 1, 5, 37),
])
def test_conv3x3_shapes(cuda_dev, B, h, H, W):
    _check(_inputs(B, h, H, W, seed=H * 100 + W + B), 0.5, H, W, cuda_dev)


@pytest.mark.parametrize("max_sms", [1, 3, 7, 0])
def test_conv3x3_sm_budgets(cuda_dev, max_sms):
    """One CTA over every tile of every unit, a few CTAs whose tile ranges cross units, and the whole
    device give the same result within tolerance."""
    _check(_inputs(3, 2, 13, 25, seed=5), 0.5, 13, 25, cuda_dev, max_sms)


def test_conv3x3_full_size_workload(cuda_dev):
    """conv3x3_6084_bf16 at its full size (8 images x 78 x 78 tokens), every unit against the oracle."""
    w = WORKLOADS["conv3x3_6084_bf16"]
    _check(make_inputs(w, seed=0), w.eta, w.H, w.W, cuda_dev)


def test_conv3x3_eta_zero_is_torch_conv2d(cuda_dev):
    x = _inputs(2, 1, 11, 18, seed=3)
    Z, W1 = _run(x, 0.0, 11, 18, cuda_dev)
    q = x["Q"].double()[:, 0].transpose(1, 2).reshape(2, 64, 11, 18)
    ref = F.conv2d(q, x["W0_c3"][0].double(), padding=1).reshape(2, 64, 198).transpose(1, 2)[:, None]
    assert rel_max_err(Z, ref.numpy()) <= TOL["bf16"]
    assert torch.equal(W1.cpu(), x["W0_c3"][None].expand_as(W1.cpu()))


def test_conv3x3_large_update(cuda_dev):
    """A large step (eta = 8) makes the update dominate the readout."""
    _check(_inputs(2, 1, 14, 14, seed=8), 8.0, 14, 14, cuda_dev)


def test_conv3x3_bitwise_deterministic(cuda_dev):
    x = _inputs(2, 2, 20, 20, seed=9)
    Z1, W1 = _run(x, 0.5, 20, 20, cuda_dev)
    Z2, W2 = _run(x, 0.5, 20, 20, cuda_dev)
    assert torch.equal(Z1, Z2) and torch.equal(W1, W2)


def test_conv3x3_rejects_fp32_and_dot_loss(cuda_dev):
    dev = cuda_dev
    t = torch.zeros((1, 1, 16, 64), device=dev)
    w = torch.zeros((1, 64, 64, 3, 3), device=dev)
    s = capi.make_shape(1, 1, 4, 4, 64, 16 * 64, 16 * 64, capi.TTT_FP32)
    assert capi.ttt_workspace_bytes(capi.TTT_HEAD_CONV3X3, s) == 0
    st = capi.ttt_forward_conv3x3(t.data_ptr(), t.data_ptr(), t.data_ptr(), w.data_ptr(), t.data_ptr() + 4096,
                                  0.5, s, None, 0, None, 0)
    assert st in (capi.TTT_ERR_UNSUPPORTED, capi.TTT_ERR_INVALID_ARG)
    s = capi.make_shape(1, 1, 4, 4, 64, 16 * 64, 16 * 64, capi.TTT_BF16, 0, 0, capi.TTT_LOSS_DOT)
    assert capi.ttt_workspace_bytes(capi.TTT_HEAD_CONV3X3, s) == 0
