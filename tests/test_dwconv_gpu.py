"""Parity of the depthwise-conv head (ttt_forward_dwconv through the C ABI) against the fp64
oracle: max|dZ| / max|Z_ref| <= 1e-2 (bf16) or 1e-5 (fp32), and the same bound on the update
W1 - W0 of the 3x3 kernels."""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from tests.parity import TOL, rel_max_err, rel_update_err
from vision_test_token_b200 import WORKLOADS, forward_dwconv, forward_layer, forward_linear, make_inputs
from vision_test_token_b200.inputs import random_unit

pytestmark = pytest.mark.gpu


def _run(x, eta, H, W, dev, max_sms=0):
    Q, K, V = (x[k].to(dev) for k in ("Q", "K", "V"))
    B, h = Q.shape[:2]
    W1 = torch.full((B, h, 64, 3, 3), float("nan"), device=dev)
    Z = forward_dwconv(Q, K, V, x["W0_conv"].to(dev), eta, H, W, W1_out=W1, max_sms=max_sms)
    torch.cuda.synchronize()
    return Z, W1


def _check(x, eta, H, W, dev, dtype, max_sms=0):
    Z, W1 = _run(x, eta, H, W, dev, max_sms)
    Zr, W1r = oracle.dwconv(x["Q"], x["K"], x["V"], x["W0_conv"], eta, H, W)
    W0 = x["W0_conv"].double().numpy()[None]
    ez, ew = rel_max_err(Z, Zr), rel_update_err(W1, W1r, W0)
    assert ez <= TOL[dtype], f"Z rel err {ez:.3g}"
    assert ew <= TOL[dtype], f"dW rel err {ew:.3g}"


def _conv_inputs(B, h, H, W, dtype, seed):
    return random_unit(B, h, H, W, dtype=dtype, seed=seed, kind="mixed", conv_heads=h)[1]


@pytest.mark.parametrize("B,h,H,W", [
    (1, 1, 1, 1), (1, 1, 1, 9), (1, 1, 9, 1), (2, 1, 5, 7), (3, 2, 14, 14), (2, 1, 33, 17), (8, 1, 78, 78),
    (1, 3, 80, 80), (40, 1, 6, 6), (5, 1, 2, 30), (1, 1, 7, 170), (2, 1, 4, 161), (300, 1, 3, 5),
])
@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_dwconv_shapes(cuda_dev, B, h, H, W, dtype):
    _check(_conv_inputs(B, h, H, W, dtype, seed=H * 100 + W), 0.5, H, W, cuda_dev, dtype)


def test_dwconv_identity_kernel_reproduces_q(cuda_dev):
    x = _conv_inputs(2, 1, 12, 10, "fp32", seed=4)
    x["V"] = x["K"].clone()
    W0 = torch.zeros(1, 64, 3, 3); W0[:, :, 1, 1] = 1.0
    x["W0_conv"] = W0
    Z, W1 = _run(x, 1.0, 12, 10, cuda_dev)
    assert torch.equal(Z.cpu(), x["Q"])
    assert torch.equal(W1.cpu(), W0[None].expand_as(W1.cpu()))


def test_dwconv_eta_zero_matches_torch_conv2d(cuda_dev):
    x = _conv_inputs(2, 1, 11, 13, "fp32", seed=6)
    Z, _ = _run(x, 0.0, 11, 13, cuda_dev)
    q = x["Q"].double()[:, 0].transpose(1, 2).reshape(2, 64, 11, 13)
    ref = F.conv2d(q, x["W0_conv"][0].double().reshape(64, 1, 3, 3), padding=1, groups=64)
    ref = ref.reshape(2, 64, 143).transpose(1, 2)[:, None]
    assert rel_max_err(Z, ref.numpy()) <= 1e-5


@pytest.mark.parametrize("max_sms", [1, 2, 3, 24, 25, 0])
@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_dwconv_sm_budget(cuda_dev, max_sms, dtype):
    """Any SM budget gives the same result within tolerance: one CTA looping over every (unit, band)
    task, a few CTAs each taking several tasks (their gradients first, then their readouts), bands
    of one row pair, and the whole device."""
    _check(_conv_inputs(8, 1, 78, 78, dtype, seed=17), 0.5, 78, 78, cuda_dev, dtype, max_sms)


@pytest.mark.parametrize("concurrent", [True, False])
def test_mixed6084_layer_full(cuda_dev, concurrent):
    """The full 6084-token layer: 5 linear heads + the depthwise-conv head (last), in the launch
    configuration the benchmark times (the conv call on a second stream, at the same time as the
    linear call, each on its share of the SMs) and one call after the other."""
    w = WORKLOADS["mixed6084_bf16"]
    x = make_inputs(w)
    dev = cuda_dev
    Q, K, V = (x[k].to(dev) for k in ("Q", "K", "V"))
    Z = torch.full_like(Q, float("nan"))
    forward_layer(Q, K, V, {k: v.to(dev) for k, v in x.items() if k.startswith("W0")}, w.eta, w.H, w.W,
                  conv_heads=w.conv_heads, Z=Z, concurrent=concurrent)
    torch.cuda.synchronize()
    nl = w.lin_heads
    Zl, _ = oracle.linear(x["Q"][:, :nl], x["K"][:, :nl], x["V"][:, :nl], x["W0_lin"], w.eta)
    Zc, _ = oracle.dwconv(x["Q"][:, nl:], x["K"][:, nl:], x["V"][:, nl:], x["W0_conv"], w.eta, w.H, w.W)
    Zr = np.concatenate([Zl, Zc], axis=1)
    assert rel_max_err(Z, Zr) <= TOL["bf16"]
    assert rel_max_err(Z[:, nl:], Zc) <= TOL["bf16"]


def test_dwconv_bitwise_deterministic(cuda_dev):
    x = _conv_inputs(4, 1, 40, 40, "bf16", seed=9)
    Z1, W1 = _run(x, 0.5, 40, 40, cuda_dev)
    Z2, W2 = _run(x, 0.5, 40, 40, cuda_dev)
    assert torch.equal(Z1, Z2) and torch.equal(W1, W2)
