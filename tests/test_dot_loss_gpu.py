"""Parity of the dot-product inner loss (ttt_shape.loss = TTT_LOSS_DOT through the C ABI) against
the fp64 oracle, for the linear head, the depthwise-conv head and the layer call that runs both.

The loss is L(W) = -(1/N) sum <f(k_n; W), v_n> (the ViT3 recipe of the press article, section on the
ViT3 model; the pages name the loss without printing it).  Tolerances as for the L2 loss:
max|dZ| / max|Z_ref| and max|dW - dW_ref| / max|dW_ref| (dW = W1 - W0) at most 1e-2 for bf16
inputs and 1e-5 for fp32 inputs.
"""
import numpy as np
import pytest
import torch

import oracle
from tests.parity import TOL, rel_max_err, rel_update_err
from vision_test_token_b200 import WORKLOADS, forward_dwconv, forward_layer, forward_linear, make_inputs
from vision_test_token_b200.inputs import random_unit

pytestmark = pytest.mark.gpu


def _lin(x, eta, H, W, dev, dtype, max_sms=0):
    Q, K, V = (x[k].to(dev) for k in ("Q", "K", "V"))
    B, h = Q.shape[:2]
    W1 = torch.full((B, h, 64, 64), float("nan"), device=dev)
    Z = forward_linear(Q, K, V, x["W0_lin"].to(dev), eta, H, W, W1_out=W1, max_sms=max_sms, loss="dot")
    torch.cuda.synchronize()
    Zr, W1r = oracle.linear_dot(x["Q"], x["K"], x["V"], x["W0_lin"], eta)
    ez, ew = rel_max_err(Z, Zr), rel_update_err(W1, W1r, x["W0_lin"].double().numpy()[None])
    assert ez <= TOL[dtype], f"Z rel err {ez:.3g}"
    assert ew <= TOL[dtype], f"dW rel err {ew:.3g}"


def _conv(x, eta, H, W, dev, dtype, max_sms=0):
    Q, K, V = (x[k].to(dev) for k in ("Q", "K", "V"))
    B, h = Q.shape[:2]
    W1 = torch.full((B, h, 64, 3, 3), float("nan"), device=dev)
    Z = forward_dwconv(Q, K, V, x["W0_conv"].to(dev), eta, H, W, W1_out=W1, max_sms=max_sms, loss="dot")
    torch.cuda.synchronize()
    Zr, W1r = oracle.dwconv_dot(x["Q"], x["K"], x["V"], x["W0_conv"], eta, H, W)
    ez, ew = rel_max_err(Z, Zr), rel_update_err(W1, W1r, x["W0_conv"].double().numpy()[None])
    assert ez <= TOL[dtype], f"Z rel err {ez:.3g}"
    assert ew <= TOL[dtype], f"dW rel err {ew:.3g}"


@pytest.mark.parametrize("B,h,H,W", [
    (1, 1, 1, 1),        # a single token
    (1, 2, 3, 43),       # one full tile + 1 token
    (37, 1, 15, 20),     # 3 tiles per unit
    (200, 1, 10, 13),    # many small units
    (2, 3, 77, 79),      # ragged large units
    (8, 5, 78, 78),      # the linear heads of the 1248^2 layer
])
@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_linear_dot_shapes(cuda_dev, B, h, H, W, dtype):
    _, x = random_unit(B, h, H, W, dtype=dtype, seed=7 * B + H * 10 + W)
    _lin(x, 1.0, H, W, cuda_dev, dtype)


@pytest.mark.parametrize("max_sms", [1, 7, 80])
def test_linear_dot_sm_budget(cuda_dev, max_sms):
    _, x = random_unit(8, 5, 30, 40, dtype="bf16", seed=max_sms)
    _lin(x, 1.0, 30, 40, cuda_dev, "bf16", max_sms=max_sms)


def test_linear_dot_eta_zero_is_plain_readout(cuda_dev):
    _, x = random_unit(2, 2, 12, 12, dtype="fp32", seed=3)
    _lin(x, 0.0, 12, 12, cuda_dev, "fp32")


@pytest.mark.parametrize("B,h,H,W", [
    (1, 1, 1, 1), (1, 1, 1, 9), (1, 1, 9, 1), (2, 1, 5, 7), (2, 1, 33, 17), (8, 1, 78, 78), (1, 1, 7, 170),
    (300, 1, 3, 5),
])
@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_dwconv_dot_shapes(cuda_dev, B, h, H, W, dtype):
    x = random_unit(B, h, H, W, dtype=dtype, seed=H * 100 + W + 1, kind="mixed", conv_heads=h)[1]
    _conv(x, 1.0, H, W, cuda_dev, dtype)


@pytest.mark.parametrize("max_sms", [1, 20])
def test_dwconv_dot_sm_budget(cuda_dev, max_sms):
    x = random_unit(4, 1, 26, 30, dtype="bf16", seed=max_sms, kind="mixed", conv_heads=1)[1]
    _conv(x, 1.0, 26, 30, cuda_dev, "bf16", max_sms=max_sms)


def test_dot_update_does_not_depend_on_w0(cuda_dev):
    """The dot-product loss's update is (eta/N) sum v k^T whatever W0 is: two W0 give the same W1 - W0
    (exactly for fp32 inputs up to the final W0 + update rounding)."""
    _, x = random_unit(3, 2, 20, 20, dtype="fp32", seed=11)
    dev = cuda_dev
    Q, K, V = (x[k].to(dev) for k in ("Q", "K", "V"))
    ups = []
    for W0 in (x["W0_lin"], torch.zeros_like(x["W0_lin"])):
        W1 = torch.empty((3, 2, 64, 64), device=dev)
        forward_linear(Q, K, V, W0.to(dev), 1.0, 20, 20, W1_out=W1, loss="dot")
        ups.append((W1.cpu().double() - W0.double()[None]).numpy())
    np.testing.assert_allclose(ups[0], ups[1], atol=1e-6, rtol=0)


@pytest.mark.parametrize("B,heads,conv,H,W", [(8, 6, 1, 78, 78), (3, 4, 2, 13, 17), (1, 2, 1, 1, 1)])
@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("concurrent", [True, False])
def test_layer_dot(cuda_dev, B, heads, conv, H, W, dtype, concurrent):
    w, x = random_unit(B, heads, H, W, dtype=dtype, seed=B + heads + H, kind="mixed", conv_heads=conv, eta=1.0)
    dev = cuda_dev
    nl = heads - conv
    Q, K, V = (x[k].to(dev) for k in ("Q", "K", "V"))
    Z = torch.full_like(Q, float("nan"))
    W1l = torch.full((B, nl, 64, 64), float("nan"), device=dev)
    W1c = torch.full((B, conv, 64, 3, 3), float("nan"), device=dev)
    weights = {k: v.to(dev) for k, v in x.items() if k.startswith("W0")}
    forward_layer(Q, K, V, weights, 1.0, H, W, conv_heads=conv, Z=Z, W1_lin_out=W1l, W1_conv_out=W1c,
                  concurrent=concurrent, loss="dot")
    torch.cuda.synchronize()
    Zl, W1lr = oracle.linear_dot(x["Q"][:, :nl], x["K"][:, :nl], x["V"][:, :nl], x["W0_lin"], 1.0)
    Zc, W1cr = oracle.dwconv_dot(x["Q"][:, nl:], x["K"][:, nl:], x["V"][:, nl:], x["W0_conv"], 1.0, H, W)
    tol = TOL[dtype]
    assert rel_update_err(W1l, W1lr, x["W0_lin"].double().numpy()[None]) <= tol
    assert rel_update_err(W1c, W1cr, x["W0_conv"].double().numpy()[None]) <= tol
    assert rel_max_err(Z[:, nl:], Zc) <= tol
    assert rel_max_err(Z, np.concatenate([Zl, Zc], axis=1)) <= tol


def test_dot_workload_full(cuda_dev):
    """The dot-loss layer workload at its full size (8 images x 6 heads x 78 x 78, 5 linear + 1 conv
    head), whole output against the oracle."""
    w = WORKLOADS["mixed6084_dot_bf16"]
    x = make_inputs(w)
    dev = cuda_dev
    Q, K, V = (x[k].to(dev) for k in ("Q", "K", "V"))
    weights = {k: v.to(dev) for k, v in x.items() if k.startswith("W0")}
    Z = forward_layer(Q, K, V, weights, w.eta, w.H, w.W, conv_heads=w.conv_heads, loss=w.loss)
    torch.cuda.synchronize()
    nl = w.lin_heads
    Zl, _ = oracle.linear_dot(x["Q"][:, :nl], x["K"][:, :nl], x["V"][:, :nl], x["W0_lin"], w.eta)
    Zc, _ = oracle.dwconv_dot(x["Q"][:, nl:], x["K"][:, nl:], x["V"][:, nl:], x["W0_conv"], w.eta, w.H, w.W)
    assert rel_max_err(Z, np.concatenate([Zl, Zc], axis=1)) <= TOL["bf16"]


def test_mlp_rejects_the_dot_loss(cuda_dev):
    from vision_test_token_b200 import capi, forward_mlp
    _, x = random_unit(1, 1, 4, 4, dtype="bf16", seed=1, kind="mlp")
    dev = cuda_dev
    with pytest.raises(capi.TttError) as e:
        forward_mlp(x["Q"].to(dev), x["K"].to(dev), x["V"].to(dev), x["Wa"].to(dev), x["Wb"].to(dev), 0.5, 4, 4,
                    loss="dot")
    assert e.value.status == capi.TTT_ERR_UNSUPPORTED
