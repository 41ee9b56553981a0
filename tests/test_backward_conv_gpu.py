"""Parity of the depthwise-conv head's backward pass (ttt_backward_dwconv through the C ABI) against
the fp64 oracle, whose gradients are pinned to central differences of the pinned forward and to torch
autograd.

Tolerances: dQ, dK, dV (rounded to the input dtype) and dW0 (fp32, summed over images):
max|d - d_ref| / max|d_ref| at most 1e-2 for bf16 inputs and 1e-5 for fp32 inputs (fp32 arithmetic
from the exact inputs either way).  deta is a sum of products whose terms may cancel, so its error is
bounded against the sum of their magnitudes: |deta - ref| <= 1e-5 * sum |dW1| |g| over all units.
"""
import numpy as np
import pytest
import torch

import oracle
from tests.parity import TOL, rel_max_err
from vision_test_token_b200 import WORKLOADS, backward_dwconv, make_inputs
from vision_test_token_b200.inputs import Workload

pytestmark = pytest.mark.gpu


def _inputs(B, h, H, W, dtype, seed):
    return make_inputs(Workload("c", B, h, H, W, dtype, 0.5, "backward_conv", conv_heads=h), seed)


def _deta_scale(x, H, W):
    """sum over units and taps of |dW1| |g|, from the oracle's own forward quantities."""
    Q, K, V, dZ = (x[k].double().numpy() for k in ("Q", "K", "V", "dZ"))
    W0 = x["W0_conv"].double().numpy()
    B, h, N, d = Q.shape
    _, W1 = oracle.dwconv(x["Q"], x["K"], x["V"], x["W0_conv"], 1.0, H, W)     # eta = 1: W0 - W1 = g
    g = W0[None] - W1
    pad = lambda X: np.pad(X.reshape(B, h, H, W, d), ((0, 0), (0, 0), (1, 1), (1, 1), (0, 0)))
    Qp = pad(Q)
    dz = dZ.reshape(B, h, H, W, d)
    dW1 = np.stack([np.stack([np.einsum("bhyxc,bhyxc->bhc", dz, Qp[:, :, a:a + H, b:b + W]) for b in range(3)], -1)
                    for a in range(3)], -2)
    return float(np.sum(np.abs(dW1) * np.abs(g)))


def _check(x, eta, H, W, dev, dtype):
    Q, K, V, dZ = (x[k].to(dev) for k in ("Q", "K", "V", "dZ"))
    dQ, dK, dV, dW0, deta = backward_dwconv(Q, K, V, x["W0_conv"].to(dev), eta, H, W, dZ)
    torch.cuda.synchronize()
    rq, rk, rv, rw, re = oracle.dwconv_backward(x["Q"], x["K"], x["V"], x["W0_conv"], eta, x["dZ"], H, W)
    for name, got, ref in (("dQ", dQ, rq), ("dK", dK, rk), ("dV", dV, rv), ("dW0", dW0, rw)):
        e = rel_max_err(got, ref)
        assert e <= TOL[dtype], f"{name} rel err {e:.3g}"
    assert abs(deta.item() - re) <= 1e-5 * _deta_scale(x, H, W) + 1e-30, (deta.item(), re)
    return dQ, dK, dV, dW0, deta


@pytest.mark.parametrize("B,h,H,W", [
    (1, 1, 1, 1), (1, 1, 1, 19), (1, 1, 17, 1), (2, 1, 9, 20), (1, 2, 16, 16), (3, 2, 13, 33), (2, 1, 40, 7),
])
@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_dwconv_backward_shapes(cuda_dev, B, h, H, W, dtype):
    _check(_inputs(B, h, H, W, dtype, seed=H * 7 + W), 0.5, H, W, cuda_dev, dtype)


def test_dwconv_backward_full_workload(cuda_dev):
    """bwdconv6084_bf16 at full size (8 images x 78 x 78) against the oracle on every unit."""
    w = WORKLOADS["bwdconv6084_bf16"]
    _check(make_inputs(w, seed=0), w.eta, w.H, w.W, cuda_dev, "bf16")


def test_dwconv_backward_eta_zero(cuda_dev):
    """eta = 0: the head is Z = f(Q; W0), so dK = dV = 0 exactly; deta = -sum dW1 g does not vanish
    (g does not depend on eta) and matches the oracle."""
    x = _inputs(2, 1, 10, 12, "fp32", seed=3)
    dev = cuda_dev
    Q, K, V, dZ = (x[k].to(dev) for k in ("Q", "K", "V", "dZ"))
    dQ, dK, dV, dW0, deta = backward_dwconv(Q, K, V, x["W0_conv"].to(dev), 0.0, 10, 12, dZ)
    torch.cuda.synchronize()
    assert torch.count_nonzero(dK).item() == 0 and torch.count_nonzero(dV).item() == 0
    rq, _, _, rw, re = oracle.dwconv_backward(x["Q"], x["K"], x["V"], x["W0_conv"], 0.0, x["dZ"], 10, 12)
    assert rel_max_err(dQ, rq) <= TOL["fp32"] and rel_max_err(dW0, rw) <= TOL["fp32"]
    assert abs(deta.item() - re) <= 1e-5 * _deta_scale(x, 10, 12)


def test_dwconv_backward_bitwise_deterministic(cuda_dev):
    x = _inputs(2, 2, 20, 21, "bf16", seed=9)
    dev = cuda_dev
    args = [x[k].to(dev) for k in ("Q", "K", "V")]
    a = backward_dwconv(*args, x["W0_conv"].to(dev), 0.5, 20, 21, x["dZ"].to(dev))
    b = backward_dwconv(*args, x["W0_conv"].to(dev), 0.5, 20, 21, x["dZ"].to(dev))
    torch.cuda.synchronize()
    assert all(torch.equal(p, q) for p, q in zip(a, b))
