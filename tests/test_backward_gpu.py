"""Parity of the linear head's backward pass (ttt_backward_linear through the C ABI) against the
fp64 oracle, whose gradients are pinned to central differences of the pinned forward and to torch
autograd.

Tolerances: dQ, dK, dV (rounded to the input dtype) and dW0 (fp32, summed over images):
max|d - d_ref| / max|d_ref| at most 1e-2 for bf16 inputs and 1e-5 for fp32 inputs (fp32 arithmetic
from the exact inputs either way).  deta is one sum of d*d products per unit whose terms may cancel,
so its error is bounded against the sum of their magnitudes: |deta - ref| <= 1e-5 * (2/N) *
sum |dW1| |W0 G - C| over all units.
"""
import numpy as np
import pytest
import torch

import oracle
from tests.parity import TOL, rel_max_err
from vision_test_token_b200 import WORKLOADS, backward_linear, make_inputs
from vision_test_token_b200.inputs import random_unit

pytestmark = pytest.mark.gpu


def _deta_scale(x, N):
    Q, K, V, dZ = (x[k].double().numpy() for k in ("Q", "K", "V", "dZ"))
    W0 = x["W0_lin"].double().numpy()
    G = np.einsum("bhni,bhnj->bhij", K, K)
    C = np.einsum("bhni,bhnj->bhij", V, K)
    dW1 = np.einsum("bhni,bhnj->bhij", dZ, Q)
    P = np.einsum("hik,bhkj->bhij", W0, G) - C
    return 2.0 / N * float(np.sum(np.abs(dW1) * np.abs(P)))


def _check(x, eta, H, W, dev, dtype):
    Q, K, V, dZ = (x[k].to(dev) for k in ("Q", "K", "V", "dZ"))
    dQ, dK, dV, dW0, deta = backward_linear(Q, K, V, x["W0_lin"].to(dev), eta, H, W, dZ)
    torch.cuda.synchronize()
    rq, rk, rv, rw, re = oracle.linear_backward(x["Q"], x["K"], x["V"], x["W0_lin"], eta, x["dZ"])
    for name, got, ref in (("dQ", dQ, rq), ("dK", dK, rk), ("dV", dV, rv), ("dW0", dW0, rw)):
        e = rel_max_err(got, ref)
        assert e <= TOL[dtype], f"{name} rel err {e:.3g}"
    assert abs(deta.item() - re) <= 1e-5 * _deta_scale(x, H * W) + 1e-30, (deta.item(), re)
    return dQ, dK, dV, dW0, deta


def _inputs(B, h, H, W, dtype, seed):
    w, x = random_unit(B, h, H, W, dtype=dtype, seed=seed, kind="backward")
    return x


@pytest.mark.parametrize("B,h,H,W", [
    (1, 1, 1, 1),        # a single token
    (2, 2, 9, 11),       # one ragged tile per unit
    (3, 1, 20, 20),      # several tiles per unit
    (1, 3, 3, 43),       # one full tile + 1 token
    (2, 3, 77, 79),      # ragged large units
    (37, 1, 15, 20),     # more units than fit one per CTA: CTAs span several units
])
@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_backward_shapes(cuda_dev, B, h, H, W, dtype):
    _check(_inputs(B, h, H, W, dtype, seed=B * 1000 + H * 10 + W), 0.5, H, W, cuda_dev, dtype)


def test_backward_eta_zero(cuda_dev):
    """eta = 0: the layer is z = W0 q, so dK = dV = 0 exactly and dQ = W0^T dz."""
    x = _inputs(2, 2, 10, 10, "fp32", seed=3)
    dev = cuda_dev
    dQ, dK, dV, dW0, deta = backward_linear(*(x[k].to(dev) for k in ("Q", "K", "V")), x["W0_lin"].to(dev), 0.0,
                                            10, 10, x["dZ"].to(dev))
    assert torch.count_nonzero(dK).item() == 0 and torch.count_nonzero(dV).item() == 0
    ref = np.einsum("hij,bhni->bhnj", x["W0_lin"].double().numpy(), x["dZ"].double().numpy())
    assert rel_max_err(dQ, ref) <= TOL["fp32"]


def test_backward_bitwise_repeatable(cuda_dev):
    x = _inputs(3, 2, 30, 30, "bf16", seed=4)
    dev = cuda_dev
    args = [x[k].to(dev) for k in ("Q", "K", "V")] + [x["W0_lin"].to(dev), 0.5, 30, 30, x["dZ"].to(dev)]
    a = backward_linear(*args)
    b = backward_linear(*args)
    for ta, tb in zip(a, b):
        assert torch.equal(ta, tb)


def test_backward_workload_full(cuda_dev):
    """The backward bench workload at full size (8 images x 5 heads x 78 x 78 tokens, bf16)."""
    w = WORKLOADS["bwd6084_bf16"]
    _check(make_inputs(w), w.eta, w.H, w.W, cuda_dev, "bf16")
