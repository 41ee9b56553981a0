"""Parity of the MLP head's backward pass (ttt_backward_mlp through the C ABI) against the fp64
oracle, whose gradients are pinned to central differences of the pinned forward and to torch autograd
through the inner gradient.

Tolerances: dQ, dK, dV (rounded to the input dtype) and dWa, dWb (fp32, summed over images):
max|d - d_ref| / max|d_ref| at most 1e-2 for bf16 inputs and 1e-5 for fp32 inputs (fp32 arithmetic
from the exact inputs either way).  deta is a sum of products whose terms may cancel, so its error is
bounded against the sum of their magnitudes: |deta - ref| <= 1e-5 * sum (|dWa1| |gWa| + |dWb1| |gWb|).
"""
import numpy as np
import pytest
import torch

import oracle
from tests.parity import TOL, rel_max_err
from vision_test_token_b200 import WORKLOADS, backward_mlp, make_inputs
from vision_test_token_b200.inputs import Workload

pytestmark = pytest.mark.gpu


def _inputs(B, h, H, W, dtype, seed, hidden_ratio=4):
    return make_inputs(Workload("m", B, h, H, W, dtype, 0.5, "backward_mlp", hidden_ratio=hidden_ratio), seed)


def _gelu(u):
    return 0.5 * u * (1 + np.tanh(np.sqrt(2 / np.pi) * (u + 0.044715 * u ** 3)))


def _deta_scale(x, eta):
    """sum over units of |dWa1| |gWa| + |dWb1| |gWb|, the terms of deta (numpy, from the definitions)."""
    Q, K, V, dZ = (x[k].double().numpy() for k in ("Q", "K", "V", "dZ"))
    Wa, Wb = x["Wa"].double().numpy(), x["Wb"].double().numpy()
    _, Wa1, Wb1 = oracle.mlp(x["Q"], x["K"], x["V"], x["Wa"], x["Wb"], 1.0)
    tot = 0.0
    B, H = Q.shape[:2]
    d1 = np.vectorize(oracle.gelu_tanh_deriv)
    for b in range(B):
        for h in range(H):
            gA, gB = Wa[h] - Wa1[b, h], Wb[h] - Wb1[b, h]
            A1, B1 = Wa[h] - eta * gA, Wb[h] - eta * gB
            hq = Q[b, h] @ A1.T
            dhq = (dZ[b, h] @ B1) * d1(hq)
            dWa1, dWb1 = dhq.T @ Q[b, h], dZ[b, h].T @ _gelu(hq)
            tot += np.sum(np.abs(dWa1 * gA)) + np.sum(np.abs(dWb1 * gB))
    return tot


def _check(x, eta, H, W, dev, dtype, tight_deta=True):
    Q, K, V, dZ = (x[k].to(dev) for k in ("Q", "K", "V", "dZ"))
    out = backward_mlp(Q, K, V, x["Wa"].to(dev), x["Wb"].to(dev), eta, H, W, dZ)
    torch.cuda.synchronize()
    ref = oracle.mlp_backward(x["Q"], x["K"], x["V"], x["Wa"], x["Wb"], eta, x["dZ"])
    for name, got, r in zip(("dQ", "dK", "dV", "dWa", "dWb"), out[:5], ref[:5]):
        e = rel_max_err(got, r)
        assert e <= TOL[dtype], f"{name} rel err {e:.3g}"
    if tight_deta:
        assert abs(out[5].item() - ref[5]) <= 1e-5 * _deta_scale(x, eta) + 1e-30, (out[5].item(), ref[5])
    return out


@pytest.mark.parametrize("B,h,H,W,ratio", [
    (1, 1, 1, 1, 1), (2, 1, 5, 7, 2), (1, 2, 16, 16, 4), (3, 2, 9, 11, 3), (2, 1, 1, 37, 4), (5, 1, 3, 3, 4),
])
@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_mlp_backward_shapes(cuda_dev, B, h, H, W, ratio, dtype):
    _check(_inputs(B, h, H, W, dtype, seed=H * 13 + W + ratio, hidden_ratio=ratio), 0.5, H, W, cuda_dev, dtype)


def test_mlp_backward_full_workload(cuda_dev):
    """bwdmlp1024_bf16 at full size (16 images x 4 heads x 1024 tokens, hidden 256) against the oracle."""
    w = WORKLOADS["bwdmlp1024_bf16"]
    _check(make_inputs(w, seed=0), w.eta, w.H, w.W, cuda_dev, "bf16", tight_deta=False)


def test_mlp_backward_eta_zero(cuda_dev):
    """eta = 0: the head is z = Wb gelu(Wa q), so dK = dV = 0 exactly."""
    x = _inputs(2, 1, 6, 6, "fp32", seed=4, hidden_ratio=2)
    dev = cuda_dev
    Q, K, V, dZ = (x[k].to(dev) for k in ("Q", "K", "V", "dZ"))
    out = backward_mlp(Q, K, V, x["Wa"].to(dev), x["Wb"].to(dev), 0.0, 6, 6, dZ)
    torch.cuda.synchronize()
    assert torch.count_nonzero(out[1]).item() == 0 and torch.count_nonzero(out[2]).item() == 0
    ref = oracle.mlp_backward(x["Q"], x["K"], x["V"], x["Wa"], x["Wb"], 0.0, x["dZ"])
    for got, r in zip((out[0], out[3], out[4]), (ref[0], ref[3], ref[4])):
        assert rel_max_err(got, r) <= TOL["fp32"]


def test_mlp_backward_bitwise_deterministic(cuda_dev):
    x = _inputs(2, 2, 8, 9, "bf16", seed=9)
    dev = cuda_dev
    args = [x[k].to(dev) for k in ("Q", "K", "V")]
    a = backward_mlp(*args, x["Wa"].to(dev), x["Wb"].to(dev), 0.5, 8, 9, x["dZ"].to(dev))
    b = backward_mlp(*args, x["Wa"].to(dev), x["Wb"].to(dev), 0.5, 8, 9, x["dZ"].to(dev))
    torch.cuda.synchronize()
    assert all(torch.equal(p, q) for p, q in zip(a, b))
