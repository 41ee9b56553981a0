"""Parity of the whole layer call (ttt_forward_layer through the C ABI: linear heads and
depthwise-conv heads of one view, the two kernels running at the same time) against the fp64
oracle, on Z and on both weight updates; bitwise reproducibility with a reused workspace."""
import numpy as np
import pytest
import torch

import oracle
from tests.parity import TOL, rel_max_err, rel_update_err
from vision_test_token_b200 import capi, forward_layer, workspace_status
from vision_test_token_b200.inputs import random_unit
from vision_test_token_b200.layer import layer_workspace, _shape_of

pytestmark = pytest.mark.gpu


def _run(x, w, dev, concurrent=True, max_sms=0):
    Q, K, V = (x[k].to(dev) for k in ("Q", "K", "V"))
    B, nl, nc = Q.shape[0], w.lin_heads, w.conv_heads
    Z = torch.full_like(Q, float("nan"))
    W1l = torch.full((B, nl, 64, 64), float("nan"), device=dev) if nl else None
    W1c = torch.full((B, nc, 64, 3, 3), float("nan"), device=dev) if nc else None
    weights = {k: v.to(dev) for k, v in x.items() if k.startswith("W0")}
    forward_layer(Q, K, V, weights, w.eta, w.H, w.W, conv_heads=nc, Z=Z, W1_lin_out=W1l, W1_conv_out=W1c,
                  concurrent=concurrent, max_sms=max_sms)
    torch.cuda.synchronize()
    return Z, W1l, W1c


def _check(x, w, dev, **kw):
    Z, W1l, W1c = _run(x, w, dev, **kw)
    nl = w.lin_heads
    tol = TOL[w.dtype]
    parts = []
    if nl:
        Zl, W1lr = oracle.linear(x["Q"][:, :nl], x["K"][:, :nl], x["V"][:, :nl], x["W0_lin"], w.eta)
        assert rel_update_err(W1l, W1lr, x["W0_lin"].double().numpy()[None]) <= tol
        parts.append(Zl)
    if w.conv_heads:
        Zc, W1cr = oracle.dwconv(x["Q"][:, nl:], x["K"][:, nl:], x["V"][:, nl:], x["W0_conv"], w.eta, w.H, w.W)
        assert rel_update_err(W1c, W1cr, x["W0_conv"].double().numpy()[None]) <= tol
        assert rel_max_err(Z[:, nl:], Zc) <= tol
        parts.append(Zc)
    assert rel_max_err(Z, np.concatenate(parts, axis=1)) <= tol
    return Z, W1l, W1c


@pytest.mark.parametrize("B,heads,conv,H,W", [
    (8, 6, 1, 78, 78), (3, 4, 2, 13, 17), (2, 3, 3, 9, 9), (2, 3, 0, 9, 9), (1, 2, 1, 1, 1), (5, 2, 1, 31, 90),
    (70, 3, 1, 14, 14),
])
@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_layer_shapes(cuda_dev, B, heads, conv, H, W, dtype):
    w, x = random_unit(B, heads, H, W, dtype=dtype, seed=B + 10 * heads + H, kind="mixed", conv_heads=conv,
                       eta=0.5)
    _check(x, w, cuda_dev)


@pytest.mark.parametrize("max_sms", [1, 9, 64])
def test_layer_sm_budget(cuda_dev, max_sms):
    w, x = random_unit(8, 6, 40, 40, dtype="bf16", seed=3, kind="mixed", conv_heads=1, eta=0.5)
    _check(x, w, cuda_dev, max_sms=max_sms)


def test_layer_bitwise_reproducible_with_reused_workspace(cuda_dev):
    w, x = random_unit(8, 6, 78, 78, dtype="bf16", seed=5, kind="mixed", conv_heads=1, eta=0.5)
    runs = [_run(x, w, cuda_dev) for _ in range(3)]
    for Z, W1l, W1c in runs[1:]:
        assert torch.equal(Z, runs[0][0]) and torch.equal(W1l, runs[0][1]) and torch.equal(W1c, runs[0][2])
    shape = _shape_of(x["Q"].to(cuda_dev), w.H, w.W)
    ws = layer_workspace(shape, w.conv_heads, cuda_dev)
    assert workspace_status(ws) == capi.TTT_OK


def test_layer_matches_the_two_calls(cuda_dev):
    """The concurrent layer call and the two separate calls give the same Z bit for bit.  At this size
    the SM budgets do not change the work split: the 10 linear units use 8-CTA clusters (the largest)
    either way and every conv row pair is its own task either way."""
    w, x = random_unit(2, 6, 30, 30, dtype="bf16", seed=8, kind="mixed", conv_heads=1, eta=0.5)
    a = _run(x, w, cuda_dev, concurrent=True)
    b = _run(x, w, cuda_dev, concurrent=False)
    for u, v in zip(a, b):
        assert torch.equal(u, v)
