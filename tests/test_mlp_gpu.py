"""Parity of the MLP head (ttt_forward_mlp through the C ABI) against the fp64 oracle:
max|dZ| / max|Z_ref| <= 1e-2 (bf16 inputs, fp32 accumulation), and the same bound on each update,
Wa1 - Wa and Wb1 - Wb."""
import numpy as np
import pytest
import torch

import oracle
from tests.parity import TOL, rel_max_err, rel_update_err
from vision_test_token_b200 import WORKLOADS, forward_mlp, make_inputs
from vision_test_token_b200.inputs import random_unit

pytestmark = pytest.mark.gpu


def _run(x, eta, H, W, dev, max_sms=0):
    Q, K, V = (x[k].to(dev) for k in ("Q", "K", "V"))
    Wa, Wb = x["Wa"].to(dev), x["Wb"].to(dev)
    B, h = Q.shape[:2]
    Wa1 = torch.full((B, h) + tuple(Wa.shape[1:]), float("nan"), device=dev)
    Wb1 = torch.full((B, h) + tuple(Wb.shape[1:]), float("nan"), device=dev)
    Z = forward_mlp(Q, K, V, Wa, Wb, eta, H, W, Wa_out=Wa1, Wb_out=Wb1, max_sms=max_sms)
    torch.cuda.synchronize()
    return Z, Wa1, Wb1


def _check(x, eta, H, W, dev, max_sms=0):
    Z, Wa1, Wb1 = _run(x, eta, H, W, dev, max_sms)
    Zr, Wa1r, Wb1r = oracle.mlp(x["Q"], x["K"], x["V"], x["Wa"], x["Wb"], eta)
    ez = rel_max_err(Z, Zr)
    ea = rel_update_err(Wa1, Wa1r, x["Wa"].double().numpy()[None])
    eb = rel_update_err(Wb1, Wb1r, x["Wb"].double().numpy()[None])
    assert ez <= TOL["bf16"], f"Z rel err {ez:.3g}"
    assert ea <= TOL["bf16"], f"dWa rel err {ea:.3g}"
    assert eb <= TOL["bf16"], f"dWb rel err {eb:.3g}"
    return ez, ea, eb


def test_mlp1024_workload_full(cuda_dev):
    w = WORKLOADS["mlp1024_bf16"]
    _check(make_inputs(w), w.eta, w.H, w.W, cuda_dev)


# (2, 1, 10, 13): two CTAs per unit, the second with a 2-token tile; (40, 2, 16, 16): more units than
# SM pairs, one CTA per unit; (200, 1, 4, 4): one tile per unit
@pytest.mark.parametrize("B,h,H,W", [(1, 1, 1, 1), (2, 1, 10, 13), (1, 3, 8, 16), (3, 2, 20, 20), (200, 1, 4, 4),
                                     (40, 2, 16, 16)])
def test_mlp_shapes(cuda_dev, B, h, H, W):
    _, x = random_unit(B, h, H, W, dtype="bf16", seed=B * 7 + H, kind="mlp")
    _check(x, 0.5, H, W, cuda_dev)


def test_mlp_eta_zero_is_plain_readout(cuda_dev):
    _, x = random_unit(2, 2, 12, 12, dtype="bf16", seed=5, kind="mlp")
    Z, Wa1, Wb1 = _run(x, 0.0, 12, 12, cuda_dev)
    Zr, _, _ = oracle.mlp(x["Q"], x["K"], x["V"], x["Wa"], x["Wb"], 0.0)
    assert rel_max_err(Z, Zr) <= TOL["bf16"]
    assert torch.equal(Wa1.cpu(), x["Wa"][None].expand_as(Wa1.cpu()))


def test_mlp_bitwise_deterministic(cuda_dev):
    _, x = random_unit(4, 2, 16, 16, dtype="bf16", seed=6, kind="mlp")
    Z1, A1, B1 = _run(x, 0.5, 16, 16, cuda_dev)
    Z2, A2, B2 = _run(x, 0.5, 16, 16, cuda_dev)
    assert torch.equal(Z1, Z2) and torch.equal(A1, A2) and torch.equal(B1, B2)


@pytest.mark.parametrize("max_sms", [1, 3, 20])
def test_mlp_sm_budget(cuda_dev, max_sms):
    """One CTA for every unit, a few persistent CTAs, and 2-CTA clusters: the same results within
    tolerance."""
    _, x = random_unit(3, 2, 20, 20, dtype="bf16", seed=11, kind="mlp")
    _check(x, 0.5, 20, 20, cuda_dev, max_sms)
