"""The seeded input recipe (vision_test_token_b200/inputs.py): shapes, the documented distributions
and reproducibility.  The module only draws random numbers; both the CUDA path and the oracle read
the tensors it returns."""
import math

import pytest
import torch

from vision_test_token_b200 import WORKLOADS, make_inputs
from vision_test_token_b200.inputs import random_unit


@pytest.mark.parametrize("kind", ["linear", "mixed", "mlp", "minibatch", "backward"])
def test_shapes_and_keys(kind):
    w, x = random_unit(2, 3, 5, 7, dtype="fp32", seed=1, kind=kind, conv_heads=1 if kind == "mixed" else 0)
    for k in ("Q", "K", "V"):
        assert x[k].shape == (2, 3, 35, 64) and x[k].dtype == torch.float32
    assert ("dZ" in x) == (kind == "backward")
    if kind in ("linear", "minibatch", "backward"):
        assert x["W0_lin"].shape == (3, 64, 64)
    if kind == "mixed":
        assert x["W0_lin"].shape == (2, 64, 64) and x["W0_conv"].shape == (1, 64, 3, 3)
    if kind == "mlp":
        assert x["Wa"].shape == (3, 256, 64) and x["Wb"].shape == (3, 64, 256)


def test_query_and_key_rows_are_unit_norm_and_values_are_not():
    _, x = random_unit(1, 2, 20, 20, dtype="fp32", seed=2)
    for k in ("Q", "K"):
        torch.testing.assert_close(x[k].norm(dim=-1), torch.ones(1, 2, 400), rtol=1e-6, atol=1e-6)
    assert abs(float(x["V"].std()) - 1.0) < 0.05
    assert abs(float(x["W0_lin"].std()) - 1 / math.sqrt(64)) < 0.01


def test_seeded_and_bf16_is_a_rounding_of_the_fp32_draws():
    w = WORKLOADS["lin196_bf16"]
    a, b = make_inputs(w, seed=3), make_inputs(w, seed=3)
    assert all(torch.equal(a[k], b[k]) for k in a)
    c = make_inputs(w, seed=4)
    assert not torch.equal(a["Q"], c["Q"])
    _, x32 = random_unit(1, 1, 14, 14, dtype="fp32", seed=5)
    _, x16 = random_unit(1, 1, 14, 14, dtype="bf16", seed=5)
    for k in ("Q", "K", "V"):
        assert torch.equal(x32[k].to(torch.bfloat16), x16[k])
    assert torch.equal(x32["W0_lin"], x16["W0_lin"])          # weights stay fp32


def test_the_backward_gradient_is_drawn_after_the_weights():
    """Adding dZ does not change the forward inputs of the same seed."""
    _, xf = random_unit(1, 2, 6, 6, dtype="fp32", seed=6)
    _, xb = random_unit(1, 2, 6, 6, dtype="fp32", seed=6, kind="backward")
    for k in ("Q", "K", "V", "W0_lin"):
        assert torch.equal(xf[k], xb[k])
