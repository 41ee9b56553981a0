"""Golden fixtures: the pages' printed figures and the oracle's regression record."""
import json
import math
import os

import numpy as np

import oracle
from vision_test_token_b200.inputs import WORKLOADS, random_unit

GOLD = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _load(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


def test_workload_grids_are_the_pages_token_counts():
    figs = _load("page_figures.json")
    counts = {g["image"]: g["tokens"] for g in figs["token_grids"]}
    for g in figs["token_grids"]:
        assert (g["image"] // g["patch"]) ** 2 == g["tokens"]
    assert WORKLOADS["lin196_bf16"].N == counts[224]
    assert WORKLOADS["lin196_fp32"].N == counts[224]
    assert WORKLOADS["mixed6084_bf16"].N == counts[1248]
    assert WORKLOADS["lin6400_bf16"].N == counts[1280]
    for w in WORKLOADS.values():
        assert w.d == figs["head_state"]["d"]
    mb = figs["minibatch_example"]
    assert math.ceil(mb["tokens"] / mb["b"]) == mb["steps"]


def test_linear_flop_model_matches_the_pages_inner_term():
    """The pages' inner complexity term 6*T*D*d with D = n_h*d is 6*d^2*T per head: the FLOP count
    used for the linear head's roofline (Gram 4 d^2 T + readout 2 d^2 T)."""
    for w in WORKLOADS.values():
        D = w.heads * w.d
        assert 6 * w.N * D * w.d == w.heads * (4 * w.d ** 2 * w.N + 2 * w.d ** 2 * w.N)


def test_oracle_regression_record():
    g = _load("oracle_regression.json")
    _, x = random_unit(1, 1, 3, 4, d=8, dtype="fp32", seed=g["linear"]["seed"])
    Z, W1 = oracle.linear(x["Q"], x["K"], x["V"], x["W0_lin"], g["linear"]["eta"])
    np.testing.assert_allclose(Z[0, 0, 0], g["linear"]["Z_row0"], rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(W1[0, 0, 0], g["linear"]["W1_row0"], rtol=1e-13, atol=1e-15)
    assert abs(Z.sum() - g["linear"]["Z_sum"]) < 1e-12
    _, x = random_unit(1, 1, 3, 4, d=8, dtype="fp32", seed=g["dwconv"]["seed"], kind="mixed",
                       conv_heads=1)
    Z, W1 = oracle.dwconv(x["Q"], x["K"], x["V"], x["W0_conv"], g["dwconv"]["eta"], 3, 4)
    np.testing.assert_allclose(Z[0, 0, 0], g["dwconv"]["Z_row0"], rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(W1[0, 0, 0].ravel(), g["dwconv"]["W1_ch0"], rtol=1e-13, atol=1e-15)
    _, x = random_unit(1, 1, 3, 4, d=8, dtype="fp32", seed=g["mlp"]["seed"], kind="mlp")
    Z, Wa1, Wb1 = oracle.mlp(x["Q"], x["K"], x["V"], x["Wa"], x["Wb"], g["mlp"]["eta"])
    np.testing.assert_allclose(Z[0, 0, 0], g["mlp"]["Z_row0"], rtol=1e-13, atol=1e-15)
    assert abs(Wa1.sum() - g["mlp"]["Wa1_sum"]) < 1e-11
    assert abs(Wb1.sum() - g["mlp"]["Wb1_sum"]) < 1e-11


def test_oracle_regression_record_of_the_variants():
    """The dot-loss, mini-batch and backward oracles reproduce their recorded values."""
    g = _load("oracle_regression.json")
    _, x = random_unit(1, 1, 3, 4, d=8, dtype="fp32", seed=g["linear_dot"]["seed"])
    Z, W1 = oracle.linear_dot(x["Q"], x["K"], x["V"], x["W0_lin"], g["linear_dot"]["eta"])
    np.testing.assert_allclose(Z[0, 0, 0], g["linear_dot"]["Z_row0"], rtol=1e-13, atol=1e-15)
    assert abs(W1.sum() - g["linear_dot"]["W1_sum"]) < 1e-12
    _, x = random_unit(1, 1, 3, 4, d=8, dtype="fp32", seed=g["dwconv_dot"]["seed"], kind="mixed", conv_heads=1)
    Z, W1 = oracle.dwconv_dot(x["Q"], x["K"], x["V"], x["W0_conv"], g["dwconv_dot"]["eta"], 3, 4)
    np.testing.assert_allclose(Z[0, 0, 0], g["dwconv_dot"]["Z_row0"], rtol=1e-13, atol=1e-15)
    assert abs(W1.sum() - g["dwconv_dot"]["W1_sum"]) < 1e-12
    for mode in ("prefix", "epoch"):
        rec = g["linear_minibatch_" + mode]
        _, x = random_unit(1, 1, 3, 4, d=8, dtype="fp32", seed=rec["seed"])
        Z, W1 = oracle.linear_minibatch(x["Q"], x["K"], x["V"], x["W0_lin"], rec["eta"], rec["b"], mode)
        np.testing.assert_allclose(Z[0, 0, 0], rec["Z_row0"], rtol=1e-13, atol=1e-15)
        assert abs(W1.sum() - rec["W1_sum"]) < 1e-12
    rec = g["linear_backward"]
    _, x = random_unit(2, 1, 3, 4, d=8, dtype="fp32", seed=rec["seed"], kind="backward")
    dQ, dK, dV, dW0, deta = oracle.linear_backward(x["Q"], x["K"], x["V"], x["W0_lin"], rec["eta"], x["dZ"])
    for name, a in (("dQ_row0", dQ), ("dK_row0", dK), ("dV_row0", dV)):
        np.testing.assert_allclose(a[0, 0, 0], rec[name], rtol=1e-13, atol=1e-15)
    assert abs(dW0.sum() - rec["dW0_sum"]) < 1e-12 and abs(deta - rec["deta"]) < 1e-12 * max(1.0, abs(deta))
