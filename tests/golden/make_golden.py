"""Writes tests/golden/oracle_regression.json from the fp64 oracle only.

It is a regression fixture: it records what the oracle computed on a tiny seeded case so that an
unintended change to the oracle's arithmetic shows up.  Rerun only when the oracle is changed on
purpose, and name the passage that justifies the change in the commit message.
"""
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402
from vision_test_token_b200.inputs import random_unit  # noqa: E402


def main():
    out = {"_about": __doc__.strip().splitlines()[0]}
    w, x = random_unit(1, 1, 3, 4, d=8, dtype="fp32", seed=7)
    Z, W1 = oracle.linear(x["Q"], x["K"], x["V"], x["W0_lin"][:, :8, :8], 0.75)
    out["linear"] = {"shape": [1, 1, 12, 8], "seed": 7, "eta": 0.75,
                     "Z_row0": Z[0, 0, 0].tolist(), "W1_row0": W1[0, 0, 0].tolist(),
                     "Z_sum": float(Z.sum()), "W1_sum": float(W1.sum())}
    w, x = random_unit(1, 1, 3, 4, d=8, dtype="fp32", seed=8, kind="mixed", conv_heads=1)
    Z, W1 = oracle.dwconv(x["Q"], x["K"], x["V"], x["W0_conv"], 0.5, 3, 4)
    out["dwconv"] = {"shape": [1, 1, 12, 8], "seed": 8, "eta": 0.5,
                     "Z_row0": Z[0, 0, 0].tolist(), "W1_ch0": W1[0, 0, 0].ravel().tolist(),
                     "Z_sum": float(Z.sum()), "W1_sum": float(W1.sum())}
    w, x = random_unit(1, 1, 3, 4, d=8, dtype="fp32", seed=9, kind="mlp")
    Z, Wa1, Wb1 = oracle.mlp(x["Q"], x["K"], x["V"], x["Wa"], x["Wb"], 0.5)
    out["mlp"] = {"shape": [1, 1, 12, 8], "seed": 9, "eta": 0.5, "hidden": 32,
                  "Z_row0": Z[0, 0, 0].tolist(), "Z_sum": float(Z.sum()),
                  "Wa1_sum": float(Wa1.sum()), "Wb1_sum": float(Wb1.sum())}
    w, x = random_unit(1, 1, 3, 4, d=8, dtype="fp32", seed=10)
    Z, W1 = oracle.linear_dot(x["Q"], x["K"], x["V"], x["W0_lin"], 1.0)
    out["linear_dot"] = {"shape": [1, 1, 12, 8], "seed": 10, "eta": 1.0,
                         "Z_row0": Z[0, 0, 0].tolist(), "Z_sum": float(Z.sum()), "W1_sum": float(W1.sum())}
    w, x = random_unit(1, 1, 3, 4, d=8, dtype="fp32", seed=11, kind="mixed", conv_heads=1)
    Z, W1 = oracle.dwconv_dot(x["Q"], x["K"], x["V"], x["W0_conv"], 1.0, 3, 4)
    out["dwconv_dot"] = {"shape": [1, 1, 12, 8], "seed": 11, "eta": 1.0,
                         "Z_row0": Z[0, 0, 0].tolist(), "Z_sum": float(Z.sum()), "W1_sum": float(W1.sum())}
    w, x = random_unit(1, 1, 3, 4, d=8, dtype="fp32", seed=12)
    for mode in ("prefix", "epoch"):
        Z, W1 = oracle.linear_minibatch(x["Q"], x["K"], x["V"], x["W0_lin"], 0.25, 5, mode)
        out["linear_minibatch_" + mode] = {"shape": [1, 1, 12, 8], "seed": 12, "eta": 0.25, "b": 5,
                                           "Z_row0": Z[0, 0, 0].tolist(), "Z_sum": float(Z.sum()),
                                           "W1_sum": float(W1.sum())}
    w, x = random_unit(2, 1, 3, 4, d=8, dtype="fp32", seed=13, kind="backward")
    dQ, dK, dV, dW0, deta = oracle.linear_backward(x["Q"], x["K"], x["V"], x["W0_lin"], 0.5, x["dZ"])
    out["linear_backward"] = {"shape": [2, 1, 12, 8], "seed": 13, "eta": 0.5,
                              "dQ_row0": dQ[0, 0, 0].tolist(), "dK_row0": dK[0, 0, 0].tolist(),
                              "dV_row0": dV[0, 0, 0].tolist(), "dW0_sum": float(dW0.sum()), "deta": deta}
    with open(os.path.join(HERE, "oracle_regression.json"), "w") as f:
        json.dump(out, f, indent=1)


if __name__ == "__main__":
    main()
