"""Host logic of bench.py, on the CPU: input-set sizing against the L2, algorithmic bytes and FLOPs,
the config object both arms print, the oracle leg on every workload kind (tiny shapes), and the
staleness check of the DRAM-traffic table."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from vision_test_token_b200.inputs import WORKLOADS, Workload, make_inputs  # noqa: E402


def test_default_sets_exceed_twice_l2_or_flush():
    for w in WORKLOADS.values():
        n = bench.default_sets(w)
        assert 3 <= n <= bench.MAX_SETS
        per = bench.workload_bytes(w)
        assert n * per > 2 * bench.L2_BYTES or bench.needs_flush(w, n)
    assert bench.needs_flush(WORKLOADS["lin196_fp32"], bench.default_sets(WORKLOADS["lin196_fp32"]))
    assert not bench.needs_flush(WORKLOADS["mixed6084_bf16"], bench.default_sets(WORKLOADS["mixed6084_bf16"]))


def test_workload_bytes_and_flops():
    w = WORKLOADS["mixed6084_bf16"]
    assert bench.workload_bytes(w) == 149_520_384            # Q, K, V read, Z written: 4 x 8 x 6 x 6084 x 64 x 2
    assert bench.workload_bytes(WORKLOADS["bwd6084_bf16"]) == 7 * 8 * 5 * 6084 * 64 * 2
    assert bench.workload_flops(w) is None                    # HBM-bound: no FLOP roofline
    c3 = WORKLOADS["conv3x3_6084_bf16"]
    assert bench.workload_flops(c3) == 8 * 6084 * 54 * 64 * 64
    m = WORKLOADS["mlp1024_bf16"]
    assert bench.workload_flops(m) == 16 * 4 * 1024 * 7 * 2 * 64 * 256


def test_config_keys_match_between_arms():
    for w in WORKLOADS.values():
        a, b = bench.config_of(w, 1), bench.config_of(w, 1)
        assert a == b
        for k in ("workload", "lin_heads", "conv_heads", "grid", "tokens", "d", "eta", "loss"):
            assert k in a


@pytest.mark.parametrize("kind,extra", [
    ("linear", {}), ("mixed", {"conv_heads": 1}), ("mlp", {}), ("minibatch", {"mb_tokens": 4}),
    ("backward", {}), ("backward_conv", {"conv_heads": 1}), ("backward_mlp", {}), ("conv3x3", {}),
])
def test_oracle_leg_runs_every_kind(kind, extra):
    heads = 1 if kind in ("backward_conv", "conv3x3") else 2
    w = Workload("tiny", 2, heads, 3, 4, "bf16", 0.5, kind, **extra)
    x = bench.oracle_inputs(w, make_inputs(w, seed=1), 2)
    bench.oracle_units(w, x, 3, 1)                          # three images: image 0 used again
    bench.oracle_units(w, x, 1, 1, heads=(heads - 1, heads))


def test_traffic_entry_refuses_a_stale_capture(monkeypatch):
    w = WORKLOADS["mixed6084_bf16"]
    monkeypatch.setattr(bench, "TRAFFIC", {})
    e, note = bench.traffic_entry(w)
    assert e is None and "no ncu capture" in note
    monkeypatch.setattr(bench, "TRAFFIC", {w.name: {"read": 1.0, "write": 2.0, "src_sha": "0" * 16}})
    e, note = bench.traffic_entry(w)
    assert e is None and note.startswith("stale")
    monkeypatch.setattr(bench, "TRAFFIC", {w.name: {"read": 1.0, "write": 2.0,
                                                    "src_sha": bench.kernel_source_hash(w.kind)}})
    e, note = bench.traffic_entry(w)
    assert e["read"] == 1.0 and note is None


def test_kernel_source_hash_is_stable_and_per_kind():
    assert bench.kernel_source_hash() == bench.kernel_source_hash()
    assert len(bench.kernel_source_hash()) == 16
    assert set(bench.KIND_SOURCES) >= {w.kind for w in WORKLOADS.values()}
    assert bench.kernel_source_hash("mixed") != bench.kernel_source_hash("mlp")


def test_source_hash_sees_code_not_comments():
    """A capture stays valid across comment edits, and only across them."""
    assert bench.code_of(b"int a; // one\n\n// two\n  int b;  \n") == bench.code_of(b"int a;\n  int b;")
    assert bench.code_of(b"int a;\n  int b;") == b"int a;\n  int b;"
    assert bench.code_of(b"int a = 1;") != bench.code_of(b"int a = 2;")


def test_launches_per_step():
    """The kernels a step launches, as the bench line's gpu_launches counts them."""
    counts = {name: bench.launches_per_step(w) for name, w in WORKLOADS.items()}
    assert counts["mixed6084_bf16"] == 2                      # linear heads and conv head at once
    assert counts["lin196_fp32"] == 1                         # one cluster kernel for a small fp32 unit
    assert counts["lin6400_bf16"] == counts["lin196_bf16"] == 1
    assert counts["conv3x3_6084_bf16"] == 4                   # W0 images, gradient, merge, readout
    assert counts["bwd6084_bf16"] == 4                        # phase 1, merge, phase 2, sums
    assert bench.launches_per_step(Workload("big32", 1, 1, 40, 40, "fp32", 0.5, "linear")) == 2
