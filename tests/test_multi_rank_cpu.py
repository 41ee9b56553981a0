"""Multi-rank plumbing of the benchmark on CPU: two `gloo` ranks shard a batch, each runs the
per-unit computation on its own images only (the oracle stands in for the device here: the GPU path
is covered by the -m gpu tests), and the gathered results must equal one run over the whole batch.
Units (image, head) are independent, so sharding the batch needs no data exchange; the only
collectives are the timing barrier and the max over ranks."""
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import oracle  # noqa: E402
from vision_test_token_b200.inputs import random_unit  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_shard_batch_covers_the_batch_once():
    for gb in range(0, 20):
        for world in range(1, 9):
            seen = []
            for r in range(world):
                a, n = bench.shard_batch(gb, r, world)
                seen.extend(range(a, a + n))
            assert seen == list(range(gb))


def _rank_main(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world), RANK=str(rank),
                      LOCAL_RANK=str(rank))
    import torch.distributed as dist
    w, x = random_unit(5, 2, 4, 5, dtype="bf16", seed=11, kind="mixed", conv_heads=1, eta=0.5)
    ws, rk, _ = bench.dist_init(world, backend="gloo")
    assert (ws, rk) == (world, rank)
    a, n = bench.shard_batch(w.batch, rank, world)
    sl = slice(a, a + n)
    nl = w.lin_heads
    Zl, W1l = oracle.linear(x["Q"][sl, :nl], x["K"][sl, :nl], x["V"][sl, :nl], x["W0_lin"], w.eta, threads=1)
    Zc, W1c = oracle.dwconv(x["Q"][sl, nl:], x["K"][sl, nl:], x["V"][sl, nl:], x["W0_conv"], w.eta, w.H, w.W,
                            threads=1)
    parts = [None] * world
    dist.all_gather_object(parts, (a, n, np.concatenate([Zl, Zc], axis=1), W1l, W1c))
    bench.barrier(world)
    t = bench.max_over_ranks(0.25 + rank, world, "cpu")
    if rank == 0:
        np.savez(os.path.join(out_dir, "gathered.npz"),
                 starts=np.array([p[0] for p in parts]), counts=np.array([p[1] for p in parts]),
                 Z=np.concatenate([p[2] for p in parts]), W1l=np.concatenate([p[3] for p in parts]),
                 W1c=np.concatenate([p[4] for p in parts]), tmax=np.array([t]))
    dist.destroy_process_group()


def test_two_gloo_ranks_shard_the_batch(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    g = np.load(tmp_path / "gathered.npz")
    assert list(g["starts"]) == [0, 3] and list(g["counts"]) == [3, 2]
    assert g["tmax"][0] == pytest.approx(1.25)           # max over ranks, not rank 0's own time
    w, x = random_unit(5, 2, 4, 5, dtype="bf16", seed=11, kind="mixed", conv_heads=1, eta=0.5)
    Zl, W1l = oracle.linear(x["Q"][:, :1], x["K"][:, :1], x["V"][:, :1], x["W0_lin"], w.eta, threads=1)
    Zc, W1c = oracle.dwconv(x["Q"][:, 1:], x["K"][:, 1:], x["V"][:, 1:], x["W0_conv"], w.eta, w.H, w.W, threads=1)
    np.testing.assert_array_equal(g["Z"], np.concatenate([Zl, Zc], axis=1))
    np.testing.assert_array_equal(g["W1l"], W1l)
    np.testing.assert_array_equal(g["W1c"], W1c)
