"""The N > 1 host path on CPU with gloo, world size 2: batch rows are sharded across
ranks with no collective on the data path, each rank computes its own rows, and the
timing reduction takes the max over ranks. Rows are independent, so the per-rank
results, put side by side, equal the whole batch."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
from gated_linear_rnn_conv1d_b200 import inputs, replicas


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    r = replicas.from_env()
    replicas.init(r, "gloo", timeout_s=60)
    w = inputs.make_forward(5, 40, 16, torch.float32, seed=9)
    rows = replicas.shard(5, r)
    p = w.params
    y, h, _ = oracle.rglru_forward(w.x[rows.start:rows.stop], p.conv_w, p.conv_b, p.W_a, p.b_a, p.W_x, p.b_x,
                                   p.Lambda)
    np.save(os.path.join(out_dir, f"y{rank}.npy"), y)
    replicas.barrier(r)
    m = replicas.max_over_ranks(r, float(rank + 1) * 1.5)
    np.save(os.path.join(out_dir, f"m{rank}.npy"), np.array([m]))
    replicas.shutdown(r)


def test_shard_covers_every_row_once():
    for n in (1, 2, 5, 8, 256):
        for world in (1, 2, 3, 8):
            got = []
            for k in range(world):
                got += list(replicas.shard(n, replicas.Rank(k, world, k)))
            assert got == list(range(n))


def test_two_gloo_ranks_equal_whole_batch(tmp_path):
    world = 2
    ctx = mp.get_context("spawn")
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(k, world, port, str(tmp_path))) for k in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    w = inputs.make_forward(5, 40, 16, torch.float32, seed=9)
    p = w.params
    y, _, _ = oracle.rglru_forward(w.x, p.conv_w, p.conv_b, p.W_a, p.b_a, p.W_x, p.b_x, p.Lambda)
    parts = np.concatenate([np.load(tmp_path / f"y{k}.npy") for k in range(world)], axis=0)
    np.testing.assert_array_equal(parts, y)
    for k in range(world):
        assert float(np.load(tmp_path / f"m{k}.npy")[0]) == 3.0
