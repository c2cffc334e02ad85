"""Multi-process host logic of replica runs, on CPU with gloo (world size 2):
each rank draws its own replica, runs the float64 oracle on it, and the ranks
combine only their timings (max over ranks)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from gen import workloads as W
from test_trained_neural_b200.replicas import aggregate_throughput, max_over_ranks, replica


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        base = W.make(2, 8, 2, 1, 2, 32, 8, index=77)
        w = replica(base, rank)
        inp = W.generate(w)
        res = oracle.run_workload(w, inp, threads=1)
        fake_seconds = 1.0 + rank          # rank 1 is the slow one
        t = max_over_ranks(fake_seconds, world)
        ys = [torch.zeros(res["y"].size, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(ys, torch.from_numpy(res["y"].ravel().copy()))
        np.save(os.path.join(out_dir, f"rank{rank}.npy"),
                np.array([t, aggregate_throughput(w.streams * w.T, world, t)]))
        np.save(os.path.join(out_dir, f"ys{rank}.npy"), torch.stack(ys).numpy())
    finally:
        dist.destroy_process_group()


def test_two_rank_replicas_with_gloo(tmp_path):
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       start_method="spawn", join=True)
    base = W.make(2, 8, 2, 1, 2, 32, 8, index=77)
    for r in range(world):
        t, thr = np.load(tmp_path / f"rank{r}.npy")
        assert t == 2.0                                   # max over ranks
        assert thr == world * base.streams * base.T / 2.0
    ys = np.load(tmp_path / "ys0.npy")
    assert np.array_equal(ys, np.load(tmp_path / "ys1.npy"))   # both ranks saw the same gather
    for r in range(world):
        w = replica(base, r)
        ref = oracle.run_workload(w, W.generate(w), threads=1)["y"].ravel()
        assert np.array_equal(ys[r], ref)                 # each rank ran its own replica
    assert not np.array_equal(ys[0], ys[1])               # replicas differ (own seeds)


def test_replica_seeds():
    w = W.get(2)
    assert replica(w, 0) is w
    assert replica(w, 3).seed == w.seed + 3000
    assert replica(w, 3).T == w.T and replica(w, 3).dims == w.dims
