"""The multi-rank plumbing on CPU: two gloo ranks, as torchrun launches them
(127.0.0.1), check bench.py's max-over-ranks time, summed iteration count and
per-rank problems, and the all-reduce of the sharded Lloyd loop's partial
sums, counts and objectives (exact_means_clustering_b200.reduce_partials)."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import bench
    import datagen
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        t, n = bench.over_ranks(torch, dist, torch.device("cpu"), 10.0 + 5.0 * rank, 7 + rank)
        w = bench.rank_workload(datagen.CONFIGS[2].scaled(B=1, N=64, K=4), rank)
        x = datagen.points(w)
        digest = float(datagen.widen(x, w.dtype).astype(np.float64).sum())
        # the sharded loop's all-reduce of partial sums / counts / objectives
        import exact_means_clustering_b200 as fkm
        sums = torch.full((2, 3, 4), float(rank + 1), dtype=torch.float64)
        counts = torch.full((2, 3), rank + 1, dtype=torch.int32)
        obj = torch.tensor([0.5 * (rank + 1), 1.0], dtype=torch.float64)
        fkm.reduce_partials((sums, counts, obj))
        reduced = (float(sums.sum()), int(counts.sum()), obj.tolist())
        dist.barrier()
        q.put((rank, t, n, w.seed, digest, reduced))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    out.sort()
    for rank, t, n, seed, _, reduced in out:
        assert t == pytest.approx(15.0)          # the slowest rank's time
        assert n == 7 + 8                          # every rank's iterations
        assert reduced == (24 * 3.0, 6 * 3, [1.5, 2.0])   # partials summed over ranks
    assert out[0][3] != out[1][3]                 # own seeds ...
    assert out[0][4] != out[1][4]                 # ... and so own points
