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
        buf, sums, counts, obj = fkm.partial_buffers(2, 3, 4, "cpu")
        sums.fill_(float(rank + 1))
        counts.fill_(float(rank + 1))
        obj.copy_(torch.tensor([0.5 * (rank + 1), 1.0], dtype=torch.float64))
        fkm.reduce_partials((buf,))      # one collective for all three
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


# ---- the sharded loop's control over two ranks, with CPU stand-ins for the
# shard step and the finalize (the GPU calls they replace are covered by
# tests/test_gpu_sharded.py)
def _cpu_steps(x):
    def partials(c, sums, counts, obj):
        for b in range(x.shape[0]):
            d = torch.cdist(x[b], c[b].double()) ** 2
            dmin, ids = d.min(1)
            sums[b].index_add_(0, ids, x[b])
            counts[b] += torch.bincount(ids, minlength=c.shape[1]).double()
            obj[b] += dmin.sum()

    def finalize(sums, counts, c, nxt, shift, counts_out):
        n = counts.unsqueeze(-1)
        new = torch.where(n > 0, sums / n.clamp(min=1), c.double())
        nxt.copy_(new.float())
        shift.copy_(((nxt.double() - c.double()) ** 2).sum((1, 2)))
        counts_out.copy_(counts.to(torch.int32))

    return partials, finalize


def _problem(seed=5, B=2, N=600, K=7, D=4):
    g = torch.Generator().manual_seed(seed)
    means = torch.randn(B, K, D, generator=g, dtype=torch.float64) * 4
    lab = torch.randint(0, K, (B, N), generator=g)
    x = torch.gather(means, 1, lab.unsqueeze(-1).expand(B, N, D)) + \
        torch.randn(B, N, D, generator=g, dtype=torch.float64)
    return x, x[:, :K].float().contiguous()


def _sharded_rank(rank, world, port, tol, q):
    sys.path.insert(0, ROOT)
    import exact_means_clustering_b200 as fkm
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        x, c0 = _problem()
        n = x.shape[1] // world
        shard = x[:, rank * n:(rank + 1) * n]
        c, counts, obj, n_iter = fkm.sharded_loop(*_cpu_steps(shard), c0.clone(), 30, tol)
        q.put((rank, c.numpy(), counts.numpy(), obj.numpy(), n_iter))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("tol", [0.0, 1e-6])
def test_sharded_loop_two_gloo_ranks_match_one_rank(tol):
    """Two ranks holding halves of every problem reach the same centroids,
    counts and objective as one rank holding all of it, and stop after the
    same number of iterations."""
    sys.path.insert(0, ROOT)
    import exact_means_clustering_b200 as fkm
    x, c0 = _problem()
    c1, k1, o1, n1 = fkm.sharded_loop(*_cpu_steps(x), c0.clone(), 30, tol)
    if tol > 0:
        assert n1 < 30                       # the stop test fired
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_sharded_rank, args=(r, world, port, tol, q))
             for r in range(world)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for _, c, k, o, n in out:
        assert n == n1
        assert np.array_equal(k, k1.numpy())
        assert np.allclose(c, c1.numpy(), rtol=1e-6, atol=1e-6)
        assert np.allclose(o, o1.numpy(), rtol=1e-9)
    assert np.array_equal(out[0][1], out[1][1])   # every rank forms the same centroids


# ---- the class API's sharded fit: shard layout and label gathering over two
# ranks (the GPU steps replaced by the CPU stand-ins above)
def _class_rank(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import exact_means_clustering_b200 as fkm
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        x, c0 = _problem(N=601)            # an odd N: the shards differ by one row
        N = x.shape[1]
        r0, r1 = fkm.shard_rows(N, rank, world)
        c, counts, obj, n_iter = fkm.sharded_loop(*_cpu_steps(x[:, r0:r1]), c0.clone(), 30)
        # the labels of the final centroids, per shard, gathered in row order
        ids = torch.cdist(x[:, r0:r1], c.double()).argmin(-1).to(torch.int32)
        full = fkm.gather_shard_ids(ids, N)
        q.put((rank, full.numpy(), c.numpy(), counts.numpy()))
    finally:
        dist.destroy_process_group()


def test_class_sharding_two_gloo_ranks():
    """shard_rows covers every row once, the two ranks reach the one-rank
    centroids and counts, and gather_shard_ids gives every rank the labels
    of all points in row order."""
    sys.path.insert(0, ROOT)
    import exact_means_clustering_b200 as fkm
    N, world = 601, 2
    spans = [fkm.shard_rows(N, r, world) for r in range(world)]
    assert spans == [(0, 301), (301, 601)]
    assert [fkm.shard_rows(10, r, 4) for r in range(4)] == [(0, 3), (3, 6), (6, 8), (8, 10)]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_class_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    x, c0 = _problem(N=N)
    c1, k1, _, _ = fkm.sharded_loop(*_cpu_steps(x), c0.clone(), 30)
    want = torch.cdist(x, c1.double()).argmin(-1).to(torch.int32).numpy()
    for rank, full, c, counts in out:
        assert np.allclose(c, c1.numpy(), rtol=1e-6, atol=1e-6)
        assert np.array_equal(counts, k1.numpy())
        assert np.array_equal(full, want)
