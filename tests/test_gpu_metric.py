"""Dot-product and cosine k-means (fkm.h, fkm_metric) on the GPU against the
oracle: teacher-forced assign and update, the loop's objective, a
free-running loop, and the Euclidean metric through the same entry points."""

import numpy as np
import pytest
import torch

import datagen
import exact_means_clustering_b200 as fkm
import oracle
from parity import (check_assign_sim, check_free_running, check_update_sim, problem, rel,
                    scored)

pytestmark = pytest.mark.gpu


def check_objective(x, dtype, ids, c, gpu_obj, metric):
    """sum_i x_i . c~_{ids_i} within 1e-6 of sum_i |x_i| . |c~_{ids_i}|."""
    ref = oracle.similarity(x, ids, c.astype(np.float64), metric, dtype=dtype)
    v = np.abs(scored(c, metric))
    for b in range(x.shape[0]):
        xf = np.abs(datagen.widen(x[b], dtype).astype(np.float64))
        scale = (xf * v[b][ids[b]]).sum()
        assert abs(gpu_obj[b] - ref[b]) <= 1e-6 * scale, (b, gpu_obj[b], ref[b], scale)


CASES = [("bf16", 2, 5000, 300, 128), ("f16", 1, 3000, 1000, 64), ("f32", 1, 4000, 64, 96),
         ("bf16", 1, 6000, 2500, 128), ("bf16", 1, 1500, 40, 512)]


@pytest.mark.parametrize("metric", ["dot", "cosine"])
@pytest.mark.parametrize("dtype,B,N,K,D", CASES)
def test_assign_and_update_teacher_forced(metric, dtype, B, N, K, D):
    w = datagen.Workload("metric", B, N, D, K, dtype, K, sigma=0.5, iters=1, seed=N + K + D)
    x, xt, c0 = problem(w)
    c = torch.from_numpy(c0).cuda()
    ids = torch.empty(B, N, dtype=torch.int32, device="cuda")
    fkm.fkm_assign_metric(xt, c, ids, metric)
    check_assign_sim(x, dtype, c0, ids.cpu().numpy(), metric)
    cen = torch.empty_like(c)
    cnt = torch.empty(B, K, dtype=torch.int32, device="cuda")
    shift = torch.empty(B, dtype=torch.float64, device="cuda")
    obj = torch.empty(B, dtype=torch.float64, device="cuda")
    fkm.fkm_update_metric(xt, ids, c, cen, cnt, metric, shift, obj)
    ids_np = ids.cpu().numpy()
    check_update_sim(x, dtype, ids_np, c0, cen.cpu().numpy(), cnt.cpu().numpy(), metric)
    check_objective(x, dtype, ids_np, c0, obj.cpu().numpy(), metric)
    cen64 = cen.cpu().numpy().astype(np.float64)
    assert np.allclose(shift.cpu().numpy(), ((cen64 - c0) ** 2).sum((1, 2)), rtol=1e-6)


def test_cosine_zero_sum_and_empty_clusters_keep_previous():
    B, N, K, D = 1, 64, 4, 32
    rng = np.random.default_rng(3)
    xv = rng.standard_normal((B, N, D)).astype(np.float32)
    xv[0, 1] = -xv[0, 0]                     # cluster 3: two opposite points
    ids = np.zeros((B, N), np.int32)
    ids[0, 0:2] = 3
    ids[0, 2:] = rng.integers(0, 2, size=N - 2)   # cluster 2 stays empty
    prev = rng.standard_normal((B, K, D)).astype(np.float32)
    xt = torch.from_numpy(xv).cuda()
    c = torch.from_numpy(prev).cuda()
    cen = torch.empty_like(c)
    cnt = torch.empty(B, K, dtype=torch.int32, device="cuda")
    fkm.fkm_update_metric(xt, torch.from_numpy(ids).cuda(), c, cen, cnt, "cosine")
    got = cen.cpu().numpy()
    assert np.array_equal(got[0, 2], prev[0, 2]) and np.array_equal(got[0, 3], prev[0, 3])
    check_update_sim(xv, "f32", ids, prev, got, cnt.cpu().numpy(), "cosine")


@pytest.mark.parametrize("metric", ["dot", "cosine"])
def test_loop_objective_is_that_of_the_last_assignment(metric):
    w = datagen.CONFIGS[2].scaled(B=2, N=6000, K=200)
    x, xt, c0 = problem(w)
    c = torch.from_numpy(c0).cuda()
    ids = torch.empty(w.B, w.N, dtype=torch.int32, device="cuda")
    cen = torch.empty_like(c)
    cnt = torch.empty(w.B, w.K, dtype=torch.int32, device="cuda")
    obj = torch.empty(w.B, dtype=torch.float64, device="cuda")
    assert fkm.fkm_lloyd_metric(xt, c, 1, 0.0, ids, cen, cnt, metric, obj) == 1
    ids_np = ids.cpu().numpy()
    check_assign_sim(x, w.dtype, c0, ids_np, metric)
    check_update_sim(x, w.dtype, ids_np, c0, cen.cpu().numpy(), cnt.cpu().numpy(), metric)
    check_objective(x, w.dtype, ids_np, c0, obj.cpu().numpy(), metric)


@pytest.mark.parametrize("metric", ["dot", "cosine"])
@pytest.mark.parametrize("cfg,B,N,K", [(1, None, None, None), (2, 2, 8192, 256)])
def test_loop_free_running_against_oracle(metric, cfg, B, N, K):
    """(i) the reported objective is the oracle's objective of the GPU's own
    last assignment against the centroids it was made with; (ii) the loop,
    walked iteration by iteration against the oracle (check_free_running),
    ends within 1e-4 of its objective."""
    it = 5
    w = datagen.CONFIGS[cfg].scaled(B=B, N=N, K=K, iters=it) if B else \
        datagen.CONFIGS[cfg].scaled(iters=it)
    x, xt, c0 = problem(w)
    c = torch.from_numpy(c0).cuda()

    def run(n_it):
        ids = torch.empty(w.B, w.N, dtype=torch.int32, device="cuda")
        cen = torch.empty_like(c)
        cnt = torch.empty(w.B, w.K, dtype=torch.int32, device="cuda")
        obj = torch.empty(w.B, dtype=torch.float64, device="cuda")
        assert fkm.fkm_lloyd_metric(xt, c, n_it, 0.0, ids, cen, cnt, metric, obj) == n_it
        return ids, cen, cnt, obj

    ids, cen, cnt, obj = run(it)
    assert np.all(cnt.cpu().numpy().sum(1) == w.N)
    _, c_prev, _, _ = run(it - 1)
    ids_t = torch.empty_like(ids)
    fkm.fkm_assign_metric(xt, c_prev, ids_t, metric)
    assert torch.equal(ids_t, ids)
    g_ids, g_obj = ids.cpu().numpy(), obj.cpu().numpy()
    check_objective(x, w.dtype, g_ids, c_prev.cpu().numpy(), g_obj, metric)

    def prefix(t):
        i, ce, n, _ = run(t)
        return i.cpu().numpy(), ce.cpu().numpy(), n.cpu().numpy()

    check_free_running(x, w.dtype, c0, it, 0.0, prefix, lambda: (g_ids, g_obj, it),
                       f"{metric} workload {cfg}", metric=metric)


def test_euclid_metric_is_the_plain_loop():
    w = datagen.CONFIGS[2].scaled(B=2, N=8192, K=256, iters=3)
    x, xt, c0 = problem(w)
    c = torch.from_numpy(c0).cuda()
    outs = []
    for use_metric in (False, True):
        ids = torch.empty(w.B, w.N, dtype=torch.int32, device="cuda")
        cen = torch.empty_like(c)
        cnt = torch.empty(w.B, w.K, dtype=torch.int32, device="cuda")
        obj = torch.empty(w.B, dtype=torch.float64, device="cuda")
        if use_metric:
            n = fkm.fkm_lloyd_metric(xt, c, 3, 0.0, ids, cen, cnt, "euclid", obj)
        else:
            n = fkm.fkm_lloyd(xt, c, 3, 0.0, ids, cen, cnt, obj)
        outs.append((n, ids, cen, cnt, obj))
    (n0, i0, c_0, k0, o0), (n1, i1, c_1, k1, o1) = outs
    assert n0 == n1 == 3
    assert (i0 != i1).float().mean().item() <= 1e-4
    assert torch.allclose(c_0, c_1, rtol=1e-6, atol=1e-6)
    assert torch.allclose(o0, o1, rtol=1e-6)


@pytest.mark.parametrize("metric", ["dot", "cosine"])
def test_batch_kmeans_metric_call(metric):
    w = datagen.CONFIGS[1].scaled(iters=3)
    x, xt, c0 = problem(w)
    ids, centers, n = fkm.batch_kmeans(xt, w.K, max_iters=3, init_centroids=torch.from_numpy(c0),
                                       metric=metric)
    i2 = torch.empty(w.B, w.N, dtype=torch.int32, device="cuda")
    c2 = torch.empty(w.B, w.K, w.D, device="cuda")
    n2 = torch.empty(w.B, w.K, dtype=torch.int32, device="cuda")
    assert n == fkm.fkm_lloyd_metric(xt, torch.from_numpy(c0).cuda(), 3, 0.0, i2, c2, n2, metric)
    assert torch.equal(ids, i2) and torch.equal(centers, c2)


@pytest.mark.parametrize("metric", ["dot", "cosine"])
@pytest.mark.parametrize("cfg,B,N,K,chunk", [(1, None, None, None, 1000),
                                             (2, 2, 8192, 256, 3000)])
def test_host_streamed_loop_against_oracle(metric, cfg, B, N, K, chunk):
    """fkm_lloyd_host_metric streams pinned points in chunks (ragged last
    chunk, several chunks per batch): (i) its objective is the oracle's
    objective of its own last assignment; (ii) walked iteration by iteration
    against the oracle (check_free_running) it ends within 1e-4 of the
    oracle's objective; (iii) its ids match the device-resident loop's up to
    near-tie flips (the two add the cluster sums in different orders)."""
    it = 4
    w = datagen.CONFIGS[cfg].scaled(B=B, N=N, K=K, iters=it) if B else \
        datagen.CONFIGS[cfg].scaled(iters=it)
    x, xt, c0 = problem(w)
    xh = xt.cpu().pin_memory()
    c = torch.from_numpy(c0).cuda()

    def run(n_it):
        ids = torch.empty(w.B, w.N, dtype=torch.int32, device="cuda")
        cen = torch.empty_like(c)
        cnt = torch.empty(w.B, w.K, dtype=torch.int32, device="cuda")
        obj = torch.empty(w.B, dtype=torch.float64, device="cuda")
        assert fkm.fkm_lloyd_host_metric(xh, c, n_it, 0.0, chunk, ids, cen, cnt, metric,
                                         obj) == n_it
        return ids, cen, cnt, obj

    ids, cen, cnt, obj = run(it)
    assert np.all(cnt.cpu().numpy().sum(1) == w.N)
    _, c_prev, _, _ = run(it - 1)
    g_ids, g_obj = ids.cpu().numpy(), obj.cpu().numpy()
    check_assign_sim(x, w.dtype, c_prev.cpu().numpy(), g_ids, metric)
    check_objective(x, w.dtype, g_ids, c_prev.cpu().numpy(), g_obj, metric)

    def prefix(t):
        i, ce, n, _ = run(t)
        return i.cpu().numpy(), ce.cpu().numpy(), n.cpu().numpy()

    check_free_running(x, w.dtype, c0, it, 0.0, prefix, lambda: (g_ids, g_obj, it),
                       f"host-streamed {metric} workload {cfg}", metric=metric)
    i2 = torch.empty_like(ids)
    c2 = torch.empty_like(c)
    n2 = torch.empty_like(cnt)
    assert fkm.fkm_lloyd_metric(xt, c, it, 0.0, i2, c2, n2, metric) == it
    assert (ids != i2).float().mean().item() <= 1e-3


def test_host_streamed_euclid_metric_is_the_plain_host_loop():
    w = datagen.CONFIGS[2].scaled(B=2, N=5000, K=200, iters=3)
    x, xt, c0 = problem(w)
    xh = xt.cpu().pin_memory()
    c = torch.from_numpy(c0).cuda()
    outs = []
    for use_metric in (False, True):
        ids = torch.empty(w.B, w.N, dtype=torch.int32, device="cuda")
        cen = torch.empty_like(c)
        cnt = torch.empty(w.B, w.K, dtype=torch.int32, device="cuda")
        obj = torch.empty(w.B, dtype=torch.float64, device="cuda")
        if use_metric:
            n = fkm.fkm_lloyd_host_metric(xh, c, 3, 0.0, 1500, ids, cen, cnt, "euclid", obj)
        else:
            n = fkm.fkm_lloyd_host(xh, c, 3, 0.0, 1500, ids, cen, cnt, obj)
        outs.append((n, ids, cen, cnt, obj))
    (n0, i0, c_0, k0, o0), (n1, i1, c_1, k1, o1) = outs
    assert n0 == n1 == 3
    assert torch.equal(i0, i1) and torch.equal(k0, k1)
    assert torch.allclose(c_0, c_1, rtol=1e-6, atol=1e-6)   # fp64 atomics: order may differ
    assert torch.allclose(o0, o1, rtol=1e-9)
