"""Parity at the workloads' full sizes, through the calls the benchmark times.

Each test runs the whole Lloyd loop of one workload at its full shape
(fkm_lloyd, or fkm_lloyd_host for the host-resident one), then checks it
against the fp64 oracle where the oracle can follow:
  - the loop equals its own last iteration replayed from the centroids one
    iteration earlier (the assignment identically, the update to rounding);
  - assign, teacher-forced: a seeded sample of points per batch against the
    centroids of the last assignment (tests/parity.py criteria);
  - update, teacher-forced: every point (counts bit-exact, centroids within
    1e-5 of the per-cluster mean |x|, empty clusters unchanged);
  - inertia: within 1e-4 of the oracle's objective of the final assignment.
The free-running trajectory at these sizes is not compared (the oracle would
need hours); the scaled runs in test_gpu_parity.py compare it.
"""
import numpy as np
import pytest
import torch

import datagen
import exact_means_clustering_b200 as fkm
import oracle
from parity import check_assign, check_update_large, problem, rel

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

HOST_CHUNK_ROWS = 1 << 23   # the benchmark's chunk of host rows


def _mirror(dtype):
    return dtype if dtype != "f32" else None


def _outputs(B, N, K, D):
    return (torch.empty(B, N, dtype=torch.int32, device="cuda"),
            torch.empty(B, K, D, dtype=torch.float32, device="cuda"),
            torch.empty(B, K, dtype=torch.int32, device="cuda"),
            torch.empty(B, dtype=torch.float64, device="cuda"))


def _sample(B, N, per_batch, seed):
    rng = np.random.default_rng(seed)
    return np.stack([np.sort(rng.choice(N, size=min(per_batch, N), replace=False))
                     for _ in range(B)])


def _check_final(x, dtype, c_prev, ids, centers, counts, inertia, sample):
    g = ids.cpu().numpy()
    cp = c_prev.cpu().numpy()
    check_assign(x, dtype, cp, g, sample=sample)
    check_update_large(x, dtype, g, cp, centers.cpu().numpy(), counts.cpu().numpy())
    J = oracle.inertia(x, g, cp.astype(np.float64), dtype=dtype, mirror=_mirror(dtype))
    gi = inertia.cpu().numpy()
    for b in range(x.shape[0]):
        assert rel(gi[b], J[b]) < 1e-4, (b, gi[b], J[b])


@pytest.mark.parametrize("wid", [2, 3, 4])
def test_full_size_device(wid):
    w = datagen.CONFIGS[wid]
    B, N, K, D = w.B, w.N, w.K, w.D
    x, xt, c0 = problem(w)
    c0t = torch.from_numpy(c0).cuda()
    ids, centers, counts, inertia = _outputs(B, N, K, D)
    n_iter = fkm.fkm_lloyd(xt, c0t, w.iters, w.tol, ids, centers, counts, inertia)
    assert 1 <= n_iter <= w.iters
    assert np.all(counts.cpu().numpy().sum(1) == N)
    # the last iteration again, from the centroids one iteration earlier
    if n_iter > 1:
        i0, c_prev, n0, _ = _outputs(B, N, K, D)
        fkm.fkm_lloyd(xt, c0t, n_iter - 1, 0.0, i0, c_prev, n0)
    else:
        c_prev = c0t
    ids1, c1, n1, in1 = _outputs(B, N, K, D)
    fkm.fkm_assign(xt, c_prev, ids1, in1)
    fkm.fkm_update(xt, ids1, c_prev, c1, n1)
    assert torch.equal(ids1, ids)
    assert torch.equal(n1, counts)
    assert torch.allclose(c1, centers, rtol=1e-6, atol=1e-7)
    # the loop sums the objective inside the update pass, fkm_assign in its own
    # pass: the same terms in another order
    assert torch.allclose(in1, inertia, rtol=1e-6)
    sample = _sample(B, N, 2048 if B > 1 else 8192, wid)
    _check_final(x, w.dtype, c_prev, ids, centers, counts, inertia, sample)


def test_full_size_host_resident():
    w = datagen.CONFIGS[5]
    B, N, K, D = w.B, w.N, w.K, w.D
    xh = torch.empty((B, N, D), dtype=torch.float32, pin_memory=True)   # 64 GiB, pinned
    for b in range(B):
        datagen.fill_points(w, b, xh[b].data_ptr())
    x = xh.numpy()
    c0 = datagen.init_centroids(x, datagen.init_indices(w), w.dtype)
    c0t = torch.from_numpy(c0).cuda()
    ids, centers, counts, inertia = _outputs(B, N, K, D)
    n_iter = fkm.fkm_lloyd_host(xh, c0t, w.iters, w.tol, HOST_CHUNK_ROWS, ids, centers, counts,
                                inertia)
    assert n_iter == w.iters
    assert np.all(counts.cpu().numpy().sum(1) == N)
    i0, c_prev, n0, _ = _outputs(B, N, K, D)
    fkm.fkm_lloyd_host(xh, c0t, n_iter - 1, 0.0, HOST_CHUNK_ROWS, i0, c_prev, n0)
    ids1, c1, n1, in1 = _outputs(B, N, K, D)
    fkm.fkm_lloyd_host(xh, c_prev, 1, 0.0, HOST_CHUNK_ROWS, ids1, c1, n1, in1)
    assert torch.equal(ids1, ids)
    assert torch.equal(n1, counts)
    assert torch.allclose(c1, centers, rtol=1e-6, atol=1e-7)
    sample = _sample(B, N, 2048, 5)
    _check_final(x, w.dtype, c_prev, ids, centers, counts, inertia, sample)
