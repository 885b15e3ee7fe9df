"""Data-parallel Lloyd over shards of the points (README "Multi-GPU Support")
on one GPU: the per-shard partial update summed over shards must equal the
update of the whole problem, and the sharded loop on a single rank must
reproduce fkm_lloyd.  (The all-reduce between ranks is covered on CPU by
tests/test_multirank.py.)"""
import numpy as np
import pytest
import torch

import datagen
import exact_means_clustering_b200 as fkm
from parity import check_update, problem, rel

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype,B,N,K,D,cuts", [("bf16", 2, 9000, 300, 128, (3000, 7001)),
                                                ("f32", 1, 8000, 2500, 64, (4096,)),
                                                ("f16", 3, 5000, 60, 512, (1, 2500))])
def test_shard_partials_add_up_to_the_whole_update(dtype, B, N, K, D, cuts):
    w = datagen.Workload("shards", B, N, D, K, dtype, K, sigma=0.5, iters=1, seed=N + K)
    x, xt, c0 = problem(w)
    c = torch.from_numpy(c0).cuda()
    ids = torch.empty(B, N, dtype=torch.int32, device="cuda")
    fkm.fkm_assign(xt, c, ids)
    sums = torch.zeros(B, K, D, dtype=torch.float64, device="cuda")
    counts = torch.zeros(B, K, dtype=torch.int32, device="cuda")
    obj = torch.zeros(B, dtype=torch.float64, device="cuda")
    edges = (0,) + tuple(cuts) + (N,)
    for a, b in zip(edges[:-1], edges[1:]):
        fkm.fkm_partial_update(xt[:, a:b].contiguous(), ids[:, a:b].contiguous(), c, sums, counts,
                               obj)
    cen = torch.empty_like(c)
    shift = torch.empty(B, dtype=torch.float64, device="cuda")
    fkm.fkm_finalize_sums(sums, counts, c, cen, shift)
    check_update(x, dtype, ids.cpu().numpy(), c0, cen.cpu().numpy(), counts.cpu().numpy())
    whole = torch.empty_like(c)
    n_whole = torch.empty(B, K, dtype=torch.int32, device="cuda")
    sh_whole = torch.empty(B, dtype=torch.float64, device="cuda")
    in_whole = torch.empty(B, dtype=torch.float64, device="cuda")
    fkm.fkm_update(xt, ids, c, whole, n_whole, sh_whole, in_whole)
    assert torch.equal(counts, n_whole)
    assert torch.allclose(cen, whole, rtol=1e-6, atol=1e-7)
    assert torch.allclose(shift, sh_whole, rtol=1e-6)
    assert torch.allclose(obj, in_whole, rtol=1e-6)


def test_sharded_loop_on_one_rank_matches_lloyd():
    w = datagen.CONFIGS[2].scaled(B=2, N=8192, K=256, iters=4)
    x, xt, c0 = problem(w)
    c0t = torch.from_numpy(c0).cuda()
    ids, cen, cnt, inertia, n = fkm.lloyd_sharded(xt, c0t, 4)
    i2 = torch.empty(w.B, w.N, dtype=torch.int32, device="cuda")
    c2 = torch.empty(w.B, w.K, w.D, device="cuda")
    n2 = torch.empty(w.B, w.K, dtype=torch.int32, device="cuda")
    in2 = torch.empty(w.B, dtype=torch.float64, device="cuda")
    assert n == fkm.fkm_lloyd(xt, c0t, 4, 0.0, i2, c2, n2, in2)
    assert (ids != i2).float().mean().item() <= 1e-4
    assert torch.allclose(cen, c2, rtol=1e-5, atol=1e-5)
    for b in range(w.B):
        assert rel(inertia[b].item(), in2[b].item()) < 1e-5


def test_sharded_loop_tol_stops_like_lloyd():
    w = datagen.CONFIGS[1].scaled(iters=40, tol=1e-2)
    x, xt, c0 = problem(w)
    c0t = torch.from_numpy(c0).cuda()
    _, _, _, _, n = fkm.lloyd_sharded(xt, c0t, 40, 1e-2)
    i2 = torch.empty(w.B, w.N, dtype=torch.int32, device="cuda")
    c2 = torch.empty(w.B, w.K, w.D, device="cuda")
    n2 = torch.empty(w.B, w.K, dtype=torch.int32, device="cuda")
    assert n == fkm.fkm_lloyd(xt, c0t, 40, 1e-2, i2, c2, n2)
