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
    buf, sums, counts, obj = fkm.partial_buffers(B, K, D, "cuda")
    edges = (0,) + tuple(cuts) + (N,)
    for a, b in zip(edges[:-1], edges[1:]):
        fkm.fkm_partial_update(xt[:, a:b].contiguous(), ids[:, a:b].contiguous(), c, sums, counts,
                               obj)
    cen = torch.empty_like(c)
    shift = torch.empty(B, dtype=torch.float64, device="cuda")
    cnt32 = torch.empty(B, K, dtype=torch.int32, device="cuda")
    fkm.fkm_finalize_sums(sums, counts, c, cen, shift, counts_out=cnt32)
    assert torch.equal(cnt32.double(), counts)
    counts = cnt32
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


@pytest.mark.parametrize("dtype,B,N,K,D,cut,chunk", [("bf16", 2, 9000, 300, 128, 5000, 2048),
                                                     ("f32", 1, 6000, 100, 96, 777, 1000)])
def test_host_shard_partials_match_device_partials(dtype, B, N, K, D, cut, chunk):
    """Shards kept in pinned host memory and streamed in chunks give the same
    ids, counts and (up to fp64 summation order) sums and objective as the
    device-resident shard step."""
    w = datagen.Workload("host-shards", B, N, D, K, dtype, K, sigma=0.5, iters=1, seed=N + D)
    x, xt, c0 = problem(w)
    c = torch.from_numpy(c0).cuda()
    ref = list(fkm.partial_buffers(B, K, D, "cuda")[1:])
    got = list(fkm.partial_buffers(B, K, D, "cuda")[1:])
    ids_ref = torch.empty(B, N, dtype=torch.int32, device="cuda")
    fkm.fkm_assign(xt, c, ids_ref)
    ids = torch.full((B, N), -1, dtype=torch.int32, device="cuda")
    for a, b in ((0, cut), (cut, N)):
        fkm.fkm_partial_update(xt[:, a:b].clone(), ids_ref[:, a:b].clone(), c, *ref)
        xh = xt[:, a:b].cpu().pin_memory()
        part_ids = torch.empty(B, b - a, dtype=torch.int32, device="cuda")
        fkm.fkm_partial_update_host(xh, c, chunk, part_ids, *got)
        ids[:, a:b] = part_ids
    assert torch.equal(ids, ids_ref)
    assert torch.equal(got[1], ref[1])
    # the segment sums add up to 16 rows in fp32 before each fp64 fold; a fold
    # of <= 16 values rounds by <= 16 * 2^-24 * 16 max|x|, so a cluster of n
    # points differs by <= n * 2^-20 * max|x| per side between two groupings
    bound = 2.0 ** -19 * got[1].double().unsqueeze(-1) * xt.abs().max().double()
    assert ((got[0] - ref[0]).abs() <= bound + 1e-12).all()
    assert torch.allclose(got[2], ref[2], rtol=1e-6)
    cen = torch.empty_like(c)
    fkm.fkm_finalize_sums(got[0], got[1], c, cen)
    check_update(x, dtype, ids.cpu().numpy(), c0, cen.cpu().numpy(),
                 got[1].cpu().numpy().astype(np.int64))


def test_sharded_loop_from_host_matches_lloyd_host():
    w = datagen.CONFIGS[2].scaled(B=2, N=8192, K=256, iters=3)
    x, xt, c0 = problem(w)
    c0t = torch.from_numpy(c0).cuda()
    xh = xt.cpu().pin_memory()
    ids, cen, cnt, inertia, n = fkm.lloyd_sharded(xh, c0t, 3, chunk_rows=3000)
    i2 = torch.empty(w.B, w.N, dtype=torch.int32, device="cuda")
    c2 = torch.empty(w.B, w.K, w.D, device="cuda")
    n2 = torch.empty(w.B, w.K, dtype=torch.int32, device="cuda")
    in2 = torch.empty(w.B, dtype=torch.float64, device="cuda")
    assert n == fkm.fkm_lloyd_host(xh, c0t, 3, 0.0, 3000, i2, c2, n2, in2) == 3
    # the fp64 atomics of runs that cross a segment-sum range may round in
    # another order, so a near tie may still flip
    assert (ids != i2).float().mean().item() <= 1e-4
    assert (cnt - n2).abs().sum().item() <= 2 * (ids != i2).sum().item()
    assert torch.allclose(cen, c2, rtol=1e-6, atol=1e-6)
    assert torch.allclose(inertia, in2, rtol=1e-6)


def test_host_shard_copy_at_once_gives_the_same_partials():
    """With FKM_HOST_COPY_AT_ONCE (the chunk buffers idle after an earlier call
    on the workspace) the first copy starts without waiting for the stream;
    the partials and ids are those of a call without the flag."""
    w = datagen.Workload("host-flags", 2, 7000, 128, 200, "bf16", 200, sigma=0.5, iters=1, seed=3)
    x, xt, c0 = problem(w)
    c = torch.from_numpy(c0).cuda()
    xh = xt.cpu().pin_memory()
    ws = fkm.workspace(fkm.fkm_host_workspace_size(w.B, w.N, w.K, w.D, xt.dtype, 2048))
    outs = []
    for at_once in (False, True, True):
        buf, sums, counts, obj = fkm.partial_buffers(w.B, w.K, w.D, "cuda")
        ids = torch.empty(w.B, w.N, dtype=torch.int32, device="cuda")
        # queued work on the stream that the flagged copy does not wait for
        torch.cuda._sleep(1_000_000)
        fkm.fkm_partial_update_host(xh, c, 2048, ids, sums, counts, obj, ws=ws,
                                    copy_at_once=at_once)
        outs.append((ids, counts.clone(), sums.clone(), obj.clone()))
    for ids, counts, sums, obj in outs[1:]:
        assert torch.equal(ids, outs[0][0]) and torch.equal(counts, outs[0][1])
        assert torch.allclose(sums, outs[0][2], rtol=1e-12, atol=1e-9)
        assert torch.allclose(obj, outs[0][3], rtol=1e-12)
