"""GPU parity: the CUDA path through the C ABI against the fp64 oracle.

Small and medium cases span several point tiles (128) and centroid tiles (256)
with ragged tails; the full-size workloads are checked on sampled points
(assign) and in full (update, objective) in the launch configuration the
benchmark times.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import datagen
import oracle
from parity import check_assign, check_free_running, check_update, problem, rel, to_torch

pytestmark = pytest.mark.gpu

fkm = pytest.importorskip("exact_means_clustering_b200")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.init()


def _mirror(dtype):
    return dtype if dtype != "f32" else None


def _empty(B, N, K, D):
    return (torch.empty(B, N, dtype=torch.int32, device="cuda"),
            torch.empty(B, K, D, dtype=torch.float32, device="cuda"),
            torch.empty(B, K, dtype=torch.int32, device="cuda"))


# ------------------------------------------------------------------ argsort
def test_argsort_pages_example(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "argsort_example.json")))
    keys = torch.tensor(g["keys"], dtype=torch.int32, device="cuda")
    idx = torch.empty_like(keys)
    sk = torch.empty_like(keys)
    fkm.fkm_argsort(keys, 4, idx, sk)
    assert idx.tolist() == g["sorted_idx"]
    assert sk.tolist() == g["sorted_keys"]


# n_keys <= 2048 takes the one-pass counting sort, larger the LSD radix sort
@pytest.mark.parametrize("n,n_keys", [(1, 1), (4096, 7), (3 * 4096 + 77, 300),
                                      (2 * 4096 + 5, 2048), (2 * 4096 + 5, 2049),
                                      (100003, 40000), (70001, 70000), (50000, 1)])
def test_argsort_matches_oracle(n, n_keys):
    rng = np.random.default_rng(n + n_keys)
    keys = rng.integers(0, n_keys, size=n).astype(np.int32)
    if n > 1000:  # a hot key, as with skewed clusters
        keys[rng.random(n) < 0.3] = n_keys // 2
    t = torch.from_numpy(keys).cuda()
    idx = torch.empty_like(t)
    fkm.fkm_argsort(t, n_keys, idx)
    assert np.array_equal(idx.cpu().numpy(), oracle.argsort_stable(keys, n_keys))


def test_argsort_rejects_bad_keys():
    t = torch.tensor([0, 5, 1], dtype=torch.int32, device="cuda")
    idx = torch.empty_like(t)
    ws = fkm.workspace(fkm.fkm_argsort_workspace_size(3, 3))
    fkm.fkm_argsort(t, 3, idx, ws=ws)
    with pytest.raises(fkm.FkmError) as e:
        fkm.fkm_sync_status(ws)
    assert e.value.code == 7


@pytest.mark.parametrize("n,n_keys", [(3 * 4096 + 77, 300), (2 * 4096 + 5, 2048),
                                      (2 * 4096 + 5, 2049), (20011, 5000)])
def test_argsort_rejected_keys_sort_last_in_index_order(n, n_keys):
    """Keys outside [0, n_keys), spread over several sort tiles, go after
    every valid key, themselves in index order (both the counting sort and
    the radix sort), and raise FKM_ERR_BAD_ID."""
    rng = np.random.default_rng(7 * n + n_keys)
    keys = rng.integers(0, n_keys, size=n).astype(np.int32)
    bad = rng.random(n) < 0.01
    keys[bad] = np.where(rng.random(bad.sum()) < 0.5, -3, n_keys + 11).astype(np.int32)
    t = torch.from_numpy(keys).cuda()
    idx = torch.empty_like(t)
    ws = fkm.workspace(fkm.fkm_argsort_workspace_size(n, n_keys))
    fkm.fkm_argsort(t, n_keys, idx, ws=ws)
    with pytest.raises(fkm.FkmError) as e:
        fkm.fkm_sync_status(ws)
    assert e.value.code == 7
    mapped = np.where(bad, n_keys, keys).astype(np.int32)
    assert np.array_equal(idx.cpu().numpy(), oracle.argsort_stable(mapped, n_keys + 1))


# ------------------------------------------------------------------ assign
def _grid(rng, B, N, K, D, dup=True):
    """Integer centroids and points: every product and sum is exact in fp32,
    so the GPU ids must equal the oracle's bit for bit, ties included.  The
    centroid set is symmetric (v, -v, and 0 when K is odd), so the mean
    centroid is exactly zero and the centred operands are the centroids."""
    h = K // 2
    half = rng.integers(-8, 9, size=(B, h, D)).astype(np.float32) * 4
    if dup and h > 3:
        half[:, h - 1] = half[:, 1]    # exact duplicates: the lower index must win
    parts = [half, -half] + ([np.zeros((B, 1, D), np.float32)] if K % 2 else [])
    c = np.concatenate(parts, axis=1)
    owner = rng.integers(0, K, size=(B, N))
    x = np.take_along_axis(c, owner[..., None], 1) + rng.integers(-3, 4, size=(B, N, D))
    return x.astype(np.float32), c


@pytest.mark.parametrize("dtype", ["bf16", "f16", "f32"])
@pytest.mark.parametrize("B,N,K,D", [(2, 1000, 300, 64), (1, 77, 5, 128), (3, 300, 513, 32)])
def test_assign_integer_grid_bit_exact(dtype, B, N, K, D):
    if dtype == "f32" and D % 4:
        pytest.skip("shape")
    rng = np.random.default_rng(B * N + K + D)
    xf, c = _grid(rng, B, N, K, D)
    xs = {"f32": xf, "f16": xf.astype(np.float16),
          "bf16": (xf.view(np.uint32) >> 16).astype(np.uint16)}[dtype]
    x = to_torch(xs, dtype)
    ids = torch.empty(B, N, dtype=torch.int32, device="cuda")
    inertia = torch.empty(B, dtype=torch.float64, device="cuda")
    fkm.fkm_assign(x, torch.from_numpy(c).cuda(), ids, inertia)
    ref_ids, d1, _, J = oracle.assign(xs, c.astype(np.float64), dtype=dtype, mirror=None)
    assert np.array_equal(ids.cpu().numpy(), ref_ids)
    assert np.allclose(inertia.cpu().numpy(), J, rtol=1e-6)


@pytest.mark.parametrize("wid,scale", [(1, {}), (2, dict(B=3, N=5000, K=700)),
                                       (3, dict(B=2, N=7560, K=1000)),
                                       (4, dict(N=20000, K=600)),
                                       (5, dict(N=30000, K=1100))])
def test_assign_teacher_forced(wid, scale):
    w = datagen.CONFIGS[wid].scaled(**scale, host_resident=False)
    x, xt, c0 = problem(w)
    # centroids part-way through a run: the oracle's after 2 iterations
    r = oracle.lloyd(x, c0, 2, dtype=w.dtype, mirror=w.dtype if w.dtype != "f32" else None)
    c = r["centers"].astype(np.float32)
    ids = torch.empty(w.B, w.N, dtype=torch.int32, device="cuda")
    inertia = torch.empty(w.B, dtype=torch.float64, device="cuda")
    fkm.fkm_assign(xt, torch.from_numpy(c).cuda(), ids, inertia)
    g = ids.cpu().numpy()
    check_assign(x, w.dtype, c, g)
    mir = w.dtype if w.dtype != "f32" else None
    J = oracle.inertia(x, g, c.astype(np.float64), dtype=w.dtype, mirror=mir)
    for b in range(w.B):
        assert rel(inertia[b].item(), J[b]) < 1e-4


# ------------------------------------------------------------------ update
# K <= 2048 takes the one-pass counting sort, larger K the LSD radix sort
@pytest.mark.parametrize("dtype,B,N,K,D", [("bf16", 2, 9000, 300, 128), ("f16", 3, 4097, 50, 64),
                                           ("f32", 1, 20000, 40, 64), ("f32", 2, 3000, 100, 128),
                                           ("bf16", 1, 70000, 9, 256), ("bf16", 2, 1, 3, 8),
                                           ("bf16", 2, 30000, 3000, 64), ("f16", 1, 9000, 2049, 32),
                                           # rows of 12, 25 and 10 16-byte vectors: lanes whose
                                           # second vector lies past the row
                                           ("bf16", 2, 5000, 200, 96), ("bf16", 1, 6000, 100, 200),
                                           ("f32", 1, 4000, 64, 40)])
def test_update_teacher_forced(dtype, B, N, K, D):
    rng = np.random.default_rng(N + K)
    w = datagen.Workload("t", B, N, D, K, dtype, 0, sigma=2.0, seed=N)
    x = datagen.points(w)
    xt = to_torch(x, dtype)
    # skewed ids: one hot cluster spanning many 512-row ranges, a few empty clusters
    p = np.r_[0.5, rng.random(K - 1)]
    if K > 3:
        p[-3:] = 0
    ids = np.stack([rng.choice(K, size=N, p=p / p.sum()) for _ in range(B)]).astype(np.int32)
    prev = rng.standard_normal((B, K, D)).astype(np.float32)
    c = torch.empty(B, K, D, dtype=torch.float32, device="cuda")
    n = torch.empty(B, K, dtype=torch.int32, device="cuda")
    shift = torch.empty(B, dtype=torch.float64, device="cuda")
    inertia = torch.empty(B, dtype=torch.float64, device="cuda")
    fkm.fkm_update(xt, torch.from_numpy(ids).cuda(), torch.from_numpy(prev).cuda(), c, n, shift,
                   inertia)
    check_update(x, dtype, ids, prev, c.cpu().numpy(), n.cpu().numpy())
    sh_ref = ((c.cpu().numpy().astype(np.float64) - prev) ** 2).sum((1, 2))
    assert np.allclose(shift.cpu().numpy(), sh_ref, rtol=1e-9)
    J = oracle.inertia(x, ids, prev.astype(np.float64), dtype=dtype, mirror=_mirror(dtype))
    assert np.allclose(inertia.cpu().numpy(), J, rtol=1e-6)


def test_update_rejects_bad_ids():
    x = torch.zeros(1, 10, 8, dtype=torch.bfloat16, device="cuda")
    ids = torch.tensor([[0, 1, 2, 3, 9, 0, 1, 2, 3, -1]], dtype=torch.int32, device="cuda")
    prev = torch.zeros(1, 4, 8, device="cuda")
    c, n = torch.empty_like(prev), torch.empty(1, 4, dtype=torch.int32, device="cuda")
    ws = fkm.workspace(fkm.fkm_workspace_size(1, 10, 4, 8, torch.bfloat16))
    fkm.fkm_update(x, ids, prev, c, n, ws=ws)
    with pytest.raises(fkm.FkmError) as e:
        fkm.fkm_sync_status(ws)
    assert e.value.code == 7
    assert n.sum().item() == 8   # the two bad rows are left out


# ------------------------------------------------------------------ lloyd

def _walk_lloyd(label, x, xt, c0, dtype, iters, tol, host_chunk=None):
    """check_free_running on fkm_lloyd (or, with host_chunk, on fkm_lloyd_host
    streaming pinned host memory in chunks of host_chunk points)."""
    B, N, D = x.shape
    K = c0.shape[1]
    c0t = torch.from_numpy(c0).cuda()
    xh = xt.cpu().pin_memory() if host_chunk else None

    def run(t, tl):
        ids, centers, counts = _empty(B, N, K, D)
        inertia = torch.empty(B, dtype=torch.float64, device="cuda")
        if host_chunk:
            n = fkm.fkm_lloyd_host(xh, c0t, t, tl, host_chunk, ids, centers, counts, inertia)
        else:
            n = fkm.fkm_lloyd(xt, c0t, t, tl, ids, centers, counts, inertia)
        return ids.cpu().numpy(), centers.cpu().numpy(), counts.cpu().numpy(), \
            inertia.cpu().numpy(), n

    def prefix(t):
        ids, centers, counts, _, n = run(t, 0.0)
        assert n == t
        assert np.all(counts.sum(1) == N)
        return ids, centers, counts

    def final():
        ids, _, _, inertia, n = run(iters, tol)
        return ids, inertia, n

    return check_free_running(x, dtype, c0, iters, tol, prefix, final, label)


@pytest.mark.parametrize("wid,scale", [(1, {}), (2, dict(B=4, N=8192, K=128)),
                                       (3, dict(B=4, N=7560, K=100)),
                                       (4, dict(N=60000, K=300)),
                                       (4, dict(N=50000, K=2500, n_comp=2500)),   # radix sort
                                       (5, dict(N=40000, K=200, iters=3))])
def test_lloyd_free_running(wid, scale):
    """(i) the reported objective is the oracle's objective of the GPU's own
    final assignment against the centroids it was made with; (ii) the free-
    running loop, walked iteration by iteration against the oracle, ends
    within 1e-4 of its objective (check_free_running: a trajectory that parts
    at a near tie is proven to, and re-seeds the oracle)."""
    w = datagen.CONFIGS[wid].scaled(**scale, host_resident=False)
    x, xt, c0 = problem(w)
    mir = _mirror(w.dtype)
    ids, centers, counts = _empty(w.B, w.N, w.K, w.D)
    inertia = torch.empty(w.B, dtype=torch.float64, device="cuda")
    n_iter = fkm.fkm_lloyd(xt, torch.from_numpy(c0).cuda(), w.iters, w.tol, ids, centers, counts,
                           inertia)
    g_in = inertia.cpu().numpy()
    g_ids = ids.cpu().numpy()
    # (i): the centroids of the last assignment come from a run one iteration shorter
    c_prev = torch.from_numpy(c0).cuda()
    if n_iter > 1:
        _, c_prev, _ = _empty(w.B, w.N, w.K, w.D)
        i1, _, n1 = _empty(w.B, w.N, w.K, w.D)
        fkm.fkm_lloyd(xt, torch.from_numpy(c0).cuda(), n_iter - 1, 0.0, i1, c_prev, n1)
    ids_t = torch.empty_like(ids)
    in_t = torch.empty_like(inertia)
    fkm.fkm_assign(xt, c_prev, ids_t, in_t)
    assert torch.equal(ids_t, ids)
    J = oracle.inertia(x, g_ids, c_prev.cpu().numpy().astype(np.float64), dtype=w.dtype,
                       mirror=mir)
    for b in range(w.B):
        assert rel(g_in[b], J[b]) < 1e-4, (b, g_in[b], J[b])
    # (ii)
    _walk_lloyd(f"workload {wid} {scale}", x, xt, c0, w.dtype, w.iters, w.tol)


def test_lloyd_steps_match_single_calls():
    """fkm_lloyd's loop (graph replay) equals stepping fkm_assign + fkm_update,
    with teacher-forced oracle checks at every step."""
    w = datagen.CONFIGS[2].scaled(B=2, N=6000, K=300, iters=4)
    x, xt, c0 = problem(w)
    c = torch.from_numpy(c0).cuda()
    ids = torch.empty(w.B, w.N, dtype=torch.int32, device="cuda")
    for t in range(w.iters):
        inertia = torch.empty(w.B, dtype=torch.float64, device="cuda")
        fkm.fkm_assign(xt, c, ids, inertia)
        g = ids.cpu().numpy()
        check_assign(x, w.dtype, c.cpu().numpy(), g)
        nxt = torch.empty_like(c)
        n = torch.empty(w.B, w.K, dtype=torch.int32, device="cuda")
        fkm.fkm_update(xt, ids, c, nxt, n)
        check_update(x, w.dtype, g, c.cpu().numpy(), nxt.cpu().numpy(), n.cpu().numpy())
        c = nxt
    ids2, centers2, counts2 = _empty(w.B, w.N, w.K, w.D)
    inertia2 = torch.empty(w.B, dtype=torch.float64, device="cuda")
    fkm.fkm_lloyd(xt, torch.from_numpy(c0).cuda(), w.iters, 0.0, ids2, centers2, counts2, inertia2)
    assert torch.equal(ids2, ids)
    assert torch.equal(counts2, n)
    assert torch.allclose(centers2, c, rtol=1e-6, atol=1e-6)
    assert torch.allclose(inertia2, inertia, rtol=1e-6)
    # and the update's own objective equals the assign's for the same ids
    obj = torch.empty(w.B, dtype=torch.float64, device="cuda")
    c_prev = torch.from_numpy(c0).cuda()
    ids_a = torch.empty_like(ids)
    inertia_a = torch.empty_like(obj)
    fkm.fkm_assign(xt, c_prev, ids_a, inertia_a)
    fkm.fkm_update(xt, ids_a, c_prev, torch.empty_like(c_prev), torch.empty_like(n), None, obj)
    assert torch.allclose(obj, inertia_a, rtol=1e-6)


def test_lloyd_tol_stops_and_repeats():
    w = datagen.CONFIGS[1].scaled(iters=50, tol=1e-3)
    x, xt, c0 = problem(w)
    ids, centers, counts = _empty(w.B, w.N, w.K, w.D)
    n1 = fkm.fkm_lloyd(xt, torch.from_numpy(c0).cuda(), 50, 1e-3, ids, centers, counts)
    ref = oracle.lloyd(x, c0, 50, 1e-3, dtype="f32")
    assert n1 == ref["n_iter"] < 50
    # graph path (tol = 0) called twice with the same buffers gives the same result
    a = _empty(w.B, w.N, w.K, w.D)
    b = _empty(w.B, w.N, w.K, w.D)
    ws = fkm.workspace(fkm.fkm_workspace_size(w.B, w.N, w.K, w.D, torch.float32))
    c0t = torch.from_numpy(c0).cuda()
    fkm.fkm_lloyd(xt, c0t, 5, 0.0, *a, ws=ws)
    ca = a[1].clone()
    fkm.fkm_lloyd(xt, c0t, 5, 0.0, *a, ws=ws)
    assert torch.equal(ca, a[1])
    fkm.fkm_lloyd(xt, c0t, 5, 0.0, *b)
    assert torch.equal(a[0], b[0])


def test_lloyd_init_may_alias_centers():
    w = datagen.CONFIGS[1].scaled(iters=3)
    x, xt, c0 = problem(w)
    ids, centers, counts = _empty(w.B, w.N, w.K, w.D)
    ref = _empty(w.B, w.N, w.K, w.D)
    fkm.fkm_lloyd(xt, torch.from_numpy(c0).cuda(), 3, 0.0, *ref)
    centers.copy_(torch.from_numpy(c0))
    fkm.fkm_lloyd(xt, centers, 3, 0.0, ids, centers, counts)
    assert torch.equal(centers, ref[1]) and torch.equal(ids, ref[0])


# ------------------------------------------------------------------ edge cases
@pytest.mark.parametrize("dtype,B,N,K,D", [
    ("bf16", 1, 1, 1, 8), ("bf16", 2, 5, 1, 8), ("f16", 1, 100, 300, 16),   # K > N: empties
    ("f32", 1, 129, 257, 4), ("bf16", 3, 128, 256, 256), ("f32", 2, 255, 2, 128),
    ("bf16", 8, 4096, 2048, 64), ("f16", 5, 3000, 700, 32),   # batches of one sort tile
])
def test_edge_shapes_free_running(dtype, B, N, K, D):
    w = datagen.Workload("edge", B, N, D, K, dtype, 0, sigma=1.0, iters=3, seed=B * N + K)
    x, xt, c0 = problem(w) if K <= N else (None, None, None)
    if K > N:
        x = datagen.points(w)
        xt = to_torch(x, dtype)
        c0 = np.random.default_rng(0).standard_normal((B, K, D)).astype(np.float32)
    _walk_lloyd(f"edge {dtype} B={B} N={N} K={K} D={D}", x, xt, c0, dtype, 3, 0.0)
    if K == 1:
        ids, centers, counts = _empty(B, N, K, D)
        fkm.fkm_lloyd(xt, torch.from_numpy(c0).cuda(), 3, 0.0, ids, centers, counts)
        assert ids.eq(0).all()


def test_offset_channels_stress():
    """A few channels offset by 64 (the massive-activation shape the README's
    "Centre your data" section warns about): the exact argmin keeps the
    objective with the oracle's, centred or not."""
    w = datagen.CONFIGS[2].scaled(B=2, N=8192, K=256, iters=10)
    x = datagen.widen(datagen.points(w), "bf16")
    x[..., :3] += 64.0
    # the offset points, rounded to bf16 (RNE) by torch: these are the inputs
    xs = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    c0 = datagen.init_centroids(xs, datagen.init_indices(w), "bf16")
    _walk_lloyd("offset channels", xs, to_torch(xs, "bf16"), c0, "bf16", 10, 0.0)


# ------------------------------------------------------------------ out-of-core
@pytest.mark.parametrize("dtype,B,N,K,D,chunk", [("f32", 1, 20000, 100, 64, 4096),
                                                 ("bf16", 2, 9000, 300, 128, 2000),
                                                 ("f16", 1, 5000, 40, 32, 100000)])
def test_lloyd_host_streams_pinned_chunks(dtype, B, N, K, D, chunk):
    w = datagen.Workload("ooc", B, N, D, K, dtype, K, sigma=0.5, iters=4, seed=N + K)
    x, xt, c0 = problem(w)
    xh = xt.cpu().pin_memory()
    _walk_lloyd(f"host-streamed {dtype}", x, xt, c0, dtype, 4, 0.0, host_chunk=chunk)
    ids, centers, counts = _empty(B, N, K, D)
    n_iter = fkm.fkm_lloyd_host(xh, torch.from_numpy(c0).cuda(), 4, 0.0, chunk, ids, centers,
                                counts)
    assert n_iter == 4
    # the same run in device memory: same counts and ids up to near-tie flips
    i2, c2, n2 = _empty(B, N, K, D)
    fkm.fkm_lloyd(xt, torch.from_numpy(c0).cuda(), 4, 0.0, i2, c2, n2)
    assert (ids != i2).float().mean().item() <= 1e-3
    assert torch.allclose(centers, c2, rtol=1e-4, atol=1e-4)


def test_lloyd_host_rejects_pageable_memory():
    xh = torch.zeros(1, 256, 64, dtype=torch.bfloat16)      # not pinned
    c0 = torch.zeros(1, 4, 64, device="cuda")
    ids, centers, counts = _empty(1, 256, 4, 64)
    with pytest.raises(fkm.FkmError) as e:
        fkm.fkm_lloyd_host(xh, c0, 1, 0.0, 128, ids, centers, counts)
    assert e.value.code == 1


def test_lloyd_host_tol_matches_device_run():
    w = datagen.CONFIGS[1].scaled(iters=40, tol=1e-2)
    x, xt, c0 = problem(w)
    ids, centers, counts = _empty(w.B, w.N, w.K, w.D)
    n_h = fkm.fkm_lloyd_host(xt.cpu().pin_memory(), torch.from_numpy(c0).cuda(), 40, 1e-2, 1000,
                             ids, centers, counts)
    ref = oracle.lloyd(x, c0, 40, 1e-2, dtype="f32")
    assert n_h == ref["n_iter"]


# ------------------------------------------------------------------ comparison kernels
@pytest.mark.parametrize("dtype,B,N,K,D", [("bf16", 2, 3000, 300, 128), ("f16", 1, 1000, 1000, 64),
                                           ("f32", 1, 2000, 64, 128)])
def test_baseline_matches_oracle(dtype, B, N, K, D):
    w = datagen.Workload("base", B, N, D, K, dtype, K, sigma=0.5, iters=1, seed=N + 7)
    x, xt, c0 = problem(w)
    c = torch.from_numpy(c0).cuda()
    dist = torch.empty(B, N, K, dtype=torch.float32, device="cuda")
    ids = torch.empty(B, N, dtype=torch.int32, device="cuda")
    fkm.fkm_baseline_assign(xt, c, dist, ids)
    g = ids.cpu().numpy()
    check_assign(x, dtype, c0, g)
    # the materialised matrix holds the distances to q(c)
    ch = oracle.chat(c0.astype(np.float64), _mirror(dtype))
    xf = datagen.widen(x, dtype).astype(np.float64)
    ref = ((xf[:, :64, None, :] - ch[:, None, :, :]) ** 2).sum(-1)
    scale = (xf[:, :64] ** 2).sum(-1)[..., None] + (ch ** 2).sum(-1)[:, None, :]
    assert np.all(np.abs(dist.cpu().numpy()[:, :64] - ref) <= 1e-5 * scale + 1e-3)
    cn = torch.empty_like(c)
    cnt = torch.empty(B, K, dtype=torch.int32, device="cuda")
    fkm.fkm_baseline_update(xt, ids, c, cn, cnt)
    c_ref, n_ref, _ = oracle.update(x, g, c0.astype(np.float64), dtype=dtype)
    assert np.array_equal(cnt.cpu().numpy(), n_ref)
    assert np.allclose(cn.cpu().numpy(), c_ref, rtol=1e-4, atol=1e-4)


def test_stage_profile_with_and_without_graph():
    """Stage timing works for the graph-captured loop (tol = 0) and for the
    stepped loop that reads the shift every iteration (tol > 0)."""
    w = datagen.CONFIGS[3].scaled(B=2, N=3000, K=100, iters=3)
    x, xt, c0 = problem(w)
    ids, centers, counts = _empty(w.B, w.N, w.K, w.D)
    fkm.fkm_profile(True)
    try:
        fkm.fkm_profile_read(reset=True)
        for tol in (0.0, 1e-12):
            n = fkm.fkm_lloyd(xt, torch.from_numpy(c0).cuda(), 3, tol, ids, centers, counts)
            torch.cuda.synchronize()
            p = fkm.fkm_profile_read(reset=True)
            assert p["iterations"] == n
            assert all(p[s] > 0 for s in fkm.STAGES), p
    finally:
        fkm.fkm_profile(False)


def test_bounded_wait_runs_out_without_a_fault():
    """Failure detection: a wait nobody satisfies ends with FKM_ERR_TIMEOUT in
    the status word after its limit, and the context stays usable."""
    w = datagen.CONFIGS[2].scaled(B=1, N=2000, K=64, iters=1)
    x, xt, c0 = problem(w)
    ws = fkm.workspace(fkm.fkm_workspace_size(w.B, w.N, w.K, w.D, xt.dtype))
    fkm.fkm_selftest_wait_timeout(2_000_000, ws)   # 2 ms
    with pytest.raises(fkm.FkmError) as e:
        fkm.fkm_sync_status(ws)
    assert e.value.code == 5
    fkm.fkm_sync_status(ws)                       # the status was cleared
    ids = torch.empty(w.B, w.N, dtype=torch.int32, device="cuda")
    fkm.fkm_assign(xt, torch.from_numpy(c0).cuda(), ids, ws=ws)
    fkm.fkm_sync_status(ws)
    check_assign(x, w.dtype, c0, ids.cpu().numpy())


def test_lloyd_host_injected_copy_failure(monkeypatch):
    """Failure detection on the host: a streamed copy made to fail (no GPU
    fault) is reported as FKM_ERR_CUDA, and the next call, without the
    injection, runs cleanly and matches a run that never failed."""
    w = datagen.Workload("ooc_fault", 1, 9000, 64, 40, "f32", 40, sigma=0.5, iters=3, seed=77)
    x, xt, c0 = problem(w)
    xh = xt.cpu().pin_memory()
    c0t = torch.from_numpy(c0).cuda()
    ids, centers, counts = _empty(w.B, w.N, w.K, w.D)
    monkeypatch.setenv("FKM_FAULT_INJECT", "h2d@chunk:4")
    with pytest.raises(fkm.FkmError) as e:
        fkm.fkm_lloyd_host(xh, c0t, 3, 0.0, 2048, ids, centers, counts)
    assert e.value.code == 3 and "injected" in str(e.value)
    monkeypatch.delenv("FKM_FAULT_INJECT")
    torch.cuda.synchronize()
    n = fkm.fkm_lloyd_host(xh, c0t, 3, 0.0, 2048, ids, centers, counts)
    i2, c2, n2 = _empty(w.B, w.N, w.K, w.D)
    fkm.fkm_lloyd_host(xh, c0t, 3, 0.0, 2048, i2, c2, n2)
    assert n == 3
    assert torch.equal(ids, i2) and torch.equal(counts, n2)
    assert torch.allclose(centers, c2, rtol=1e-6, atol=1e-7)


# ------------------------------------------------------------------ large D
# D above 256 (fp32 points: 128): the assign kernel streams the point tile
# chunk by chunk with the centroids (the accumulator persists across the D
# chunks), and the segment sums run over 512-byte column slabs of each row.
@pytest.mark.parametrize("dtype,B,N,K,D", [("bf16", 2, 3000, 300, 512), ("f16", 1, 2500, 257, 1024),
                                           ("bf16", 1, 1500, 64, 2048), ("bf16", 1, 700, 40, 264),
                                           ("f32", 1, 1200, 50, 132), ("f32", 2, 900, 70, 512),
                                           ("f32", 1, 800, 30, 2048)])
def test_large_d(dtype, B, N, K, D):
    w = datagen.Workload("large_d", B, N, D, K, dtype, K, sigma=0.5, iters=3, seed=D + N)
    x, xt, c0 = problem(w)
    c0t = torch.from_numpy(c0).cuda()
    mir = _mirror(dtype)
    # assign, teacher-forced, from the oracle's centroids after one iteration
    c1 = oracle.lloyd(x, c0, 1, dtype=dtype, mirror=mir)["centers"].astype(np.float32)
    ids = torch.empty(B, N, dtype=torch.int32, device="cuda")
    inertia = torch.empty(B, dtype=torch.float64, device="cuda")
    fkm.fkm_assign(xt, torch.from_numpy(c1).cuda(), ids, inertia)
    g = ids.cpu().numpy()
    check_assign(x, dtype, c1, g)
    J = oracle.inertia(x, g, c1.astype(np.float64), dtype=dtype, mirror=mir)
    for b in range(B):
        assert rel(inertia[b].item(), J[b]) < 1e-4
    # update, teacher-forced on those ids
    c = torch.empty(B, K, D, device="cuda")
    n = torch.empty(B, K, dtype=torch.int32, device="cuda")
    fkm.fkm_update(xt, ids, torch.from_numpy(c1).cuda(), c, n)
    check_update(x, dtype, g, c1, c.cpu().numpy(), n.cpu().numpy())
    # the loop against the oracle, walked iteration by iteration
    _walk_lloyd(f"large D {dtype} D={D}", x, xt, c0, dtype, 3, 0.0)


def test_large_d_host_streaming():
    w = datagen.Workload("large_d_host", 1, 6000, 512, 100, "bf16", 100, sigma=0.5, iters=2, seed=9)
    x, xt, c0 = problem(w)
    ids, centers, counts = _empty(1, w.N, w.K, w.D)
    fkm.fkm_lloyd_host(xt.cpu().pin_memory(), torch.from_numpy(c0).cuda(), 2, 0.0, 2048, ids,
                       centers, counts)
    i2, c2, n2 = _empty(1, w.N, w.K, w.D)
    fkm.fkm_lloyd(xt, torch.from_numpy(c0).cuda(), 2, 0.0, i2, c2, n2)
    assert (ids != i2).float().mean().item() <= 1e-3
    assert torch.allclose(centers, c2, rtol=1e-4, atol=1e-4)


def test_inputs_written_by_a_kernel_just_before_the_call():
    """The loop's kernels are launched as programmatic dependents of the work
    before them on the stream; an input written by a torch kernel right
    before the call must be seen in full (every kernel waits for its
    predecessor before touching memory)."""
    w = datagen.CONFIGS[2].scaled(B=2, N=6000, K=300, iters=3)
    x, xt, c0 = problem(w)
    ref = _empty(w.B, w.N, w.K, w.D)
    fkm.fkm_lloyd(xt, torch.from_numpy(c0).cuda(), 3, 0.0, *ref)
    ids_a = torch.empty(w.B, w.N, dtype=torch.int32, device="cuda")
    fkm.fkm_assign(xt, torch.from_numpy(c0).cuda(), ids_a)
    torch.cuda.synchronize()
    for _ in range(3):
        xs = torch.zeros_like(xt)
        cs = torch.zeros(w.B, w.K, w.D, device="cuda")
        got = _empty(w.B, w.N, w.K, w.D)
        xs.add_(xt)                          # elementwise kernels on the same stream,
        cs.add_(torch.from_numpy(c0).cuda())  # launched just before the library's
        fkm.fkm_lloyd(xs, cs, 3, 0.0, *got)
        assert torch.equal(got[0], ref[0]) and torch.equal(got[2], ref[2])
        assert torch.allclose(got[1], ref[1], rtol=1e-6, atol=1e-6)
        xs2 = torch.zeros_like(xt)
        ids = torch.full((w.B, w.N), -1, dtype=torch.int32, device="cuda")
        xs2.add_(xt)
        fkm.fkm_assign(xs2, cs, ids)
        assert torch.equal(ids, ids_a)
