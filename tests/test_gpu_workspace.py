"""The workspace, checked from the outside.

Atomics: the Sort-Inverse Update makes one atomic add per segment boundary,
O((K + N/B_N) d) in all, where a scatter update makes O(N d) ("Flash-KMeans：
快速且内存高效精确K-Means聚类" summary, sections 前置知识 / argsort与分段规约 and
方法步骤详情 step (2)).  The library counts the fp64 element atomics its
segment sums make; the count must equal the one implied by the sorted order
(D per run that crosses a range boundary, per range it touches) and stay
within the pages' bound, on skewed (Zipf) and many-empty-cluster ids.

Uninitialised scratch: only the first 256 bytes (status words) of a
workspace must start at zero.  With every other byte poisoned (0xFF: NaN
floats, -1 integers; 0x7F: huge finite values) assign, update and the loops
on odd shapes must give what they give on a zeroed workspace (ids and counts
bit for bit, floating-point outputs to 1e-6: fp64 sums made with atomics
differ in their last bits between any two runs), and pass the oracle
checks: no kernel may read scratch it did not write.
"""
import math

import numpy as np
import pytest
import torch

import datagen
import exact_means_clustering_b200 as fkm
import oracle
from parity import check_assign, check_update, problem, to_torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _crossing_flushes(sk, R):
    """Flushes of runs that cross a range boundary, ranges of R sorted rows:
    per range, its first run if the key continues from the previous range,
    its last run if the key continues into the next (once if they are the
    same run)."""
    n = len(sk)
    W = -(-n // R)
    starts = np.arange(W) * R
    ends = np.minimum(starts + R, n)
    left = np.zeros(W, bool)
    left[1:] = sk[starts[1:] - 1] == sk[starts[1:]]
    right = np.zeros(W, bool)
    inner = ends < n
    right[inner] = sk[ends[inner] - 1] == sk[ends[inner]]
    single = sk[starts] == sk[ends - 1]
    return int(left.sum() + right.sum() - (left & right & single).sum()), W


@pytest.mark.parametrize("case", ["zipf", "many_empty", "one_cluster"])
@pytest.mark.parametrize("dtype,D", [("bf16", 64), ("f32", 32), ("bf16", 512)])
def test_update_atomics_meet_the_pages_bound(case, dtype, D):
    B, N, K = 2, 300_000, 1000
    rng = np.random.default_rng(11)
    if case == "zipf":
        p = (np.arange(K) + 1.0) ** -1.1
    elif case == "many_empty":
        p = np.zeros(K)
        p[::10] = 1.0
    else:
        p = np.zeros(K)
        p[K // 2] = 1.0
    ids = np.stack([rng.choice(K, size=N, p=p / p.sum()) for _ in range(B)]).astype(np.int32)
    w = datagen.Workload("atomics", B, N, D, K, dtype, 0, sigma=1.0, seed=5)
    x = datagen.points(w)
    xt = to_torch(x, dtype)
    prev = torch.zeros(B, K, D, device="cuda")
    c = torch.empty_like(prev)
    n = torch.empty(B, K, dtype=torch.int32, device="cuda")
    ws = fkm.workspace(fkm.fkm_workspace_size(B, N, K, D, xt.dtype))
    fkm.fkm_update(xt, torch.from_numpy(ids).cuda(), prev, c, n, ws=ws)
    count, R = fkm.fkm_segsum_stats(ws, B * N, reset=True)
    keys = (np.arange(B)[:, None] * K + ids).reshape(-1)
    sk = np.sort(keys, kind="stable")
    flushes, W = _crossing_flushes(sk, R)
    assert count == D * flushes, (count, D * flushes, R)
    assert count <= (B * K + W) * D            # the pages' O((K + N/B_N) d)
    assert count <= 2 * W * D                  # at most two crossing runs per range
    assert count * 50 < B * N * D              # a scatter update makes N*D
    # the counter was reset by the read
    assert fkm.fkm_segsum_stats(ws, B * N)[0] == 0
    check_update(x, dtype, ids, np.zeros((B, K, D), np.float32), c.cpu().numpy(),
                 n.cpu().numpy())


def _poisoned(nbytes, fill):
    ws = torch.full((max(int(nbytes), 256),), fill, dtype=torch.uint8, device="cuda")
    ws[:256] = 0
    return ws


def _run_all(xt, c0t, ws, tol_iters):
    """assign, update, the graph loop, the stepped loop and a cosine loop on one
    workspace."""
    B, N, D = xt.shape
    K = c0t.shape[1]
    out = {}
    ids = torch.full((B, N), -7, dtype=torch.int32, device="cuda")
    inertia = torch.full((B,), -1.0, dtype=torch.float64, device="cuda")
    fkm.fkm_assign(xt, c0t, ids, inertia, ws=ws)
    out["assign_ids"], out["assign_obj"] = ids.clone(), inertia.clone()
    cen = torch.full_like(c0t, -3.0)
    cnt = torch.full((B, K), -5, dtype=torch.int32, device="cuda")
    sh = torch.full((B,), -1.0, dtype=torch.float64, device="cuda")
    ob = torch.full((B,), -1.0, dtype=torch.float64, device="cuda")
    fkm.fkm_update(xt, ids, c0t, cen, cnt, sh, ob, ws=ws)
    out["update"] = (cen.clone(), cnt.clone(), sh.clone(), ob.clone())
    for tol in (0.0, 1e-12):
        i2 = torch.full((B, N), -7, dtype=torch.int32, device="cuda")
        c2 = torch.full_like(c0t, -3.0)
        n2 = torch.full((B, K), -5, dtype=torch.int32, device="cuda")
        o2 = torch.full((B,), -1.0, dtype=torch.float64, device="cuda")
        it = fkm.fkm_lloyd(xt, c0t, tol_iters, tol, i2, c2, n2, o2, ws=ws)
        out[f"lloyd{tol}"] = (it, i2, c2, n2, o2)
    i3 = torch.full((B, N), -7, dtype=torch.int32, device="cuda")
    c3 = torch.full_like(c0t, -3.0)
    n3 = torch.full((B, K), -5, dtype=torch.int32, device="cuda")
    o3 = torch.full((B,), -1.0, dtype=torch.float64, device="cuda")
    it = fkm.fkm_lloyd_metric(xt, c0t, tol_iters, 0.0, i3, c3, n3, "cosine", o3, ws=ws)
    out["cosine"] = (it, i3, c3, n3, o3)
    fkm.fkm_sync_status(ws)
    return out


@pytest.mark.parametrize("fill", [0xFF, 0x7F])
@pytest.mark.parametrize("dtype,B,N,K,D", [("bf16", 3, 1000, 300, 64), ("f16", 2, 4097, 257, 32),
                                           ("f32", 1, 3001, 70, 132), ("bf16", 1, 9000, 2500, 128),
                                           ("bf16", 2, 777, 33, 264)])
def test_poisoned_workspace_gives_the_zeroed_result(fill, dtype, B, N, K, D):
    w = datagen.Workload("poison", B, N, D, K, dtype, K, sigma=0.5, iters=3, seed=N + K + fill)
    x, xt, c0 = problem(w)
    c0t = torch.from_numpy(c0).cuda()
    nbytes = fkm.fkm_workspace_size(B, N, K, D, xt.dtype)
    clean = _run_all(xt, c0t, fkm.workspace(nbytes), 3)
    dirty = _run_all(xt, c0t, _poisoned(nbytes, fill), 3)
    for k in clean:
        a, b = clean[k], dirty[k]
        a = a if isinstance(a, tuple) else (a,)
        b = b if isinstance(b, tuple) else (b,)
        for u, v in zip(a, b):
            if not torch.is_tensor(u):
                assert u == v, k
            elif u.is_floating_point():
                # fp64 sums made with atomics vary in their last bits from
                # run to run; a read of poisoned scratch would not be small
                assert torch.allclose(u, v, rtol=1e-6, atol=1e-6), \
                    f"{k} differs on a poisoned workspace"
            else:
                assert torch.equal(u, v), f"{k} differs on a poisoned workspace"
    ids = dirty["assign_ids"].cpu().numpy()
    check_assign(x, dtype, c0, ids)
    cen, cnt = dirty["update"][0].cpu().numpy(), dirty["update"][1].cpu().numpy()
    check_update(x, dtype, ids, c0, cen, cnt)
    mir = dtype if dtype != "f32" else None
    J = oracle.inertia(x, ids, c0.astype(np.float64), dtype=dtype, mirror=mir)
    got = dirty["assign_obj"].cpu().numpy()
    assert np.all(np.abs(got - J) <= 1e-4 * np.abs(J)), (got, J)
    assert math.isfinite(float(dirty["update"][2].sum()))
