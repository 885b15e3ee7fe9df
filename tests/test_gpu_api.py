"""The centring helper and the class-style API on the GPU.

Centring follows the "Flash-KMeans" GitHub README, section "Centre your data":
the mean is checked against the oracle's within one fp32 ulp (the sums are
taken in another order), and the centred points bit for bit against the
oracle's subtraction of the GPU's own mean.  FlashKMeans must reproduce the
C ABI calls it wraps (README, section "Usage": fit / predict / fit_predict /
train)."""
import numpy as np
import pytest
import torch

import datagen
import exact_means_clustering_b200 as fkm
import oracle
from parity import problem, to_torch

pytestmark = pytest.mark.gpu


def _offset_points(dtype, B, N, D, seed):
    w = datagen.Workload("centre", B, N, D, 16, dtype, 16, sigma=0.5, seed=seed)
    x = datagen.points(w)
    xf = datagen.widen(x, dtype)
    xf[..., :3] += 64.0                    # a few channels far from the origin
    if dtype == "bf16":
        xs = torch.from_numpy(xf).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    else:
        xs = xf.astype(np.float16 if dtype == "f16" else np.float32)
    return xs


@pytest.mark.parametrize("dtype,B,N,D", [("bf16", 3, 5000, 128), ("f16", 2, 3001, 64),
                                         ("f32", 1, 2500, 32), ("bf16", 1, 1, 8)])
def test_centre_matches_oracle(dtype, B, N, D):
    xs = _offset_points(dtype, B, N, D, seed=N)
    xt = to_torch(xs, dtype)
    out, mu = fkm.fkm_centre(xt)
    _, mu_ref = oracle.centre(xs, dtype)
    g_mu = mu.cpu().numpy()
    assert np.all(np.abs(g_mu.view(np.int32).astype(np.int64) - mu_ref.view(np.int32)) <= 1)
    xc_ref, _ = oracle.centre(xs, dtype, mu=g_mu)
    g = out.cpu()
    g = g.view(torch.int16).numpy().view(np.uint16) if dtype == "bf16" else g.numpy()
    assert np.array_equal(g.view(np.uint8), xc_ref.view(np.uint8))
    # in place
    fkm.fkm_centre(xt, out=xt)
    assert torch.equal(xt, out)


def test_class_fit_predict_match_the_c_calls():
    w = datagen.CONFIGS[2].scaled(B=2, N=6000, K=200, iters=5)
    x, xt, c0 = problem(w)
    c0t = torch.from_numpy(c0).cuda()
    km = fkm.FlashKMeans(d=w.D, k=w.K, niter=5, tol=0.0)
    labels = km.fit_predict(xt, init_centroids=c0t)
    ids = torch.empty(w.B, w.N, dtype=torch.int32, device="cuda")
    cen = torch.empty(w.B, w.K, w.D, device="cuda")
    cnt = torch.empty(w.B, w.K, dtype=torch.int32, device="cuda")
    n = fkm.fkm_lloyd(xt, c0t, 5, 0.0, ids, cen, cnt)
    assert km.n_iter == n
    assert torch.equal(labels, ids)
    assert torch.equal(km.centroids, cen)
    p = km.predict(xt)
    ref = torch.empty_like(ids)
    fkm.fkm_assign(xt, cen, ref)
    assert torch.equal(p, ref)
    # 2-D input: one problem
    km1 = fkm.FlashKMeans(d=w.D, k=w.K, niter=5)
    l1 = km1.fit_predict(xt[0], init_centroids=c0t[0])
    assert l1.shape == (w.N,) and torch.equal(l1, ids[0])


def test_class_centre_runs_on_the_centred_points():
    xs = _offset_points("bf16", 2, 4000, 64, seed=11)
    xt = to_torch(xs, "bf16")
    K = 40
    init = xt[:, :K, :].float().contiguous()
    km = fkm.FlashKMeans(d=64, k=K, niter=4, centre=True)
    km.fit(xt, init_centroids=init)
    # the same run by hand: centre, cluster from the shifted init, shift back
    xc, mu = fkm.fkm_centre(xt)
    ids = torch.empty(2, 4000, dtype=torch.int32, device="cuda")
    cen = torch.empty(2, K, 64, device="cuda")
    cnt = torch.empty(2, K, dtype=torch.int32, device="cuda")
    fkm.fkm_lloyd(xc, (init - mu[:, None, :]).contiguous(), 4, 0.0, ids, cen, cnt)
    assert torch.equal(km.labels_, ids)
    assert torch.equal(km.centroids, cen + mu[:, None, :])


def test_class_train_on_host_data_streams_it():
    w = datagen.Workload("train", 1, 20000, 64, 50, "f32", 50, sigma=0.5, iters=3, seed=3)
    x, xt, c0 = problem(w)
    xh = xt.cpu()                                  # pageable: train pins a copy
    c0t = torch.from_numpy(c0).cuda()
    km = fkm.FlashKMeans(d=64, k=50, niter=3, chunk_rows=4096)
    km.train(xh, init_centroids=c0t)
    ids = torch.empty(1, w.N, dtype=torch.int32, device="cuda")
    cen = torch.empty(1, 50, 64, device="cuda")
    cnt = torch.empty(1, 50, dtype=torch.int32, device="cuda")
    fkm.fkm_lloyd_host(xh.pin_memory(), c0t, 3, 0.0, 4096, ids, cen, cnt)
    assert torch.equal(km.labels_, ids)
    assert torch.equal(km.centroids, cen)


@pytest.mark.parametrize("sign", [1, -1])
def test_shift_centroids_is_one_fp32_operation(sign):
    """fkm_shift_centroids: out = fp32(c + sign * mu) per batch, exactly the
    single IEEE fp32 operation numpy performs; in place as well."""
    rng = np.random.default_rng(3 + sign)
    B, K, D = 3, 1000, 40
    c = (rng.standard_normal((B, K, D)) * 100).astype(np.float32)
    mu = (rng.standard_normal((B, D)) * 1e4).astype(np.float32)
    ref = c + mu[:, None, :] if sign > 0 else c - mu[:, None, :]
    ct = torch.from_numpy(c).cuda()
    out = fkm.fkm_shift_centroids(ct, torch.from_numpy(mu).cuda(), sign)
    assert np.array_equal(out.cpu().numpy(), ref)
    fkm.fkm_shift_centroids(ct, torch.from_numpy(mu).cuda(), sign, out=ct)
    assert np.array_equal(ct.cpu().numpy(), ref)


def test_verbose_progress_lines(capfd):
    """fkm_set_verbose: one progress line per iteration on stderr (README
    "Usage", verbose), the same results as a quiet run, and the last line's
    objective is the loop's reported objective."""
    w = datagen.CONFIGS[2].scaled(B=2, N=3000, K=100, iters=3)
    x, xt, c0 = problem(w)
    c0t = torch.from_numpy(c0).cuda()
    outs = []
    for verbose in (0, 1):
        ids = torch.empty(w.B, w.N, dtype=torch.int32, device="cuda")
        cen = torch.empty(w.B, w.K, w.D, device="cuda")
        cnt = torch.empty(w.B, w.K, dtype=torch.int32, device="cuda")
        obj = torch.empty(w.B, dtype=torch.float64, device="cuda")
        fkm.fkm_set_verbose(verbose)
        try:
            n = fkm.fkm_lloyd(xt, c0t, 3, 0.0, ids, cen, cnt, obj)
        finally:
            fkm.fkm_set_verbose(0)
        outs.append((n, ids, cen, cnt, obj))
    err = capfd.readouterr().err
    lines = [l for l in err.splitlines() if l.startswith("fkm_lloyd: iteration")]
    assert [l.split()[2] for l in lines] == ["1/3", "2/3", "3/3"]
    (n0, i0, c_0, k0, o0), (n1, i1, c_1, k1, o1) = outs
    assert n0 == n1 == 3
    assert torch.equal(i0, i1) and torch.equal(k0, k1)
    assert torch.allclose(c_0, c_1, rtol=1e-6, atol=1e-7)
    printed = float(lines[-1].split("objective")[1].split()[0])
    assert abs(printed - o1.sum().item()) <= 1e-6 * abs(printed)
