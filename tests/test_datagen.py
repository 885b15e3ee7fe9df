"""The shared input generator: published Philox answers, reproducibility, shapes."""
import json
import os

import numpy as np

import datagen


def test_philox_known_answers(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "philox4x32_10_kat.json")))
    for case in g["cases"]:
        ctr = [int(v, 16) for v in case["ctr"]]
        key = [int(v, 16) for v in case["key"]]
        assert datagen.philox4x32_10(ctr, key) == [int(v, 16) for v in case["out"]]


def test_points_reproducible_and_distributed():
    w = datagen.CONFIGS[3].scaled(B=2, N=5000, D=16)
    a = datagen.points(w)
    b = datagen.points(w)
    assert a.dtype == np.float16 and a.shape == (2, 5000, 16)
    assert np.array_equal(a, b)
    v = a.astype(np.float64)
    assert abs(v.mean()) < 0.02 and abs(v.std() - 1.0) < 0.02
    assert not np.array_equal(a[0], a[1])     # batches are independent streams


def test_mixture_labels_and_weights():
    w = datagen.CONFIGS[4].scaled(N=200000, K=64, n_comp=64)
    x, lab = datagen.points(w, with_labels=True)
    cnt = np.bincount(lab[0], minlength=64) / w.N
    zipf = np.arange(1, 65) ** -1.1
    zipf /= zipf.sum()
    assert np.allclose(cnt, zipf, atol=0.004)
    # points sit within a few sigma of their component's empirical centre
    xf = datagen.widen(x, "bf16")[0].astype(np.float64)
    c0 = xf[lab[0] == 0].mean(0)
    assert np.sqrt(((xf[lab[0] == 0] - c0) ** 2).sum(1)).mean() < 0.3 * np.sqrt(w.D) * 1.2


def test_dirichlet_weights_unbalanced():
    w = datagen.CONFIGS[2].scaled(B=1, N=100000, K=64, n_comp=64)
    _, lab = datagen.points(w, with_labels=True)
    frac = np.bincount(lab[0], minlength=64) / w.N
    assert frac.max() > 3.0 / 64 and frac.min() < 0.3 / 64


def test_perm_prefix_is_a_permutation_prefix():
    w = datagen.CONFIGS[1]
    idx = datagen.init_indices(w)
    assert idx.shape == (1, 64) and len(set(idx[0].tolist())) == 64
    assert idx.min() >= 0 and idx.max() < w.N
    full = datagen.init_indices(w.scaled(N=50, K=50))[0]
    assert sorted(full.tolist()) == list(range(50))
    assert np.array_equal(datagen.init_indices(w.scaled(N=50, K=20))[0], full[:20])


def test_init_centroids_are_exact_points():
    w = datagen.CONFIGS[2].scaled(B=2, N=1000, K=10, D=8)
    x = datagen.points(w)
    idx = datagen.init_indices(w)
    c = datagen.init_centroids(x, idx, "bf16")
    assert c.dtype == np.float32
    for b in range(2):
        assert np.array_equal(c[b], datagen.widen(x[b][idx[b]], "bf16"))
