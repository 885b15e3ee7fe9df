"""Pins for the fp64 oracle: each checks it against something other than itself.

What pins what:
  argsort      the pages' worked example (golden fixture) and numpy's stable sort
  assign       integer-grid constructions with a known nearest centroid and exact
               distances; the D = 1 midpoint (bisection) rule; numpy's argmin of a
               distance table on tiny random inputs
  update       numpy means / bincount; the empty-cluster rule
  lloyd        exhaustive search over all partitions of a tiny set; K = 1 and
               K = N closed forms; duplicate centroids; translation invariance;
               monotone objective; fixed point after convergence; tol semantics
  mirror mode  storage rounding against numpy float16 and torch bfloat16
"""
import itertools
import json
import os

import numpy as np
import pytest

import datagen
import oracle
import torch


def _bf16_bits(a):
    import torch
    t = torch.tensor(np.asarray(a, np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def _bf16_value(a):
    import torch
    return torch.tensor(np.asarray(a, np.float32)).to(torch.bfloat16).to(torch.float64).numpy()


# ----------------------------------------------------------------- argsort
def test_argsort_pages_example(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "argsort_example.json")))
    idx = oracle.argsort_stable(g["keys"])
    assert idx.tolist() == g["sorted_idx"]
    assert np.asarray(g["keys"])[idx].tolist() == g["sorted_keys"]


def test_argsort_matches_numpy_stable():
    rng = np.random.default_rng(1)
    for n, nk in [(1, 1), (17, 3), (1000, 7), (5000, 300)]:
        keys = rng.integers(0, nk, size=n)
        assert np.array_equal(oracle.argsort_stable(keys, nk), np.argsort(keys, kind="stable"))


def test_argsort_rejects_out_of_range():
    with pytest.raises(RuntimeError):
        oracle.argsort_stable(np.array([0, 5]), 3)


# ------------------------------------------------------------------ assign
def _grid_problem(rng, B, N, K, D, spacing=16, jitter=3):
    """Centroids on a coarse integer lattice, points = centroid + small integer offset.
    Neighbouring lattice centroids are `spacing` apart, so a point at most
    `jitter` from its own centroid in every coordinate is strictly nearest to
    it.  The centroid set is symmetric (v and -v), so its mean is exactly zero
    and the centred operand of mirror mode equals the centroid itself."""
    c = np.zeros((B, K, D))
    for b in range(B):
        pts = set()
        while len(pts) < K // 2:
            v = tuple(rng.integers(-4, 5, size=D) * spacing)
            if any(v) and tuple(-t for t in v) not in pts:
                pts.add(v)
        half = np.array(sorted(pts), dtype=np.float64)
        full = np.concatenate([half, -half] + ([np.zeros((1, D))] if K % 2 else []))
        c[b] = full[rng.permutation(K)]
    owner = rng.integers(0, K, size=(B, N))
    off = rng.integers(-jitter, jitter + 1, size=(B, N, D))
    x = np.take_along_axis(c, owner[..., None], axis=1) + off
    return x, c, owner, off


@pytest.mark.parametrize("dtype", ["f32", "bf16", "f16"])
def test_assign_integer_grid_known_owner(dtype):
    rng = np.random.default_rng(7)
    B, N, K, D = 2, 300, 9, 4
    x, c, owner, off = _grid_problem(rng, B, N, K, D)
    # small integers are exact in every storage type
    xs = {"f32": x.astype(np.float32), "f16": x.astype(np.float16),
          "bf16": _bf16_bits(x)}[dtype]
    ids, d1, d2, J = oracle.assign(xs, c, dtype=dtype, mirror=dtype)
    assert np.array_equal(ids, owner)
    assert np.array_equal(d1, (off.astype(np.float64) ** 2).sum(-1))
    assert np.allclose(J, d1.sum(1), rtol=0, atol=0)
    assert np.all(d2 >= d1)


def test_assign_ties_go_to_lowest_index():
    # every point equidistant from centroids 1 and 3 (and farther from 0, 2)
    x = np.array([[[0.0, 0.0]], [[2.0, 0.0]]], dtype=np.float32).reshape(1, 2, 2)
    c = np.array([[[9, 9], [1, 1], [9, -9], [1, -1]]], dtype=np.float64)
    ids, d1, d2, _ = oracle.assign(x, c)
    assert ids.tolist() == [[1, 1]]
    assert np.array_equal(d1, d2)  # exact tie: best == second best


def test_assign_d1_bisection_rule():
    """D = 1: the nearest centroid is found by bisecting the sorted centroids'
    midpoints, an algorithm unrelated to the oracle's scan."""
    rng = np.random.default_rng(3)
    K, N = 37, 2000
    cvals = rng.choice(np.arange(-500, 500), size=K, replace=False).astype(np.float64) / 4
    x = (rng.integers(-2200, 2200, size=N) / 8.0).astype(np.float32)
    order = np.argsort(cvals)
    cs = cvals[order]
    mids = (cs[:-1] + cs[1:]) / 2
    xd = x.astype(np.float64)
    pos = np.searchsorted(mids, xd, side="left")   # mids[pos-1] < x <= mids[pos]
    exp = order[pos].copy()
    # on an exact midpoint both neighbours tie: the lower original index wins
    tie = (pos < K - 1) & (mids[np.minimum(pos, K - 2)] == xd)
    exp[tie] = np.minimum(order[pos[tie]], order[pos[tie] + 1])
    assert tie.sum() > 0
    ids, d1, d2, _ = oracle.assign(x.reshape(1, N, 1), cvals.reshape(1, K, 1))
    assert np.array_equal(ids[0], exp)
    assert np.array_equal(d1[0], (x.astype(np.float64) - cvals[exp]) ** 2)
    # second best: the smaller of the two sorted neighbours' distances
    dist = (x.astype(np.float64)[:, None] - cvals[None, :]) ** 2
    assert np.array_equal(d2[0], np.sort(dist, axis=1)[:, 1])


def test_assign_matches_numpy_table_tiny():
    rng = np.random.default_rng(11)
    for (N, K, D) in [(1, 1, 1), (5, 3, 2), (64, 8, 4), (33, 7, 3)]:
        x = rng.standard_normal((2, N, D)).astype(np.float32)
        c = rng.standard_normal((2, K, D))
        ids, d1, _, J = oracle.assign(x, c)
        tab = np.linalg.norm(x.astype(np.float64)[:, :, None, :] - c[:, None, :, :], axis=-1) ** 2
        assert np.array_equal(ids, np.argmin(tab, axis=-1))
        assert np.allclose(d1, tab.min(-1), rtol=1e-12, atol=1e-12)
        assert np.allclose(J, tab.min(-1).sum(-1), rtol=1e-12)


def _symmetric_set(rng, B, h, D, scale):
    """Centroid sets {v, -v} (and 0 when odd): their mean is exactly zero in
    any summation order, so the centred operand must be the plain storage
    rounding of the centroids."""
    v = rng.standard_normal((B, h, D)) * scale
    return np.concatenate([v, -v], axis=1)


@pytest.mark.parametrize("mirror", ["bf16", "f16"])
def test_centred_operand_of_a_zero_mean_set_is_the_storage_rounding(mirror):
    """m = 0 exactly (a set closed under negation): c_hat = q(fp32(c)), which
    torch (bf16) and numpy (fp16) round independently of the oracle."""
    rng = np.random.default_rng(31)
    c = _symmetric_set(rng, 3, 40, 16, 5.0)
    ref = (_bf16_value(c) if mirror == "bf16"
           else c.astype(np.float32).astype(np.float16).astype(np.float64))
    assert np.array_equal(oracle.chat(c, mirror), ref)


@pytest.mark.parametrize("mirror", ["bf16", "f16"])
def test_centred_operand_of_a_single_centroid_is_exact(mirror):
    """K = 1: the mean is the centroid itself, its offset is zero, so c_hat is
    the fp32 centroid however far it lies from the origin."""
    rng = np.random.default_rng(32)
    c = rng.standard_normal((4, 1, 24)) * 1000.0 + 777.0
    assert np.array_equal(oracle.chat(c, mirror), c.astype(np.float32).astype(np.float64))


@pytest.mark.parametrize("mirror", ["bf16", "f16"])
def test_centred_operand_of_a_translated_zero_mean_set(mirror):
    """A zero-mean set moved by an integer vector mu: the mean is exactly mu
    and every offset is the original centroid, so c_hat = q(c) + mu exactly
    (values on a 1/64 grid keep the fp32 steps exact)."""
    rng = np.random.default_rng(33)
    c = np.round(_symmetric_set(rng, 2, 20, 8, 3.0) * 64) / 64
    mu = rng.integers(-300, 300, size=(2, 1, 8)).astype(np.float64)
    q = (_bf16_value(c) if mirror == "bf16"
         else c.astype(np.float32).astype(np.float16).astype(np.float64))
    assert np.array_equal(oracle.chat(c + mu, mirror), q + mu)


def test_mirror_mode_is_assign_against_centred_rounded_centroids():
    """The mirror-mode assign measures distances to oracle.chat(c): it equals
    a pure-mode assign against those points (ids and distances)."""
    rng = np.random.default_rng(5)
    x = (rng.standard_normal((2, 500, 16)) + 20).astype(np.float16)
    c = rng.standard_normal((2, 40, 16)) + 20
    ch = oracle.chat(c, "f16")
    ids_m, d1_m, _, _ = oracle.assign(x, c, dtype="f16", mirror="f16")
    ids_p, d1_p, _, _ = oracle.assign(x, ch, dtype="f16", mirror=None)
    assert np.array_equal(ids_m, ids_p) and np.array_equal(d1_m, d1_p)
    xb = _bf16_bits(rng.standard_normal((1, 500, 16)) * 3 - 40)
    cb = rng.standard_normal((1, 40, 16)) * 3 - 40
    ids_m, _, _, _ = oracle.assign(xb, cb, dtype="bf16", mirror="bf16")
    ids_p, _, _, _ = oracle.assign(xb, oracle.chat(cb, "bf16"), dtype="bf16", mirror=None)
    assert np.array_equal(ids_m, ids_p)


def test_centred_operand_error_scales_with_spread_not_offset():
    """RNE to bf16 moves each offset by at most half an ulp: |c_hat - c| is
    bounded by 2^-8 |c - m| (plus the fp32 rounding of c, of m and of c - m),
    however far the centroids sit from the origin."""
    rng = np.random.default_rng(21)
    for offset in (0.0, 64.0, -5000.0):
        c = rng.standard_normal((3, 30, 8)) + offset
        c32 = c.astype(np.float32).astype(np.float64)
        ch = oracle.chat(c, "bf16")
        spread = np.abs(c32 - c32.mean(axis=1, keepdims=True))
        assert np.all(np.abs(ch - c32) <= 2.0 ** -8 * spread + 2.0 ** -21 * np.abs(c32))


def test_centred_operand_is_translation_invariant():
    """Shifting every centroid by a small integer vector shifts c_hat by the
    same vector exactly (values on a 1/64 grid keep every step exact)."""
    rng = np.random.default_rng(22)
    c = np.round(rng.standard_normal((2, 16, 8)) * 64) / 64
    mu = rng.integers(-20, 20, size=(2, 1, 8)).astype(np.float64)
    for mir in ("bf16", "f16"):
        assert np.array_equal(oracle.chat(c + mu, mir), oracle.chat(c, mir) + mu)


# ---------------------------------------------------------- storage rounding
def test_quantise_bf16_against_torch():
    rng = np.random.default_rng(2)
    vals = np.concatenate([
        rng.standard_normal(20000) * 10.0 ** rng.integers(-8, 8, 20000),
        [1 + 2 ** -8, 1 + 3 * 2 ** -8, -(1 + 2 ** -8), 0.0, -0.0, 3.0e38, 1e-40]])
    q = oracle.quantise(vals, "bf16")
    assert np.array_equal(q, _bf16_value(vals))
    assert q[-7] == 1.0 and q[-6] == 1 + 2 ** -6     # ties to even


def test_quantise_f16_against_numpy():
    rng = np.random.default_rng(4)
    vals = np.concatenate([rng.standard_normal(20000) * 10.0 ** rng.integers(-6, 5, 20000),
                           [1 + 2 ** -11, 1 + 3 * 2 ** -11, 65519.0, 65520.0, 6e-8]])
    q = oracle.quantise(vals, "f16")
    with np.errstate(over="ignore"):
        ref = vals.astype(np.float32).astype(np.float16).astype(np.float64)
    assert np.array_equal(q, ref)
    assert q[-5] == 1.0 and q[-4] == 1 + 2 ** -9 and np.isinf(q[-2])


def test_quantise_goes_through_fp32_first():
    v = np.array([1.0 + 2 ** -8 + 2 ** -40])  # fp32 rounding drops 2^-40, leaving a bf16 tie
    assert oracle.quantise(v, "bf16")[0] == 1.0
    assert oracle.quantise(v, None)[0] == v[0]


# ------------------------------------------------------------------ update
def test_update_means_counts_and_empty_rule():
    rng = np.random.default_rng(9)
    B, N, K, D = 3, 400, 12, 5
    x = rng.standard_normal((B, N, D)).astype(np.float32)
    ids = rng.integers(0, K - 2, size=(B, N)).astype(np.int32)  # clusters K-2, K-1 stay empty
    ids[1, :] = 0                                               # batch 1: one cluster only
    c_prev = rng.standard_normal((B, K, D))
    c_new, counts, shift = oracle.update(x, ids, c_prev)
    for b in range(B):
        assert np.array_equal(counts[b], np.bincount(ids[b], minlength=K))
        for k in range(K):
            m = ids[b] == k
            if m.any():
                assert np.allclose(c_new[b, k], x[b][m].astype(np.float64).mean(0), rtol=1e-13)
            else:
                assert np.array_equal(c_new[b, k], c_prev[b, k])
        assert np.isclose(shift[b], np.sum((c_new[b] - c_prev[b]) ** 2), rtol=1e-13)
    assert counts.sum(1).tolist() == [N] * B


def test_update_is_exact_on_small_integers():
    rng = np.random.default_rng(10)
    x = rng.integers(-50, 50, size=(1, 256, 8)).astype(np.float32)
    ids = (np.arange(256) % 4).astype(np.int32).reshape(1, 256)
    c_new, counts, _ = oracle.update(x, ids, np.zeros((1, 4, 8)))
    for k in range(4):
        s = x[0][ids[0] == k].astype(np.int64).sum(0)
        assert np.array_equal(c_new[0, k] * 64, s)   # 64 points each: exact division


def test_update_rejects_bad_ids():
    x = np.zeros((1, 4, 2), np.float32)
    with pytest.raises(RuntimeError):
        oracle.update(x, np.array([[0, 1, 2, 3]]), np.zeros((1, 3, 2)))


# ------------------------------------------------------------------- lloyd
def _within_ss(x, labels, K):
    tot = 0.0
    for k in range(K):
        m = labels == k
        if m.any():
            tot += m.sum() * np.var(x[m], axis=0).sum()
    return tot


def test_lloyd_from_exhaustive_optimum_stays_there():
    """Enumerate every partition of 7 points into 2 clusters: Lloyd started at the
    optimal partition's means must keep that partition and report its objective."""
    rng = np.random.default_rng(12)
    x = np.concatenate([rng.standard_normal((4, 2)) + [6, 0], rng.standard_normal((3, 2)) - [6, 0]])
    x = x.astype(np.float32)
    xd = x.astype(np.float64)
    best, best_lab = np.inf, None
    for bits in itertools.product([0, 1], repeat=7):
        lab = np.array(bits)
        if lab.min() == lab.max():
            continue
        v = _within_ss(xd, lab, 2)
        if v < best:
            best, best_lab = v, lab
    c0 = np.stack([xd[best_lab == k].mean(0) for k in range(2)])
    r = oracle.lloyd(x[None], c0[None], max_iters=3)
    assert np.array_equal(r["ids"][0], best_lab)
    assert np.isclose(r["inertia"][0], best, rtol=1e-12)
    assert np.allclose(r["centers"][0], c0, rtol=1e-13)


def test_lloyd_never_beats_exhaustive_optimum():
    rng = np.random.default_rng(13)
    for trial in range(5):
        x = rng.standard_normal((8, 2)).astype(np.float32)
        xd = x.astype(np.float64)
        best = min(_within_ss(xd, np.array(l), 3)
                   for l in itertools.product(range(3), repeat=8) if len(set(l)) == 3)
        c0 = xd[rng.permutation(8)[:3]]
        r = oracle.lloyd(x[None], c0[None], max_iters=20)
        # objective of the final partition with its own means >= the global optimum
        assert _within_ss(xd, r["ids"][0], 3) >= best - 1e-12


def test_lloyd_k1_closed_form():
    rng = np.random.default_rng(14)
    x = (rng.standard_normal((2, 300, 6)) * 3 + 1).astype(np.float32)
    r = oracle.lloyd(x, np.zeros((2, 1, 6)), max_iters=2)
    xd = x.astype(np.float64)
    assert np.all(r["ids"] == 0) and r["counts"].tolist() == [[300], [300]]
    assert np.allclose(r["centers"][:, 0], xd.mean(1), rtol=1e-13)
    # second assignment is against the mean: objective = N * sum of variances
    assert np.allclose(r["inertia"], 300 * np.var(xd, axis=1).sum(-1), rtol=1e-11)


def test_lloyd_k_equals_n_identity():
    rng = np.random.default_rng(15)
    x = rng.standard_normal((1, 50, 4)).astype(np.float32)
    r = oracle.lloyd(x, x.astype(np.float64), max_iters=3)
    assert np.array_equal(r["ids"][0], np.arange(50))
    assert np.array_equal(r["centers"], x.astype(np.float64))
    assert r["inertia"][0] == 0.0 and np.all(r["counts"] == 1)


def test_lloyd_duplicate_centroid_empties_higher_index():
    rng = np.random.default_rng(16)
    x = rng.standard_normal((1, 200, 3)).astype(np.float32)
    c0 = np.stack([x[0, 0], x[0, 0], x[0, 1] + 5]).astype(np.float64)
    r = oracle.lloyd(x, c0[None], max_iters=1)
    assert r["counts"][0, 1] == 0
    assert np.array_equal(r["centers"][0, 1], c0[1])
    assert not np.any(r["ids"] == 1)


def test_lloyd_translation_invariance():
    """k-means is translation invariant (README, "Centre your data"): x + mu gives
    the same ids and centers + mu.  Values are multiples of 1/64 so x + mu is exact."""
    rng = np.random.default_rng(17)
    x = (np.round(rng.standard_normal((2, 500, 8)) * 64) / 64).astype(np.float32)
    mu = rng.integers(-20, 20, size=(2, 1, 8)).astype(np.float32)
    c0 = x[:, :10].astype(np.float64)
    a = oracle.lloyd(x, c0, max_iters=6)
    bb = oracle.lloyd(x + mu, c0 + mu, max_iters=6)
    assert np.array_equal(a["ids"], bb["ids"])
    assert np.allclose(bb["centers"], a["centers"] + mu, rtol=1e-12, atol=1e-12)
    assert np.allclose(bb["inertia"], a["inertia"], rtol=1e-10)


def test_lloyd_objective_monotone_and_counts_sum():
    import datagen
    w = datagen.CONFIGS[2].scaled(B=2, N=3000, K=40, D=16)
    x = datagen.points(w)
    c0 = datagen.init_centroids(x, datagen.init_indices(w), w.dtype)
    r = oracle.lloyd(x, c0, max_iters=12, dtype="bf16", mirror=None)
    J = r["J_hist"]
    assert np.all(J[1:] <= J[:-1] * (1 + 1e-12))
    assert np.all(r["counts"].sum(1) == w.N)


def test_lloyd_fixed_point_after_convergence():
    rng = np.random.default_rng(18)
    x = np.concatenate([rng.standard_normal((100, 2)) + o for o in ([0, 8], [8, 0], [-8, -8])])
    x = x.astype(np.float32)[None]
    r = oracle.lloyd(x, x[:, [0, 100, 200]].astype(np.float64), max_iters=50, tol=1e-300)
    assert r["n_iter"] < 50
    ids2, _, _, _ = oracle.assign(x, r["centers"])
    c2, _, sh = oracle.update(x, ids2, r["centers"])
    assert np.array_equal(ids2, r["ids"]) and np.array_equal(c2, r["centers"]) and sh[0] == 0


def test_lloyd_wiring_matches_step_chain():
    """ids = last assignment, centers = the update after it, inertia = that
    assignment's objective, in mirror mode too."""
    import datagen
    w = datagen.CONFIGS[3].scaled(B=2, N=700, K=9, D=8)
    x = datagen.points(w)
    c = datagen.init_centroids(x, datagen.init_indices(w), w.dtype).astype(np.float64)
    r = oracle.lloyd(x, c, max_iters=4, dtype="f16", mirror="f16")
    for _ in range(4):
        ids, _, _, J = oracle.assign(x, c, dtype="f16", mirror="f16")
        c, counts, _ = oracle.update(x, ids, c, dtype="f16")
    assert np.array_equal(r["ids"], ids) and np.array_equal(r["centers"], c)
    assert np.array_equal(r["counts"], counts) and np.array_equal(r["inertia"], J)


def test_lloyd_tol_semantics():
    rng = np.random.default_rng(19)
    x = rng.standard_normal((2, 300, 4)).astype(np.float32)
    c0 = x[:, :5].astype(np.float64)
    assert oracle.lloyd(x, c0, max_iters=7, tol=0.0)["n_iter"] == 7
    assert oracle.lloyd(x, c0, max_iters=7, tol=1e30)["n_iter"] == 1
    r = oracle.lloyd(x, c0, max_iters=30, tol=1e-3)
    sh = r["shift_hist"]
    assert sh[-1].max() < 1e-3 and np.all(sh[:-1].max(1) >= 1e-3)


# ---------------------------------------------------------------- centring
# README "Centre your data": k-means is translation invariant; centring
# subtracts the per-batch mean of the points.

def _store(x32, dtype):
    if dtype == "bf16":
        return (torch.from_numpy(x32).to(torch.bfloat16).view(torch.int16).numpy()
                .view(np.uint16))
    return x32.astype(np.float16 if dtype == "f16" else np.float32)


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
def test_centre_integer_grid_is_exact(dtype):
    rng = np.random.default_rng(5)
    B, N, D = 2, 64, 8
    x = rng.integers(-20, 21, size=(B, N, D)).astype(np.float32)
    x -= x.mean(axis=1, keepdims=True).round()       # column sums now small integers
    x[:, -1, :] -= x.sum(axis=1)                      # ... and exactly zero: mean 0
    x += np.arange(D, dtype=np.float32) * 4           # mean = 4 d, exact
    xs = _store(x, dtype)
    xc, mu = oracle.centre(xs, dtype)
    assert np.array_equal(mu, np.broadcast_to(np.arange(D, dtype=np.float32) * 4, (B, D)))
    assert np.array_equal(datagen.widen(xc, dtype), x - mu[:, None, :])


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
def test_centre_subtraction_matches_library_rounding(dtype):
    rng = np.random.default_rng(6)
    B, N, D = 2, 300, 16
    x32 = (rng.standard_normal((B, N, D)) * 3 + 50).astype(np.float32)
    xs = _store(x32, dtype)
    mu = rng.standard_normal((B, D)).astype(np.float32) * 7
    xc, mu_used = oracle.centre(xs, dtype, mu=mu)
    assert np.array_equal(mu_used, mu)
    ref = _store(datagen.widen(xs, dtype) - mu[:, None, :], dtype)   # fp32 subtract, library RNE
    assert np.array_equal(xc.view(np.uint8), ref.view(np.uint8))


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_centre_mean_matches_numpy(dtype):
    rng = np.random.default_rng(7)
    x32 = (rng.standard_normal((3, 1000, 24)) + 64).astype(np.float32)
    xs = _store(x32, dtype)
    _, mu = oracle.centre(xs, dtype)
    ref = datagen.widen(xs, dtype).astype(np.float64).mean(axis=1).astype(np.float32)
    assert np.all(np.abs(mu.view(np.int32).astype(np.int64) - ref.view(np.int32)) <= 1)


def test_centre_is_translation_free():
    """Centring x and x + t (t exact, every value exact) gives the same points."""
    rng = np.random.default_rng(8)
    x = rng.integers(-50, 50, size=(1, 128, 8)).astype(np.float32)
    t = np.array([64, -32, 0, 8, 1, 2, 3, 4], np.float32)
    a, _ = oracle.centre(x, "f32")
    b, _ = oracle.centre(x + t, "f32")
    assert np.array_equal(a, b)


# ---------------------------------------------------- dot-product and cosine
def _unit_centroids(D, K, rng):
    """K distinct rows of exactly unit norm in fp32: signed axis vectors and
    (+-1/2, +-1/2, +-1/2, +-1/2) on a random choice of four axes."""
    rows = set()
    while len(rows) < K:
        v = np.zeros(D)
        if rng.random() < 0.5:
            v[rng.integers(D)] = rng.choice([-1.0, 1.0])
        else:
            v[rng.choice(D, 4, replace=False)] = rng.choice([-0.5, 0.5], 4)
        rows.add(tuple(v))
    return np.array(sorted(rows))


def _clear_of_ties(d1, d2, eps=1e-9):
    return (d2 - d1) > eps


def test_cosine_equals_euclid_on_unit_centroids():
    """||x - c||^2 = ||x||^2 + 1 - 2 x.c for unit c: nearest = most similar."""
    rng = np.random.default_rng(21)
    B, N, K, D = 2, 300, 12, 8
    x = rng.standard_normal((B, N, D)).astype(np.float32)
    c = np.stack([_unit_centroids(D, K, rng) for _ in range(B)])
    ids_e, d1, d2, _ = oracle.assign(x, c)
    ok = _clear_of_ties(d1, d2)
    for metric in ("cosine", "dot"):
        ids_s, s1, s2 = oracle.assign_sim(x, c, metric)
        assert ok.mean() > 0.99
        assert np.array_equal(ids_s[ok], ids_e[ok])
        assert np.all(s1 >= s2)


def test_dot_equals_euclid_for_equal_norm_centroids():
    rng = np.random.default_rng(22)
    B, N, K, D = 1, 400, 10, 8
    x = rng.standard_normal((B, N, D)).astype(np.float32)
    c = 3.0 * _unit_centroids(D, K, rng)[None]       # every row of norm exactly 3
    ids_e, d1, d2, _ = oracle.assign(x, c)
    ids_s, _, _ = oracle.assign_sim(x, c, "dot")
    ok = _clear_of_ties(d1, d2)
    assert np.array_equal(ids_s[ok], ids_e[ok])


def test_sim_assign_matches_numpy_argmax_tiny():
    rng = np.random.default_rng(23)
    x = rng.standard_normal((1, 40, 5)).astype(np.float32)
    c = rng.standard_normal((1, 7, 5))
    xd = x[0].astype(np.float64)
    dot = xd @ c[0].T
    u = (c[0] / np.linalg.norm(c[0], axis=1, keepdims=True)).astype(np.float32).astype(np.float64)
    cos = xd @ u.T
    assert np.array_equal(oracle.assign_sim(x, c, "dot")[0][0], dot.argmax(1))
    assert np.array_equal(oracle.assign_sim(x, c, "cosine")[0][0], cos.argmax(1))


def test_sim_assign_mirror_scores_against_the_centred_rounded_operand():
    rng = np.random.default_rng(24)
    x = rng.standard_normal((1, 60, 16)).astype(np.float32)
    c = rng.standard_normal((1, 9, 16)) + 5.0
    xd = x[0].astype(np.float64)
    ch = oracle.chat(c, "bf16")[0]
    assert np.array_equal(oracle.assign_sim(x, c, "dot", mirror="bf16")[0][0],
                          (xd @ ch.T).argmax(1))
    u = (c[0] / np.linalg.norm(c[0], axis=1, keepdims=True)).astype(np.float32)
    chu = oracle.chat(u.astype(np.float64)[None], "bf16")[0]
    assert np.array_equal(oracle.assign_sim(x, c, "cosine", mirror="bf16")[0][0],
                          (xd @ chu.T).argmax(1))


def test_cosine_assign_is_scale_invariant():
    """Scaling points and centroid rows by powers of two (exact in fp32)
    leaves every cosine assignment unchanged."""
    rng = np.random.default_rng(25)
    x = rng.standard_normal((2, 200, 12)).astype(np.float32)
    c = rng.standard_normal((2, 9, 12))
    ids0, _, _ = oracle.assign_sim(x, c, "cosine")
    xs = (x * (2.0 ** rng.integers(-3, 4, size=(2, 200, 1)))).astype(np.float32)
    cs = c * 2.0 ** rng.integers(-3, 4, size=(2, 9, 1))
    assert np.array_equal(oracle.assign_sim(xs, cs, "cosine")[0], ids0)


def test_sim_ties_go_to_lowest_index():
    x = np.array([[[1.0, 2.0]]], np.float32)
    c = np.array([[[0.0, 1.0], [2.0, 0.0], [0.0, 1.0]]])   # dot: 2, 2, 2
    assert oracle.assign_sim(x, c, "dot")[0][0, 0] == 0
    c2 = np.array([[[0.0, 5.0], [0.0, 1.0]]])              # cosine: equal directions
    assert oracle.assign_sim(x, c2, "cosine")[0][0, 0] == 0


def test_update_sim_dot_is_the_mean_cosine_the_unit_sum():
    rng = np.random.default_rng(26)
    B, N, K, D = 2, 300, 8, 6
    x = rng.standard_normal((B, N, D)).astype(np.float32)
    ids = rng.integers(0, K - 1, size=(B, N)).astype(np.int32)     # cluster K-1 empty
    ids[0, :2] = K - 2
    ids[0, 2:][ids[0, 2:] == K - 2] = 0
    x[0, 1] = -x[0, 0]                                             # cluster K-2: zero sum
    c_prev = rng.standard_normal((B, K, D))
    cd, nd, shd = oracle.update_sim(x, ids, c_prev, "dot")
    cc, nc, shc = oracle.update_sim(x, ids, c_prev, "cosine")
    for b in range(B):
        assert np.array_equal(nd[b], np.bincount(ids[b], minlength=K))
        assert np.array_equal(nc[b], nd[b])
        for k in range(K):
            m = ids[b] == k
            s = x[b][m].astype(np.float64).sum(0)
            if not m.any() or not s.any():
                assert np.array_equal(cc[b, k], c_prev[b, k])
            else:
                assert np.allclose(cd[b, k], s / m.sum(), rtol=1e-13)
                assert np.isclose(np.linalg.norm(cc[b, k]), 1.0, rtol=1e-14)
                assert np.allclose(cc[b, k] * np.linalg.norm(s), s, rtol=1e-12, atol=1e-12)
        assert np.isclose(shc[b], np.sum((cc[b] - c_prev[b]) ** 2), rtol=1e-13)


def test_similarity_closed_forms():
    """Dot: J = sum_k s_k . c_k over the cluster sums.  Cosine, against the
    centroids the update just formed: J = sum_k ||s_k||."""
    rng = np.random.default_rng(27)
    B, N, K, D = 2, 250, 7, 5
    x = rng.standard_normal((B, N, D)).astype(np.float32)
    ids = rng.integers(0, K, size=(B, N)).astype(np.int32)
    c = rng.standard_normal((B, K, D))
    sums = np.zeros((B, K, D))
    for b in range(B):
        np.add.at(sums[b], ids[b], x[b].astype(np.float64))
    assert np.allclose(oracle.similarity(x, ids, c, "dot"), np.einsum("bkd,bkd->b", sums, c),
                       rtol=1e-12)
    cc, _, _ = oracle.update_sim(x, ids, c, "cosine")
    # the update's rows are unit length in fp64; the objective rounds them to fp32 first
    J = oracle.similarity(x, ids, cc, "cosine")
    assert np.allclose(J, np.linalg.norm(sums, axis=2).sum(1), rtol=1e-6)


def test_spherical_lloyd_objective_never_decreases():
    """Assignment maximises each point's similarity and the unit sum maximises
    each cluster's, so J can only grow (pure mode)."""
    rng = np.random.default_rng(28)
    w = datagen.CONFIGS[1].scaled(B=2, N=600, K=9, iters=8)
    x = datagen.points(w)
    c0 = datagen.init_centroids(x, datagen.init_indices(w), w.dtype)
    r = oracle.lloyd_sim(x, c0, 8, "cosine", dtype=w.dtype)
    J = r["J_hist"]
    assert np.all(np.diff(J, axis=0) >= -1e-9 * np.abs(J[1:]))
    assert np.all(r["counts"].sum(1) == w.N)
    assert np.allclose(np.linalg.norm(r["centers"], axis=2)[r["counts"] > 0], 1.0, rtol=1e-12)


@pytest.mark.parametrize("metric", ["dot", "cosine"])
def test_lloyd_sim_wiring_matches_step_chain(metric):
    rng = np.random.default_rng(29)
    x = rng.standard_normal((2, 120, 6)).astype(np.float32)
    c0 = x[:, :5].astype(np.float64)
    r = oracle.lloyd_sim(x, c0, 2, metric)
    c = c0
    for _ in range(2):
        ids, _, _ = oracle.assign_sim(x, c, metric)
        J = oracle.similarity(x, ids, c, metric)
        c, counts, _ = oracle.update_sim(x, ids, c, metric)
    assert np.array_equal(r["ids"], ids)
    assert np.array_equal(r["centers"], c)
    assert np.array_equal(r["inertia"], J)
    assert r["n_iter"] == 2
