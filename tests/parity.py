"""Shared helpers for the GPU parity tests: inputs from the shared generator,
marshalling to torch, and the acceptance criteria (written out here).

Criteria (the tolerance contract of the exact Lloyd iteration):
  assign   given the same centroids, ids equal the oracle's except at points
           where the GPU's choice is within 1e-4 * (||x||^2 + ||c_oracle||^2) of
           the best distance (a near tie), and such points number at most
           ceil(1e-4 * points).  Distances are to c_hat, the centroid the
           assignment measures against (oracle.chat: the centred operand
           m + q(c - m) for 16-bit points, c itself for fp32).
  update   given the same ids: counts bit-exact; empty clusters keep the
           previous centroid bit for bit; every other element within
           1e-5 * (sum over the cluster of |x_d|) / n_k of the fp64 mean.
  inertia  within 1e-4 relative.
  free run a loop is walked one iteration at a time against the oracle.  Where
           the GPU's ids first differ from the oracle's own trajectory, every
           differing point must lie in the near-tie band above (and number at
           most ceil(1e-4 * points)), the GPU's update of that step must pass
           the update criterion, and the oracle then continues from the GPU's
           centroids (re-seeded).  The final objective is held to 1e-4 of the
           oracle's at the last step, and such runs are reported by warning.
"""
import math
import warnings

import numpy as np
import torch

import datagen
import oracle

TORCH_DT = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}


def to_torch(x: np.ndarray, dtype: str, device="cuda") -> torch.Tensor:
    if dtype == "bf16":
        t = torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16)
    else:
        t = torch.from_numpy(np.ascontiguousarray(x))
    return t.to(device)


def problem(w: datagen.Workload):
    """(x numpy storage, x torch cuda, init centroids float32 numpy)."""
    x = datagen.points(w)
    c0 = datagen.init_centroids(x, datagen.init_indices(w), w.dtype)
    return x, to_torch(x, w.dtype), c0


def check_assign(x, dtype, c, gpu_ids, mirror=True, sample=None):
    """Teacher-forced assign check.  c: the float32 centroids both sides use.
    sample: optional (B, S) int array of point indices checked (full size runs)."""
    B = x.shape[0]
    mir = dtype if mirror and dtype != "f32" else None
    bad_total, pts_total = 0, 0
    for b in range(B):
        xb = x[b] if sample is None else x[b][sample[b]]
        gb = gpu_ids[b] if sample is None else gpu_ids[b][sample[b]]
        ids, d1, _, _ = oracle.assign(xb[None], c[b][None].astype(np.float64), dtype=dtype,
                                      mirror=mir)
        ids, d1 = ids[0], d1[0]
        mism = np.nonzero(ids != gb)[0]
        pts_total += len(gb)
        if len(mism) == 0:
            continue
        ch = oracle.chat(c[b][None].astype(np.float64), mir)[0]
        xf = datagen.widen(xb[mism], dtype).astype(np.float64)
        d_gpu = ((xf - ch[gb[mism]]) ** 2).sum(1)
        band = 1e-4 * ((xf ** 2).sum(1) + (ch[ids[mism]] ** 2).sum(1))
        over = d_gpu - d1[mism] > band
        assert not over.any(), (
            f"batch {b}: {over.sum()} points assigned outside the near-tie band, e.g. point "
            f"{mism[over][0]} gpu {gb[mism][over][0]} oracle {ids[mism][over][0]} "
            f"excess {(d_gpu - d1[mism])[over][0]:.3e} band {band[over][0]:.3e}")
        bad_total += len(mism)
    assert bad_total <= math.ceil(1e-4 * pts_total), f"{bad_total} near-tie flips of {pts_total}"
    return bad_total


def check_update(x, dtype, ids, prev, gpu_centers, gpu_counts):
    c_ref, n_ref, _ = oracle.update(x, ids, prev.astype(np.float64), dtype=dtype)
    assert np.array_equal(gpu_counts.astype(np.int64), n_ref), "counts differ"
    empty = n_ref == 0
    assert np.array_equal(gpu_centers[empty], prev[empty]), "empty clusters moved"
    B, K, D = prev.shape
    for b in range(B):
        xf = datagen.widen(x[b], dtype).astype(np.float64)
        absum = np.zeros((K, D))
        np.add.at(absum, ids[b], np.abs(xf))
        nk = np.maximum(n_ref[b], 1)[:, None]
        tol = 1e-5 * absum / nk + 1e-30
        err = np.abs(gpu_centers[b].astype(np.float64) - c_ref[b])
        occ = n_ref[b] > 0
        worst = (err[occ] / tol[occ]).max() if occ.any() else 0.0
        assert np.all(err[occ] <= tol[occ]), f"batch {b}: centroid error {worst:.2f}x tolerance"
    return c_ref, n_ref


def rel(a, b):
    return abs(float(a) - float(b)) / max(abs(float(b)), 1e-300)


def abs_storage(x: np.ndarray, dtype: str) -> np.ndarray:
    """|x| in the same storage form (bf16 bits: the sign bit cleared)."""
    if dtype == "bf16":
        return x & np.uint16(0x7FFF)
    return np.abs(x)


def cluster_abs_mean(x, dtype, ids, K, chunk_rows=1 << 24):
    """Per cluster mean of |x| over its points, [B, K, D] float64: the scale of
    the update tolerance.  Formed with the oracle's update on |x|, chunk by
    chunk of rows, so no full-size temporary is needed."""
    B, N, D = x.shape
    tot = np.zeros((B, K, D))
    cnt = np.zeros((B, K))
    zero = np.zeros((1, K, D))
    for b in range(B):
        for r0 in range(0, N, chunk_rows):
            xa = abs_storage(x[b, r0:r0 + chunk_rows], dtype)
            c, n, _ = oracle.update(xa[None], ids[b, r0:r0 + chunk_rows][None], zero, dtype=dtype)
            tot[b] += c[0] * n[0][:, None]
            cnt[b] += n[0]
    return tot / np.maximum(cnt, 1)[..., None]


def check_update_large(x, dtype, ids, prev, gpu_centers, gpu_counts):
    """check_update's criteria for full-size problems (no per-element Python work)."""
    c_ref, n_ref, _ = oracle.update(x, ids, prev.astype(np.float64), dtype=dtype)
    assert np.array_equal(gpu_counts.astype(np.int64), n_ref), "counts differ"
    empty = n_ref == 0
    assert np.array_equal(gpu_centers[empty], prev[empty]), "empty clusters moved"
    tol = 1e-5 * cluster_abs_mean(x, dtype, ids, prev.shape[1]) + 1e-30
    err = np.abs(gpu_centers.astype(np.float64) - c_ref)
    occ = ~empty
    ratio = err[occ] / tol[occ]
    assert np.all(ratio <= 1.0), f"centroid error {ratio.max():.2f}x tolerance"
    return c_ref, n_ref


# ------------------------------------------------ dot-product / cosine criteria
def scored(c, metric):
    """The vectors a metric scores against: c, or its rows rounded to fp32 after
    scaling to unit length."""
    v = c.astype(np.float64)
    if metric == "cosine":
        n = np.linalg.norm(v, axis=-1, keepdims=True)
        v = np.where(n > 0, v / np.where(n > 0, n, 1), 0).astype(np.float32).astype(np.float64)
    return v


def check_assign_sim(x, dtype, c, gpu_ids, metric):
    """A point may differ from the oracle only at a near tie: the oracle's best
    score beats the score of the GPU's choice by at most 1e-4 (||x||^2 +
    ||c_hat||^2); at most ceil(1e-4 points) such points."""
    mir = dtype if dtype != "f32" else None
    bad = pts = 0
    for b in range(x.shape[0]):
        ids, s1, _ = oracle.assign_sim(x[b][None], c[b][None].astype(np.float64), metric,
                                       dtype=dtype, mirror=mir)
        ids, s1, gb = ids[0], s1[0], gpu_ids[b]
        pts += len(gb)
        mism = np.nonzero(ids != gb)[0]
        if len(mism) == 0:
            continue
        ch = oracle.chat(scored(c[b], metric)[None], mir)[0]
        xf = datagen.widen(x[b][mism], dtype).astype(np.float64)
        s_gpu = (xf * ch[gb[mism]]).sum(1)
        band = 1e-4 * ((xf ** 2).sum(1) + (ch[ids[mism]] ** 2).sum(1))
        over = s1[mism] - s_gpu > band
        assert not over.any(), f"batch {b}: {over.sum()} points outside the near-tie band"
        bad += len(mism)
    assert bad <= math.ceil(1e-4 * pts), f"{bad} near-tie flips of {pts}"
    return bad


def check_update_sim(x, dtype, ids, prev, gpu_centers, gpu_counts, metric):
    """counts exact; clusters that keep prev bit-identical; the mean (dot)
    within 1e-5 of the cluster's mean |x|, the unit direction (cosine) within
    1e-5 of the cluster's sum of |x| over the length of its sum."""
    c_ref, n_ref, _ = oracle.update_sim(x, ids, prev.astype(np.float64), metric, dtype=dtype)
    assert np.array_equal(gpu_counts.astype(np.int64), n_ref), "counts differ"
    B, K, D = prev.shape
    for b in range(B):
        xf = datagen.widen(x[b], dtype).astype(np.float64)
        absum = np.zeros((K, D))
        s = np.zeros((K, D))
        np.add.at(absum, ids[b], np.abs(xf))
        np.add.at(s, ids[b], xf)
        kept = (n_ref[b] == 0) | ((metric == "cosine") & ~s.any(1))
        assert np.array_equal(gpu_centers[b][kept], prev[b][kept]), "kept clusters moved"
        occ = ~kept
        if metric == "dot":
            tol = 1e-5 * absum / np.maximum(n_ref[b], 1)[:, None] + 1e-30
        else:
            tol = 1e-5 * absum / np.maximum(np.linalg.norm(s, axis=1), 1e-300)[:, None] + 2e-7
        err = np.abs(gpu_centers[b].astype(np.float64) - c_ref[b])
        assert np.all(err[occ] <= tol[occ]), \
            f"batch {b}: centroid error {(err[occ] / tol[occ]).max():.2f}x tolerance"
        if metric == "cosine":
            nrm = np.linalg.norm(gpu_centers[b][occ].astype(np.float64), axis=1)
            assert np.allclose(nrm, 1.0, atol=1e-6)


# ------------------------------------------------------------ free-running loops
class NearTieDivergence(UserWarning):
    """A free-running loop whose trajectory parted from the oracle's at a
    proven near tie (the oracle was re-seeded from the GPU's centroids)."""


def check_free_running(x, dtype, c0, iters, tol, gpu_prefix, gpu_final, label,
                       metric="euclid"):
    """Walk a free-running GPU loop against the oracle one iteration at a time.

    gpu_prefix(t) -> (ids [B,N], centers [B,K,D] float32, counts [B,K]) of the
    loop run for t iterations with tol = 0 from c0; gpu_final -> (ids,
    objective [B], n_iter) of the loop under test (tol applied).

    At every step the oracle takes one Lloyd iteration from its current
    centroids.  If the GPU's ids of that step differ, the differing points
    must all be near ties of the oracle's assignment (check_assign's band and
    count), the GPU's update of the step must pass the update criterion
    against the oracle on the GPU's own ids, and the oracle continues from
    the GPU's centroids.  The stop step under tol and the final objective
    (1e-4 relative; objectives below 1e-9 count as zero) must match.
    Returns the steps (1-based) at which the oracle was re-seeded."""
    euclid = metric == "euclid"
    mir = dtype if dtype != "f32" else None
    B = x.shape[0]
    c_o = np.asarray(c0, np.float64)
    c_g = np.asarray(c0, np.float32)
    reseeds = []
    n_stop = iters
    J_ref = None
    for t in range(iters):
        if euclid:
            r = oracle.lloyd(x, c_o, 1, 0.0, dtype=dtype, mirror=mir)
        else:
            r = oracle.lloyd_sim(x, c_o, 1, metric, dtype=dtype, mirror=mir)
        g_ids, g_c, g_n = gpu_prefix(t + 1)
        J_ref = r["inertia"]
        if np.array_equal(g_ids, r["ids"]):
            c_o = r["centers"]
        else:
            if euclid:
                check_assign(x, dtype, c_o, g_ids)
                check_update(x, dtype, g_ids, c_g, g_c, g_n)
            else:
                check_assign_sim(x, dtype, c_o, g_ids, metric)
                check_update_sim(x, dtype, g_ids, c_g, g_c, g_n, metric)
            reseeds.append(t + 1)
            c_o = g_c.astype(np.float64)
        c_g = g_c
        if tol > 0.0 and float(np.max(r["shift_hist"][0])) < tol:
            n_stop = t + 1
            break
    f_ids, f_obj, f_n = gpu_final()
    assert f_n == n_stop, f"{label}: the GPU loop ran {f_n} iterations, the oracle {n_stop}"
    assert np.array_equal(f_ids, gpu_prefix(n_stop)[0]), f"{label}: loop and prefix runs differ"
    for b in range(B):
        if abs(J_ref[b]) < 1e-9 and abs(f_obj[b]) < 1e-9:
            continue
        assert rel(f_obj[b], J_ref[b]) < 1e-4, (label, b, f_obj[b], J_ref[b], reseeds)
    if reseeds:
        warnings.warn(f"{label}: trajectory parted from the oracle's at near ties at "
                      f"iteration(s) {reseeds}; each proven in the band, oracle re-seeded from "
                      f"the GPU's centroids there; final objective within 1e-4",
                      NearTieDivergence)
    return reseeds
