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
"""
import math

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
