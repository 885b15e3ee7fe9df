"""fp64 CPU oracle for exact batched Lloyd k-means -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg (and its ``--impl reference`` arm) may import this package.  The product
path (the CUDA library and its binding) never imports or calls it.

The arithmetic lives in ``oracle.c`` (plain C, fp64, OpenMP over independent
points / dimensions), which cites the page and section each function follows.
This module only compiles it and marshals numpy arrays.

Parity pins: every function here is pinned by ``tests/test_oracle.py``
(the pages' argsort example, brute force on tiny inputs, closed forms for
K = 1 and K = N, the D = 1 nearest-neighbour rule, exact integer-grid cases,
translation invariance, monotone objective, fixed point, storage rounding).
The dot-product and cosine functions are pinned against the Euclidean ones
where the metrics coincide (unit-norm points and centroids; centroids of
equal norm), by scale invariance, and by the spherical objective's monotone
ascent.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

F32, F16, BF16 = 0, 1, 2
PURE = -1
DTYPE_CODE = {"f32": F32, "f16": F16, "bf16": BF16}


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (gcc -O2, OpenMP) if missing or stale."""
    if (not force and os.path.exists(_LIB)
            and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)):
        return _LIB
    tmp = _LIB + f".tmp{os.getpid()}"
    subprocess.run(["gcc", "-O2", "-std=gnu11", "-fPIC", "-shared", "-fopenmp", _SRC,
                    "-o", tmp, "-lm"], check=True)
    os.replace(tmp, _LIB)
    return _LIB


_lib = None
_P = ctypes.c_void_p
_I = ctypes.c_int64


def _load():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        L.orc_quantise.argtypes = [_P, _I, ctypes.c_int, _P]
        L.orc_quantise.restype = None
        L.orc_chat.argtypes = [_P, _I, _I, _I, ctypes.c_int, _P]
        L.orc_chat.restype = None
        L.orc_assign.argtypes = [_I, _I, _I, _I, _P, ctypes.c_int, _P, ctypes.c_int, _P, _P, _P, _P]
        L.orc_inertia.argtypes = [_I, _I, _I, _I, _P, ctypes.c_int, _P, _P, ctypes.c_int, _P]
        L.orc_update.argtypes = [_I, _I, _I, _I, _P, ctypes.c_int, _P, _P, _P, _P, _P]
        L.orc_lloyd.argtypes = [_I, _I, _I, _I, _P, ctypes.c_int, _P, ctypes.c_int,
                                ctypes.c_double, ctypes.c_int, _P, _P, _P, _P, _P, _P, _P]
        L.orc_argsort_stable.argtypes = [_P, _I, _I, _P]
        L.orc_centre.argtypes = [_I, _I, _I, _P, ctypes.c_int, _P, _P, _P]
        _c = ctypes.c_int
        L.orc_assign_sim.argtypes = [_I, _I, _I, _I, _P, _c, _P, _c, _c, _P, _P, _P]
        L.orc_similarity.argtypes = [_I, _I, _I, _I, _P, _c, _P, _P, _c, _P]
        L.orc_update_sim.argtypes = [_I, _I, _I, _I, _P, _c, _P, _P, _c, _P, _P, _P]
        L.orc_lloyd_sim.argtypes = [_I, _I, _I, _I, _P, _c, _P, _c, ctypes.c_double, _c, _c,
                                    _P, _P, _P, _P, _P, _P, _P]
        for f in ("orc_assign", "orc_inertia", "orc_update", "orc_lloyd", "orc_argsort_stable",
                  "orc_centre", "orc_assign_sim", "orc_similarity", "orc_update_sim",
                  "orc_lloyd_sim"):
            getattr(L, f).restype = ctypes.c_int
        _lib = L
    return _lib


def _ptr(a):
    return ctypes.c_void_p(a.ctypes.data) if a is not None else ctypes.c_void_p(0)


def _x3(x, dtype):
    if x.ndim == 2:
        x = x[None]
    x = np.ascontiguousarray(x)
    code = DTYPE_CODE[dtype]
    want = {F32: np.float32, F16: np.float16, BF16: np.uint16}[code]
    if x.dtype != want:
        raise TypeError(f"points for dtype {dtype} must be stored as {want}, got {x.dtype}")
    return x, code


def _c3(c, B):
    c = np.ascontiguousarray(c, dtype=np.float64)
    if c.ndim == 2:
        c = c[None]
    if c.shape[0] != B:
        raise ValueError("centroid batch does not match points")
    return c


def _mirror(mirror):
    if mirror is None or mirror == "pure":
        return PURE
    return DTYPE_CODE[mirror]


def quantise(c, mirror):
    """Elementwise q(fp32(c)) rounded RNE to ``mirror`` ('bf16'/'f16'/'f32'), or c in pure mode."""
    c = np.ascontiguousarray(c, dtype=np.float64)
    out = np.empty_like(c)
    _load().orc_quantise(_ptr(c), c.size, _mirror(mirror), _ptr(out))
    return out


def chat(c, mirror):
    """The centroids the assign step measures against, [B, K, D] (or [K, D]):
    m + q(fp32(fp32(c) - m)) per batch with m the mean fp32 centroid (mirror
    mode), or c itself in pure mode."""
    c = np.ascontiguousarray(c, dtype=np.float64)
    squeeze = c.ndim == 2
    c3 = c[None] if squeeze else c
    out = np.empty_like(c3)
    B, K, D = c3.shape
    _load().orc_chat(_ptr(c3), B, K, D, _mirror(mirror), _ptr(out))
    return out[0] if squeeze else out


def assign(x, c, dtype="f32", mirror=None):
    """Nearest centroid per point: returns (ids int32 [B,N], d1, d2 float64 [B,N], J [B])."""
    x, code = _x3(x, dtype)
    B, N, D = x.shape
    c = _c3(c, B)
    K = c.shape[1]
    ids = np.empty((B, N), np.int32)
    d1 = np.empty((B, N), np.float64)
    d2 = np.empty((B, N), np.float64)
    J = np.empty(B, np.float64)
    rc = _load().orc_assign(B, N, K, D, _ptr(x), code, _ptr(c), _mirror(mirror), _ptr(ids),
                            _ptr(d1), _ptr(d2), _ptr(J))
    if rc:
        raise RuntimeError("orc_assign failed")
    return ids, d1, d2, J


def inertia(x, ids, c, dtype="f32", mirror=None):
    """Objective of a given assignment against c_hat: J [B] float64."""
    x, code = _x3(x, dtype)
    B, N, D = x.shape
    c = _c3(c, B)
    ids = np.ascontiguousarray(ids, dtype=np.int32).reshape(B, N)
    J = np.empty(B, np.float64)
    rc = _load().orc_inertia(B, N, c.shape[1], D, _ptr(x), code, _ptr(ids), _ptr(c),
                             _mirror(mirror), _ptr(J))
    if rc:
        raise RuntimeError("orc_inertia failed (id out of range?)")
    return J


def update(x, ids, c_prev, dtype="f32"):
    """Centroid update: returns (c_new float64 [B,K,D], counts int64 [B,K], shift [B])."""
    x, code = _x3(x, dtype)
    B, N, D = x.shape
    c_prev = _c3(c_prev, B)
    K = c_prev.shape[1]
    ids = np.ascontiguousarray(ids, dtype=np.int32).reshape(B, N)
    c_new = np.empty_like(c_prev)
    counts = np.empty((B, K), np.int64)
    shift = np.empty(B, np.float64)
    rc = _load().orc_update(B, N, K, D, _ptr(x), code, _ptr(ids), _ptr(c_prev), _ptr(c_new),
                            _ptr(counts), _ptr(shift))
    if rc:
        raise RuntimeError("orc_update failed (id out of range?)")
    return c_new, counts, shift


def lloyd(x, c0, max_iters, tol=0.0, dtype="f32", mirror=None):
    """Full Lloyd run.  Returns a dict: ids, centers, counts, inertia, n_iter, J_hist, shift_hist."""
    x, code = _x3(x, dtype)
    B, N, D = x.shape
    c0 = _c3(c0, B)
    K = c0.shape[1]
    ids = np.empty((B, N), np.int32)
    centers = np.empty_like(c0)
    counts = np.empty((B, K), np.int64)
    inert = np.empty(B, np.float64)
    n_iter = ctypes.c_int(0)
    J_hist = np.full((max_iters, B), np.nan)
    sh_hist = np.full((max_iters, B), np.nan)
    rc = _load().orc_lloyd(B, N, K, D, _ptr(x), code, _ptr(c0), max_iters, float(tol),
                           _mirror(mirror), _ptr(ids), _ptr(centers), _ptr(counts), _ptr(inert),
                           ctypes.byref(n_iter), _ptr(J_hist), _ptr(sh_hist))
    if rc:
        raise RuntimeError("orc_lloyd failed")
    n = n_iter.value
    return dict(ids=ids, centers=centers, counts=counts, inertia=inert, n_iter=n,
                J_hist=J_hist[:n], shift_hist=sh_hist[:n])


# ---- dot-product and cosine k-means (see oracle.c for the readings) ----
METRIC_CODE = {"dot": 1, "cosine": 2}


def assign_sim(x, c, metric, dtype="f32", mirror=None):
    """Most similar centroid per point under ``metric`` ('dot' or 'cosine'):
    returns (ids int32 [B,N], s1 best score, s2 second-best score [B,N])."""
    x, code = _x3(x, dtype)
    B, N, D = x.shape
    c = _c3(c, B)
    K = c.shape[1]
    ids = np.empty((B, N), np.int32)
    s1 = np.empty((B, N), np.float64)
    s2 = np.empty((B, N), np.float64)
    rc = _load().orc_assign_sim(B, N, K, D, _ptr(x), code, _ptr(c), METRIC_CODE[metric],
                                _mirror(mirror), _ptr(ids), _ptr(s1), _ptr(s2))
    if rc:
        raise RuntimeError("orc_assign_sim failed")
    return ids, s1, s2


def similarity(x, ids, c, metric, dtype="f32"):
    """Objective of an assignment: J [B] = sum_i x_i . v_{ids_i}, v = c (dot) or c/||c||."""
    x, code = _x3(x, dtype)
    B, N, D = x.shape
    c = _c3(c, B)
    ids = np.ascontiguousarray(ids, dtype=np.int32).reshape(B, N)
    J = np.empty(B, np.float64)
    rc = _load().orc_similarity(B, N, c.shape[1], D, _ptr(x), code, _ptr(ids), _ptr(c),
                                METRIC_CODE[metric], _ptr(J))
    if rc:
        raise RuntimeError("orc_similarity failed (id out of range?)")
    return J


def update_sim(x, ids, c_prev, metric, dtype="f32"):
    """Update under ``metric``: returns (c_new float64 [B,K,D], counts [B,K], shift [B])."""
    x, code = _x3(x, dtype)
    B, N, D = x.shape
    c_prev = _c3(c_prev, B)
    K = c_prev.shape[1]
    ids = np.ascontiguousarray(ids, dtype=np.int32).reshape(B, N)
    c_new = np.empty_like(c_prev)
    counts = np.empty((B, K), np.int64)
    shift = np.empty(B, np.float64)
    rc = _load().orc_update_sim(B, N, K, D, _ptr(x), code, _ptr(ids), _ptr(c_prev),
                                METRIC_CODE[metric], _ptr(c_new), _ptr(counts), _ptr(shift))
    if rc:
        raise RuntimeError("orc_update_sim failed (id out of range?)")
    return c_new, counts, shift


def lloyd_sim(x, c0, max_iters, metric, tol=0.0, dtype="f32", mirror=None):
    """Lloyd run under ``metric``; the same dict as lloyd()."""
    x, code = _x3(x, dtype)
    B, N, D = x.shape
    c0 = _c3(c0, B)
    K = c0.shape[1]
    ids = np.empty((B, N), np.int32)
    centers = np.empty_like(c0)
    counts = np.empty((B, K), np.int64)
    inert = np.empty(B, np.float64)
    n_iter = ctypes.c_int(0)
    J_hist = np.full((max_iters, B), np.nan)
    sh_hist = np.full((max_iters, B), np.nan)
    rc = _load().orc_lloyd_sim(B, N, K, D, _ptr(x), code, _ptr(c0), max_iters, float(tol),
                               METRIC_CODE[metric], _mirror(mirror), _ptr(ids), _ptr(centers),
                               _ptr(counts), _ptr(inert), ctypes.byref(n_iter), _ptr(J_hist),
                               _ptr(sh_hist))
    if rc:
        raise RuntimeError("orc_lloyd_sim failed")
    n = n_iter.value
    return dict(ids=ids, centers=centers, counts=counts, inertia=inert, n_iter=n,
                J_hist=J_hist[:n], shift_hist=sh_hist[:n])


def argsort_stable(keys, n_keys=None):
    """Stable argsort of non-negative integer keys (counting sort)."""
    keys = np.ascontiguousarray(keys, dtype=np.int64)
    if n_keys is None:
        n_keys = int(keys.max()) + 1 if keys.size else 1
    idx = np.empty(keys.size, np.int64)
    rc = _load().orc_argsort_stable(_ptr(keys), keys.size, int(n_keys), _ptr(idx))
    if rc:
        raise RuntimeError("orc_argsort_stable failed")
    return idx


def centre(x, dtype="f32", mu=None):
    """Centred points and their mean (README "Centre your data"): returns
    (xc in the storage form of dtype, mu float32 [B, D]).  mu: optional given
    mean [B, D] (float32) to subtract instead of the computed one."""
    x, code = _x3(x, dtype)
    B, N, D = x.shape
    xc = np.empty_like(x)
    mu_out = np.empty((B, D), np.float32)
    mu_in = None if mu is None else np.ascontiguousarray(mu, dtype=np.float32).reshape(B, D)
    rc = _load().orc_centre(B, N, D, _ptr(x), code, _ptr(mu_in), _ptr(mu_out), _ptr(xc))
    if rc:
        raise RuntimeError("orc_centre failed")
    return xc, mu_out
