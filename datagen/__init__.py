"""Seeded synthetic inputs for exact batched k-means runs.

This package is shared by the oracle's tests and by the GPU path's tests and
benchmark.  It holds no k-means arithmetic: it draws random numbers (see
``gen.c`` for the generator's definition and citations), lays out points in
their storage dtype, and picks initial-centroid indices as the first K entries
of a seeded per-batch permutation.  Rounding a generated value to bf16/fp16 is
input preparation: the rounded value is the input both sides read.

The workload recipes (``CONFIGS``) follow the Flash-KMeans pages' usage shapes
(GitHub README "Usage": B=32, N=75600, D=128, K=1000; paper summary
"Motivation": B=32, N=65536, K=1024, d=128; README "Large tensor Benchmark":
fp32, K ~ sqrt(N), N up to 2^28, data in host pinned memory).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass, field

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gen.c")
_LIB = os.path.join(_HERE, "libfkmgen.so")

DT_F32, DT_F16, DT_BF16 = 0, 1, 2
DTYPE_CODE = {"f32": DT_F32, "f16": DT_F16, "bf16": DT_BF16}
DTYPE_BYTES = {"f32": 4, "f16": 2, "bf16": 2}
NP_STORAGE = {"f32": np.float32, "f16": np.float16, "bf16": np.uint16}
W_EQUAL, W_DIRICHLET, W_ZIPF = 0, 1, 2


def build(force: bool = False) -> str:
    """Compile gen.c into libfkmgen.so (gcc, OpenMP) if it is missing or stale."""
    if (not force and os.path.exists(_LIB)
            and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)):
        return _LIB
    tmp = _LIB + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=gnu11", "-fPIC", "-shared", "-fopenmp", _SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        L.fkmgen_philox.argtypes = [ctypes.POINTER(ctypes.c_uint32)] * 3
        L.fkmgen_philox.restype = None
        L.fkmgen_points.argtypes = [
            ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_uint64, ctypes.c_uint32,
            ctypes.c_int, ctypes.c_int, ctypes.c_double, ctypes.c_double, ctypes.c_double,
            ctypes.c_void_p, ctypes.c_void_p]
        L.fkmgen_points.restype = ctypes.c_int
        L.fkmgen_perm_prefix.argtypes = [ctypes.c_int64, ctypes.c_int64, ctypes.c_uint64,
                                         ctypes.c_uint32, ctypes.c_void_p]
        L.fkmgen_perm_prefix.restype = ctypes.c_int
        _lib = L
    return _lib


def philox4x32_10(ctr, key):
    """Raw Philox4x32-10 block (exposed for the generator's known-answer test)."""
    c = (ctypes.c_uint32 * 4)(*ctr)
    k = (ctypes.c_uint32 * 2)(*key)
    o = (ctypes.c_uint32 * 4)()
    lib().fkmgen_philox(c, k, o)
    return [int(v) for v in o]


@dataclass(frozen=True)
class Workload:
    """One synthetic k-means workload (shape, storage dtype and distribution)."""
    name: str
    B: int
    N: int
    D: int
    K: int
    dtype: str
    n_comp: int            # 0: plain N(0, sigma^2 I), no cluster structure
    wkind: int = W_EQUAL
    wparam: float = 0.0
    mean_std: float = 1.0
    sigma: float = 1.0
    iters: int = 10
    tol: float = 0.0
    seed: int = 0
    host_resident: bool = False
    note: str = field(default="", compare=False)

    @property
    def elem_bytes(self) -> int:
        return DTYPE_BYTES[self.dtype]

    @property
    def x_bytes(self) -> int:
        return self.B * self.N * self.D * self.elem_bytes

    def scaled(self, **kw) -> "Workload":
        d = dict(self.__dict__)
        d.update(kw)
        return Workload(**d)


# The five workloads: small fp32 mixture; batched bf16 unbalanced mixture;
# DiT-token-shaped structureless fp16; one large bf16 problem with Zipf-skewed
# (hot) clusters; an out-of-core fp32 problem held in host pinned memory.
CONFIGS = {
    1: Workload("mixture64_f32_B1_N4096_D128_K64", 1, 4096, 128, 64, "f32", 64, W_EQUAL, 0.0,
                4.0, 1.0, 10, 0.0, 20260001),
    2: Workload("dirichlet_bf16_B32_N65536_D128_K1024", 32, 65536, 128, 1024, "bf16", 1024,
                W_DIRICHLET, 0.5, 1.0, 0.5, 10, 0.0, 20260002),
    3: Workload("normal_f16_B32_N75600_D128_K1000", 32, 75600, 128, 1000, "f16", 0, W_EQUAL,
                0.0, 1.0, 1.0, 10, 1e-4, 20260003),
    4: Workload("zipf_bf16_B1_N16777216_D128_K4096", 1, 1 << 24, 128, 4096, "bf16", 4096, W_ZIPF,
                1.1, 1.0, 0.3, 5, 0.0, 20260004),
    5: Workload("mixture_f32_host_B1_N268435456_D64_K16384", 1, 1 << 28, 64, 16384, "f32", 16384,
                W_EQUAL, 0.0, 1.0, 0.5, 3, 0.0, 20260005, host_resident=True),
    # large D (README "Large-D and dtype support" runs d = 2048): the assign
    # kernel streams the point tile with the centroids
    6: Workload("mixture_bf16_B1_N1048576_D2048_K1024", 1, 1 << 20, 2048, 1024, "bf16", 1024,
                W_EQUAL, 0.0, 1.0, 0.5, 10, 0.0, 20260006),
    # the README's "d=2048, k=1024, fp32" shape: split-bf16 operands, streamed
    7: Workload("mixture_f32_B1_N262144_D2048_K1024", 1, 1 << 18, 2048, 1024, "f32", 1024,
                W_EQUAL, 0.0, 1.0, 0.5, 10, 0.0, 20260007),
}


def fill_points(w: Workload, b: int, ptr: int, n_rows: int | None = None,
                labels_ptr: int | None = None) -> None:
    """Write batch b's points ([N, D] in w.dtype) to the raw host address ptr."""
    n = w.N if n_rows is None else n_rows
    rc = lib().fkmgen_points(n, w.D, DTYPE_CODE[w.dtype], w.seed, b, w.n_comp, w.wkind,
                             w.wparam, w.mean_std, w.sigma, ctypes.c_void_p(ptr),
                             ctypes.c_void_p(labels_ptr or 0))
    if rc != 0:
        raise RuntimeError("fkmgen_points failed")


def points(w: Workload, with_labels: bool = False):
    """Points [B, N, D] as a numpy array in storage form (bf16 as uint16 bits)."""
    x = np.empty((w.B, w.N, w.D), dtype=NP_STORAGE[w.dtype])
    lab = np.empty((w.B, w.N), dtype=np.int32) if with_labels else None
    for b in range(w.B):
        fill_points(w, b, x[b].ctypes.data, None, lab[b].ctypes.data if with_labels else None)
    return (x, lab) if with_labels else x


def init_indices(w: Workload) -> np.ndarray:
    """Per batch, the first K entries of a seeded permutation of [0, N): [B, K] int64."""
    out = np.empty((w.B, w.K), dtype=np.int64)
    for b in range(w.B):
        rc = lib().fkmgen_perm_prefix(w.N, w.K, w.seed, b, out[b].ctypes.data)
        if rc != 0:
            raise RuntimeError("fkmgen_perm_prefix failed")
    return out


def widen(x: np.ndarray, dtype: str) -> np.ndarray:
    """Exact widening of stored values to float32 (bf16 bits -> f32 by a 16-bit shift)."""
    if dtype == "bf16":
        return (x.astype(np.uint32) << 16).view(np.float32)
    return x.astype(np.float32)


def init_centroids(x: np.ndarray, idx: np.ndarray, dtype: str) -> np.ndarray:
    """Initial centroids [B, K, D] float32: the points picked by idx (exact in every dtype)."""
    B = x.shape[0]
    return np.stack([widen(x[b][idx[b]], dtype) for b in range(B)], axis=0)
