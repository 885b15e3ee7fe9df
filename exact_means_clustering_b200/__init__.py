"""exact_means_clustering_b200 -- exact batched Lloyd k-means on NVIDIA B200.

A thin ctypes binding over ``libfkm.so`` (C ABI in ``include/fkm.h``).  Every
step of an iteration runs in the library's sm_100a kernels; this module only
marshals torch tensors (device memory, streams) into pointers and sizes.  If
the shared library is missing or a call fails, it raises: there is no
fallback implementation.

Functions named ``fkm_*`` mirror the C entry points one to one.  The
convenience wrapper ``batch_kmeans_Euclid`` follows the call shape the
Flash-KMeans README shows ("Usage": ``cluster_ids, centers, _ =
batch_kmeans_Euclid(x, n_clusters, max_iters, tol)``); its third value is the
number of iterations run.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# FKM_LIB_VARIANT=checked loads the checked build (kernels verify their
# gather / scatter indices and report an out-of-range one in the status word)
LIB_PATH = os.path.join(_HERE, "libfkm_checked.so" if os.environ.get("FKM_LIB_VARIANT") ==
                        "checked" else "libfkm.so")

FKM_OK = 0
STATUS_NAMES = {0: "FKM_OK", 1: "FKM_ERR_INVALID_ARG", 2: "FKM_ERR_UNSUPPORTED",
                3: "FKM_ERR_CUDA", 4: "FKM_ERR_WORKSPACE_TOO_SMALL", 5: "FKM_ERR_TIMEOUT",
                6: "FKM_ERR_INTERNAL", 7: "FKM_ERR_BAD_ID"}
DTYPES = {torch.float32: 0, torch.float16: 1, torch.bfloat16: 2}
METRICS = {"euclid": 0, "dot": 1, "cosine": 2}

# every entry point of include/fkm.h: name -> (argtypes, restype)
_P, _I, _L, _Z, _F = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t, ctypes.c_float
_SIG = {
    "fkm_workspace_size": ([_I, _I, _I, _I, _I, ctypes.POINTER(_Z)], _I),
    "fkm_selftest_wait_timeout": ([ctypes.c_uint64, _P, _Z, _P], _I),
    "fkm_centre_workspace_size": ([_I, _I, _I, ctypes.POINTER(_Z)], _I),
    "fkm_partial_update": ([_I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _Z, _P], _I),
    "fkm_finalize_sums": ([_I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _Z, _P], _I),
    "fkm_partial_update_host": ([_I, _I, _I, _I, _I, _P, _P, _L, _P, _P, _P, _P, _I, _P, _Z,
                                 _P], _I),
    "fkm_centre": ([_I, _I, _I, _I, _P, _P, _P, _P, _Z, _P], _I),
    "fkm_shift_centroids": ([_I, _I, _I, _P, _P, _I, _P, _P], _I),
    "fkm_assign": ([_I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _Z, _P], _I),
    "fkm_update": ([_I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _P, _Z, _P], _I),
    "fkm_lloyd": ([_I, _I, _I, _I, _I, _P, _P, _I, _F, _P, _P, _P, _P, ctypes.POINTER(_I), _P, _Z,
                   _P], _I),
    "fkm_assign_metric": ([_I, _I, _I, _I, _I, _I, _P, _P, _P, _P, _Z, _P], _I),
    "fkm_update_metric": ([_I, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _P, _Z, _P], _I),
    "fkm_lloyd_metric": ([_I, _I, _I, _I, _I, _I, _P, _P, _I, _F, _P, _P, _P, _P,
                          ctypes.POINTER(_I), _P, _Z, _P], _I),
    "fkm_host_workspace_size": ([_I, _I, _I, _I, _I, _L, ctypes.POINTER(_Z)], _I),
    "fkm_lloyd_host": ([_I, _I, _I, _I, _I, _P, _P, _I, _F, _L, _P, _P, _P, _P,
                        ctypes.POINTER(_I), _P, _Z, _P], _I),
    "fkm_lloyd_host_metric": ([_I, _I, _I, _I, _I, _I, _P, _P, _I, _F, _L, _P, _P, _P, _P,
                               ctypes.POINTER(_I), _P, _Z, _P], _I),
    "fkm_argsort_workspace_size": ([_L, _I, ctypes.POINTER(_Z)], _I),
    "fkm_argsort": ([_P, _L, _I, _P, _P, _P, _Z, _P], _I),
    "fkm_baseline_assign": ([_I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _Z, _P], _I),
    "fkm_baseline_update": ([_I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _Z, _P], _I),
    "fkm_assign_noalloc": ([_I, _I, _I, _I, _I, _P, _P, _P, _P], _I),
    "fkm_assign_noalloc_status": ([_P], _I),
    "fkm_sync_status": ([_P, _Z, _P], _I),
    "fkm_segsum_stats": ([_P, _Z, _L, _I, ctypes.POINTER(ctypes.c_ulonglong),
                          ctypes.POINTER(_I), _P], _I),
    "fkm_profile": ([_I], _I),
    "fkm_set_verbose": ([_I], _I),
    "fkm_profile_read": ([_P, ctypes.POINTER(ctypes.c_longlong), _I], _I),
    "fkm_kernel_launches": ([], ctypes.c_longlong),
    "fkm_status_string": ([_I], ctypes.c_char_p),
    "fkm_last_error": ([], ctypes.c_char_p),
    "fkm_version": ([], ctypes.c_char_p),
}

_lib = None


class FkmError(RuntimeError):
    def __init__(self, fn, code, detail):
        self.code = code
        super().__init__(f"{fn} failed: {STATUS_NAMES.get(code, code)}: {detail}")


def lib() -> ctypes.CDLL:
    """Load libfkm.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m exact_means_clustering_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (args, res) in _SIG.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = res
        _lib = L
    return _lib


def _check(fn, code):
    if code != FKM_OK:
        raise FkmError(fn, code, lib().fkm_last_error().decode(errors="replace"))


def _ptr(t, dtype=None):
    """Address of a tensor's data for the C calls, which read every array as
    dense row-major memory of a fixed type: a strided view or a wrong dtype
    would be misread, so both are refused here.  Raw integer addresses and
    None (an optional argument left out) pass through."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_contiguous():
        raise ValueError(f"a {tuple(t.shape)} tensor passed to the library is not contiguous "
                         "(call .contiguous())")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"expected a {dtype} tensor, got {t.dtype}")
    return t.data_ptr()


class _Args:
    """Argument checks of one call, made before the C call: every tensor must
    hold exactly the elements its role needs (the C side trusts the sizes it
    derives from B, N, K, D) and sit on the call's CUDA device (the stream's,
    else that of the first device tensor given, else the current one); only
    the host-streamed calls take their points from (pinned) host memory.
    Contiguity, dtype and size are checked as each argument is marshalled;
    a device mismatch is raised by done() (ws() calls it), after every
    argument has passed those."""

    def __init__(self, fn, stream=None, *tensors):
        self.fn = fn
        self.pending = None
        self.device = None
        if stream is not None and not isinstance(stream, int):
            self.device = stream.device
        else:
            for t in tensors:
                if torch.is_tensor(t) and t.is_cuda:
                    self.device = t.device
                    break

    def _count(self, name, t, shape):
        want = 1
        for n in shape:
            want *= int(n)
        if t.numel() != want:
            raise ValueError(f"{self.fn}: {name} has shape {tuple(t.shape)}, expected "
                             f"{tuple(int(n) for n in shape)}")

    def dev(self, name, t, shape, dtype=None):
        """Pointer of a device tensor of `shape` (None and raw addresses pass)."""
        if t is None or isinstance(t, int):
            return t
        p = _ptr(t, dtype)
        self._count(name, t, shape)
        if not t.is_cuda:
            self.pending = self.pending or f"{name} must be a CUDA tensor, got one on {t.device}"
        elif self.device is None:
            self.device = t.device
        elif t.device != self.device:
            self.pending = self.pending or (f"{name} is on {t.device}, the call runs on "
                                            f"{self.device}")
        return p

    def done(self):
        if self.pending:
            raise ValueError(f"{self.fn}: {self.pending}")

    def ws(self, t):
        """Pointer and size of a workspace tensor on the call's device."""
        self.done()
        if not t.is_cuda:
            raise ValueError(f"{self.fn}: the workspace must be a CUDA tensor")
        if self.device is not None and t.device != self.device:
            raise ValueError(f"{self.fn}: the workspace is on {t.device}, the call runs on "
                             f"{self.device}")
        return _ptr(t), t.numel() * t.element_size()

    def host(self, name, t, shape, dtype=None):
        """Pointer of a host tensor of `shape` (raw addresses pass)."""
        if isinstance(t, int):
            return t
        p = _ptr(t, dtype)
        self._count(name, t, shape)
        if t.is_cuda:
            raise ValueError(f"{self.fn}: {name} must be in (pinned) host memory")
        return p


def _dims(fn, t, n, what):
    if t.dim() != n:
        raise ValueError(f"{fn}: {what} must be {n}-D, got shape {tuple(t.shape)}")
    return tuple(t.shape)


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _dt(x):
    if isinstance(x, int):
        return x
    try:
        return DTYPES[x if isinstance(x, torch.dtype) else x.dtype]
    except KeyError as e:
        raise TypeError(f"unsupported point dtype {x}") from e


# ---------------------------------------------------------------- C mirrors
def fkm_workspace_size(B, N, K, D, dtype) -> int:
    out = ctypes.c_size_t(0)
    _check("fkm_workspace_size", lib().fkm_workspace_size(B, N, K, D, _dt(dtype), ctypes.byref(out)))
    return out.value


def fkm_host_workspace_size(B, N, K, D, dtype, chunk_rows) -> int:
    out = ctypes.c_size_t(0)
    _check("fkm_host_workspace_size",
           lib().fkm_host_workspace_size(B, N, K, D, _dt(dtype), chunk_rows, ctypes.byref(out)))
    return out.value


def fkm_argsort_workspace_size(n, n_keys) -> int:
    out = ctypes.c_size_t(0)
    _check("fkm_argsort_workspace_size",
           lib().fkm_argsort_workspace_size(n, n_keys, ctypes.byref(out)))
    return out.value


def workspace(nbytes, device=None) -> torch.Tensor:
    """A zero-filled device workspace (the library expects zeros on first use)."""
    return torch.zeros(max(int(nbytes), 256), dtype=torch.uint8, device=device or "cuda")


def _ws(ws, nbytes, device):
    return ws if ws is not None else workspace(nbytes, device)


def fkm_assign(x, centers, ids, inertia=None, ws=None, stream=None):
    f = "fkm_assign"
    B, N, D = _dims(f, x, 3, "x")
    K = _dims(f, centers, 3, "centers")[1]
    A = _Args(f, stream, x)
    args = (A.dev("x", x, (B, N, D)), A.dev("centers", centers, (B, K, D), torch.float32),
            A.dev("ids", ids, (B, N), torch.int32), A.dev("inertia", inertia, (B,), torch.float64))
    wp, wn = A.ws(_ws(ws, fkm_workspace_size(B, N, K, D, x.dtype), x.device))
    _check(f, lib().fkm_assign(B, N, K, D, _dt(x), *args, wp, wn, _stream(stream)))


def fkm_update(x, ids, prev_centers, centers, counts, shift=None, inertia=None, ws=None,
               stream=None):
    f = "fkm_update"
    B, N, D = _dims(f, x, 3, "x")
    K = _dims(f, prev_centers, 3, "prev_centers")[1]
    A = _Args(f, stream, x)
    args = (A.dev("x", x, (B, N, D)), A.dev("ids", ids, (B, N), torch.int32),
            A.dev("prev_centers", prev_centers, (B, K, D), torch.float32),
            A.dev("centers", centers, (B, K, D), torch.float32),
            A.dev("counts", counts, (B, K), torch.int32),
            A.dev("shift", shift, (B,), torch.float64),
            A.dev("inertia", inertia, (B,), torch.float64))
    wp, wn = A.ws(_ws(ws, fkm_workspace_size(B, N, K, D, x.dtype), x.device))
    _check(f, lib().fkm_update(B, N, K, D, _dt(x), *args, wp, wn, _stream(stream)))


def fkm_lloyd(x, init_centers, max_iters, tol, ids, centers, counts, inertia=None, ws=None,
              stream=None) -> int:
    f = "fkm_lloyd"
    B, N, D = _dims(f, x, 3, "x")
    K = _dims(f, init_centers, 3, "init_centers")[1]
    A = _Args(f, stream, x)
    px = A.dev("x", x, (B, N, D))
    pi = A.dev("init_centers", init_centers, (B, K, D), torch.float32)
    outs = (A.dev("ids", ids, (B, N), torch.int32),
            A.dev("centers", centers, (B, K, D), torch.float32),
            A.dev("counts", counts, (B, K), torch.int32),
            A.dev("inertia", inertia, (B,), torch.float64))
    wp, wn = A.ws(_ws(ws, fkm_workspace_size(B, N, K, D, x.dtype), x.device))
    n_iter = ctypes.c_int(0)
    _check(f, lib().fkm_lloyd(B, N, K, D, _dt(x), px, pi, max_iters, float(tol), *outs,
                              ctypes.byref(n_iter), wp, wn, _stream(stream)))
    return n_iter.value


def _metric(metric) -> int:
    if isinstance(metric, str):
        return METRICS[metric]
    return int(metric)


def fkm_assign_metric(x, centers, ids, metric, ws=None, stream=None):
    """ids = the most similar centroid under metric ('euclid', 'dot', 'cosine')."""
    f = "fkm_assign_metric"
    B, N, D = _dims(f, x, 3, "x")
    K = _dims(f, centers, 3, "centers")[1]
    A = _Args(f, stream, x)
    args = (A.dev("x", x, (B, N, D)), A.dev("centers", centers, (B, K, D), torch.float32),
            A.dev("ids", ids, (B, N), torch.int32))
    wp, wn = A.ws(_ws(ws, fkm_workspace_size(B, N, K, D, x.dtype), x.device))
    _check(f, lib().fkm_assign_metric(B, N, K, D, _dt(x), _metric(metric), *args, wp, wn,
                                      _stream(stream)))


def fkm_update_metric(x, ids, prev_centers, centers, counts, metric, shift=None, objective=None,
                      ws=None, stream=None):
    f = "fkm_update_metric"
    B, N, D = _dims(f, x, 3, "x")
    K = _dims(f, prev_centers, 3, "prev_centers")[1]
    A = _Args(f, stream, x)
    args = (A.dev("x", x, (B, N, D)), A.dev("ids", ids, (B, N), torch.int32),
            A.dev("prev_centers", prev_centers, (B, K, D), torch.float32),
            A.dev("centers", centers, (B, K, D), torch.float32),
            A.dev("counts", counts, (B, K), torch.int32),
            A.dev("shift", shift, (B,), torch.float64),
            A.dev("objective", objective, (B,), torch.float64))
    wp, wn = A.ws(_ws(ws, fkm_workspace_size(B, N, K, D, x.dtype), x.device))
    _check(f, lib().fkm_update_metric(B, N, K, D, _dt(x), _metric(metric), *args, wp, wn,
                                      _stream(stream)))


def fkm_lloyd_metric(x, init_centers, max_iters, tol, ids, centers, counts, metric,
                     objective=None, ws=None, stream=None) -> int:
    f = "fkm_lloyd_metric"
    B, N, D = _dims(f, x, 3, "x")
    K = _dims(f, init_centers, 3, "init_centers")[1]
    A = _Args(f, stream, x)
    px = A.dev("x", x, (B, N, D))
    pi = A.dev("init_centers", init_centers, (B, K, D), torch.float32)
    outs = (A.dev("ids", ids, (B, N), torch.int32),
            A.dev("centers", centers, (B, K, D), torch.float32),
            A.dev("counts", counts, (B, K), torch.int32),
            A.dev("objective", objective, (B,), torch.float64))
    wp, wn = A.ws(_ws(ws, fkm_workspace_size(B, N, K, D, x.dtype), x.device))
    n_iter = ctypes.c_int(0)
    _check(f, lib().fkm_lloyd_metric(B, N, K, D, _dt(x), _metric(metric), px, pi, max_iters,
                                     float(tol), *outs, ctypes.byref(n_iter), wp, wn,
                                     _stream(stream)))
    return n_iter.value


def fkm_lloyd_host(x_host, init_centers, max_iters, tol, chunk_rows, ids, centers, counts,
                   inertia=None, ws=None, stream=None, dtype=None, shape=None) -> int:
    """x_host: a pinned CPU tensor [B, N, D] (or a raw address with dtype and shape)."""
    f = "fkm_lloyd_host"
    if isinstance(x_host, int):
        B, N, D = shape
        dt = _dt(dtype)
    else:
        B, N, D = _dims(f, x_host, 3, "x_host")
        dt = _dt(x_host)
    K = _dims(f, init_centers, 3, "init_centers")[1]
    A = _Args(f, stream, init_centers)
    px = A.host("x_host", x_host, (B, N, D))
    pi = A.dev("init_centers", init_centers, (B, K, D), torch.float32)
    outs = (A.dev("ids", ids, (B, N), torch.int32),
            A.dev("centers", centers, (B, K, D), torch.float32),
            A.dev("counts", counts, (B, K), torch.int32),
            A.dev("inertia", inertia, (B,), torch.float64))
    wp, wn = A.ws(_ws(ws, fkm_host_workspace_size(B, N, K, D, dt, chunk_rows),
                      init_centers.device))
    n_iter = ctypes.c_int(0)
    _check(f, lib().fkm_lloyd_host(B, N, K, D, dt, px, pi, max_iters, float(tol),
                                   int(chunk_rows), *outs, ctypes.byref(n_iter), wp, wn,
                                   _stream(stream)))
    return n_iter.value


def fkm_lloyd_host_metric(x_host, init_centers, max_iters, tol, chunk_rows, ids, centers,
                          counts, metric, objective=None, ws=None, stream=None) -> int:
    """fkm_lloyd_host under metric ('euclid', 'dot', 'cosine'); x_host: a pinned
    CPU tensor [B, N, D]."""
    f = "fkm_lloyd_host_metric"
    B, N, D = _dims(f, x_host, 3, "x_host")
    dt = _dt(x_host)
    K = _dims(f, init_centers, 3, "init_centers")[1]
    A = _Args(f, stream, init_centers)
    px = A.host("x_host", x_host, (B, N, D))
    pi = A.dev("init_centers", init_centers, (B, K, D), torch.float32)
    outs = (A.dev("ids", ids, (B, N), torch.int32),
            A.dev("centers", centers, (B, K, D), torch.float32),
            A.dev("counts", counts, (B, K), torch.int32),
            A.dev("objective", objective, (B,), torch.float64))
    wp, wn = A.ws(_ws(ws, fkm_host_workspace_size(B, N, K, D, dt, chunk_rows),
                      init_centers.device))
    n_iter = ctypes.c_int(0)
    _check(f, lib().fkm_lloyd_host_metric(B, N, K, D, dt, _metric(metric), px, pi, max_iters,
                                          float(tol), int(chunk_rows), *outs,
                                          ctypes.byref(n_iter), wp, wn, _stream(stream)))
    return n_iter.value


def fkm_argsort(keys, n_keys, idx, sorted_keys=None, ws=None, stream=None):
    f = "fkm_argsort"
    n = keys.numel()
    A = _Args(f, stream, keys)
    args = (A.dev("keys", keys, (n,), torch.int32), n, n_keys,
            A.dev("idx", idx, (n,), torch.int32),
            A.dev("sorted_keys", sorted_keys, (n,), torch.int32))
    wp, wn = A.ws(_ws(ws, fkm_argsort_workspace_size(n, n_keys), keys.device))
    _check(f, lib().fkm_argsort(*args, wp, wn, _stream(stream)))


def fkm_baseline_assign(x, centers, dist, ids, ws=None, stream=None):
    f = "fkm_baseline_assign"
    B, N, D = _dims(f, x, 3, "x")
    K = _dims(f, centers, 3, "centers")[1]
    A = _Args(f, stream, x)
    args = (A.dev("x", x, (B, N, D)), A.dev("centers", centers, (B, K, D), torch.float32),
            A.dev("dist", dist, (B, N, K), torch.float32), A.dev("ids", ids, (B, N), torch.int32))
    wp, wn = A.ws(_ws(ws, fkm_workspace_size(B, N, K, D, x.dtype), x.device))
    _check(f, lib().fkm_baseline_assign(B, N, K, D, _dt(x), *args, wp, wn, _stream(stream)))


def fkm_baseline_update(x, ids, prev_centers, centers, counts, ws=None, stream=None):
    f = "fkm_baseline_update"
    B, N, D = _dims(f, x, 3, "x")
    K = _dims(f, prev_centers, 3, "prev_centers")[1]
    A = _Args(f, stream, x)
    args = (A.dev("x", x, (B, N, D)), A.dev("ids", ids, (B, N), torch.int32),
            A.dev("prev_centers", prev_centers, (B, K, D), torch.float32),
            A.dev("centers", centers, (B, K, D), torch.float32),
            A.dev("counts", counts, (B, K), torch.int32))
    wp, wn = A.ws(_ws(ws, fkm_workspace_size(B, N, K, D, x.dtype), x.device))
    _check(f, lib().fkm_baseline_update(B, N, K, D, _dt(x), *args, wp, wn, _stream(stream)))


def fkm_assign_noalloc(x, centers, ids, stream=None):
    """fkm_assign without a workspace, for callers that cannot allocate device
    memory: its scratch is a static 16 MiB device array inside the library
    (bf16/fp16 points only; calls that overlap on the GPU race)."""
    f = "fkm_assign_noalloc"
    B, N, D = _dims(f, x, 3, "x")
    K = _dims(f, centers, 3, "centers")[1]
    A = _Args(f, stream, x)
    args = (A.dev("x", x, (B, N, D)), A.dev("centers", centers, (B, K, D), torch.float32),
            A.dev("ids", ids, (B, N), torch.int32))
    A.done()
    _check(f, lib().fkm_assign_noalloc(B, N, K, D, _dt(x), *args, _stream(stream)))


def fkm_assign_noalloc_status(stream=None):
    """Wait for the stream, then read and clear the status word of the
    fkm_assign_noalloc calls on the current device (raises FkmError with
    FKM_ERR_TIMEOUT if a device-side bounded wait ran out)."""
    _check("fkm_assign_noalloc_status", lib().fkm_assign_noalloc_status(_stream(stream)))


def fkm_partial_update(x, ids, prev, sums, counts, obj=None, ws=None, stream=None):
    """Add one shard's per-cluster sums / counts (and objective) to sums [B, K, D],
    counts [B, K] (and obj [B]), all float64; see fkm.h."""
    f = "fkm_partial_update"
    B, N, D = _dims(f, x, 3, "x")
    K = _dims(f, prev, 3, "prev")[1]
    A = _Args(f, stream, x)
    args = (A.dev("x", x, (B, N, D)), A.dev("ids", ids, (B, N), torch.int32),
            A.dev("prev", prev, (B, K, D), torch.float32),
            A.dev("sums", sums, (B, K, D), torch.float64),
            A.dev("counts", counts, (B, K), torch.float64),
            A.dev("obj", obj, (B,), torch.float64))
    wp, wn = A.ws(_ws(ws, fkm_workspace_size(B, N, K, D, x.dtype), x.device))
    _check(f, lib().fkm_partial_update(B, N, K, D, _dt(x), *args, wp, wn, _stream(stream)))


FKM_HOST_COPY_AT_ONCE = 1


def fkm_partial_update_host(x_host, centers, chunk_rows, ids, sums, counts, obj=None, ws=None,
                            stream=None, copy_at_once=False):
    """fkm_partial_update for a shard in pinned host memory x_host [B, N, D],
    streamed in chunks of chunk_rows points; also writes the shard's ids.
    copy_at_once: the workspace's chunk buffers are idle (an earlier call on
    it returned), so the first copy need not wait for the stream (fkm.h)."""
    f = "fkm_partial_update_host"
    B, N, D = _dims(f, x_host, 3, "x_host")
    K = _dims(f, centers, 3, "centers")[1]
    A = _Args(f, stream, centers)
    px = A.host("x_host", x_host, (B, N, D))
    args = (A.dev("centers", centers, (B, K, D), torch.float32), int(chunk_rows),
            A.dev("ids", ids, (B, N), torch.int32),
            A.dev("sums", sums, (B, K, D), torch.float64),
            A.dev("counts", counts, (B, K), torch.float64),
            A.dev("obj", obj, (B,), torch.float64),
            FKM_HOST_COPY_AT_ONCE if copy_at_once else 0)
    wp, wn = A.ws(_ws(ws, fkm_host_workspace_size(B, N, K, D, _dt(x_host), chunk_rows),
                      centers.device))
    _check(f, lib().fkm_partial_update_host(B, N, K, D, _dt(x_host), px, *args, wp, wn,
                                            _stream(stream)))


def fkm_finalize_sums(sums, counts, prev, centers, shift=None, ws=None, stream=None,
                      counts_out=None):
    """centers = sums / counts (prev where a cluster is empty; sums and counts
    float64); shift [B] and counts_out [B, K] int32 optional."""
    f = "fkm_finalize_sums"
    B, K, D = _dims(f, prev, 3, "prev")
    A = _Args(f, stream, prev)
    args = (A.dev("sums", sums, (B, K, D), torch.float64),
            A.dev("counts", counts, (B, K), torch.float64),
            A.dev("prev", prev, (B, K, D), torch.float32),
            A.dev("centers", centers, (B, K, D), torch.float32),
            A.dev("counts_out", counts_out, (B, K), torch.int32),
            A.dev("shift", shift, (B,), torch.float64))
    wp, wn = A.ws(_ws(ws, 256 + 8 * B * K, prev.device))
    _check(f, lib().fkm_finalize_sums(B, K, D, *args, wp, wn, _stream(stream)))


def reduce_partials(tensors, group=None):
    """Sum the shards' partials over the ranks of a torch.distributed group
    (NCCL over NVLink for CUDA tensors): one all-reduce per tensor given --
    the sharded loop gives one packed buffer.  A no-op without an
    initialised group of 2+ ranks."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size(group) < 2:
        return
    for t in tensors:
        dist.all_reduce(t, op=dist.ReduceOp.SUM, group=group)


def partial_buffers(B, K, D, device):
    """One float64 buffer holding a shard's partials, and its views (sums
    [B, K, D], counts [B, K], obj [B]); each view starts 16-byte aligned.
    Reducing the buffer reduces all three with one collective."""
    def up2(n):
        return n + (n & 1)
    o1 = up2(B * K * D)
    o2 = o1 + up2(B * K)
    buf = torch.zeros(o2 + up2(B), dtype=torch.float64, device=device)
    return (buf, buf[:B * K * D].view(B, K, D), buf[o1:o1 + B * K].view(B, K),
            buf[o2:o2 + B])


def lloyd_sharded(x, init_centers, max_iters, tol=0.0, group=None, ws=None, chunk_rows=None):
    """Data-parallel Lloyd k-means over the ranks of a torch.distributed group
    (README "Multi-GPU Support"): every rank passes its own contiguous shard
    x [B, N_r, D] of the same B problems and the same init_centers [B, K, D];
    per iteration each rank assigns its shard, forms its partial sums and
    counts, the partials are all-reduced (one packed buffer, one
    collective), and every rank forms the same centroids.  A shard in pinned
    host memory (x on the CPU) is streamed to init_centers' device in chunks
    of chunk_rows points every iteration, as fkm_lloyd_host does.  Returns
    (ids of this shard [B, N_r], centers [B, K, D], counts [B, K] int32 of
    all shards, inertia [B] of all shards, n_iter)."""
    B, N, D = x.shape
    K = init_centers.shape[1]
    on_host = not x.is_cuda
    dev = init_centers.device if on_host else x.device
    if dev.type != "cuda":
        raise ValueError("lloyd_sharded: init_centers must be on the GPU when x is on the host")
    if on_host:
        chunk_rows = int(chunk_rows or min(N, 1 << 20))
        if ws is None:
            ws = workspace(fkm_host_workspace_size(B, N, K, D, _dt(x), chunk_rows), dev)
    elif ws is None:
        ws = workspace(fkm_workspace_size(B, N, K, D, x.dtype), dev)
    c = init_centers.to(dev, torch.float32).contiguous().clone()
    ids = torch.empty(B, N, dtype=torch.int32, device=dev)
    calls = [0]

    def partials(c, sums, counts, obj):
        if on_host:
            # after the first call the chunk buffers are idle, so the next
            # iteration's first copy overlaps this iteration's all-reduce
            fkm_partial_update_host(x, c, chunk_rows, ids, sums, counts, obj, ws=ws,
                                    copy_at_once=calls[0] > 0)
            calls[0] += 1
        else:
            fkm_assign(x, c, ids, ws=ws)
            fkm_partial_update(x, ids, c, sums, counts, obj, ws=ws)

    def finalize(sums, counts, c, nxt, shift, counts_out):
        fkm_finalize_sums(sums, counts, c, nxt, shift, ws=ws, counts_out=counts_out)

    c, counts, obj, n_iter = sharded_loop(partials, finalize, c, max_iters, tol, group)
    fkm_sync_status(ws)
    return ids, c, counts, obj, n_iter


def _group_size(group=None):
    """Ranks of an initialised torch.distributed group (1 without one)."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return 1
    return dist.get_world_size(group)


def shard_rows(N, rank, world):
    """Contiguous rows [r0, r1) of N that rank `rank` of `world` holds: the
    first N % world ranks take one row more."""
    q, r = divmod(int(N), int(world))
    r0 = rank * q + min(rank, r)
    return r0, r0 + q + (1 if rank < r else 0)


def gather_shard_ids(ids, N, group=None):
    """All ranks' shard labels [B, N_r] put back in row order, [B, N] on every
    rank (shards from shard_rows; one all_gather of equal-size padded
    blocks)."""
    import torch.distributed as dist
    world = _group_size(group)
    if world < 2:
        return ids
    B = ids.shape[0]
    width = shard_rows(N, 0, world)[1]
    pad = torch.full((B, width), -1, dtype=ids.dtype, device=ids.device)
    pad[:, :ids.shape[1]] = ids
    parts = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(parts, pad, group=group)
    out = torch.empty(B, N, dtype=ids.dtype, device=ids.device)
    for r, part in enumerate(parts):
        r0, r1 = shard_rows(N, r, world)
        out[:, r0:r1] = part[:, :r1 - r0]
    return out


def sharded_loop(partials, finalize, c, max_iters, tol=0.0, group=None):
    """The rank-side control of the data-parallel loop, independent of where
    the shard lives: per iteration partials(c, sums, counts, obj) adds this
    rank's shard into the zeroed float64 views sums [B, K, D], counts [B, K]
    and obj [B] of one packed buffer; reduce_partials sums that buffer over
    the group with one all-reduce; finalize(sums, counts, c, nxt, shift,
    counts_out) forms the next centroids, the shift [B] and the int32 counts.
    The stop test (max shift < tol) reads reduced values only, so every rank
    takes the same number of iterations and the same collectives.  Returns
    (centers, counts [B, K] int32 and objective [B] of all shards, n_iter)."""
    B, K, D = c.shape
    dev = c.device
    buf, sums, counts, obj = partial_buffers(B, K, D, dev)
    counts_out = torch.empty(B, K, dtype=torch.int32, device=dev)
    shift = torch.empty(B, dtype=torch.float64, device=dev)
    n_iter = 0
    for t in range(max_iters):
        buf.zero_()
        partials(c, sums, counts, obj)
        reduce_partials((buf,), group)
        nxt = torch.empty_like(c)
        finalize(sums, counts, c, nxt, shift, counts_out)
        c = nxt
        n_iter = t + 1
        if tol > 0.0 and shift.max().item() < tol:
            break
    return c, counts_out, obj, n_iter


def fkm_centre_workspace_size_bytes(B, N, D) -> int:
    n = ctypes.c_size_t(0)
    _check("fkm_centre_workspace_size", lib().fkm_centre_workspace_size(B, N, D, ctypes.byref(n)))
    return n.value


def fkm_centre(x, mu=None, out=None, ws=None, stream=None):
    """Per-batch mean of x [B, N, D] and x minus it, rounded to x's dtype (see
    fkm.h).  out may be x itself.  Returns (out, mu float32 [B, D])."""
    f = "fkm_centre"
    B, N, D = _dims(f, x, 3, "x")
    mu = mu if mu is not None else torch.empty(B, D, dtype=torch.float32, device=x.device)
    out = out if out is not None else torch.empty_like(x)
    A = _Args(f, stream, x)
    args = (A.dev("x", x, (B, N, D)), A.dev("mu", mu, (B, D), torch.float32),
            A.dev("out", out, (B, N, D), x.dtype))
    wp, wn = A.ws(_ws(ws, fkm_centre_workspace_size_bytes(B, N, D), x.device))
    _check(f, lib().fkm_centre(B, N, D, _dt(x), *args, wp, wn, _stream(stream)))
    return out, mu


def fkm_shift_centroids(centers, mu, sign, out=None, stream=None):
    """out = centers + sign * mu per batch (fp32, sign +1 or -1; out may be
    centers): the centroid side of centring.  Returns out."""
    f = "fkm_shift_centroids"
    B, K, D = _dims(f, centers, 3, "centers")
    out = out if out is not None else torch.empty_like(centers)
    A = _Args(f, stream, centers)
    args = (A.dev("centers", centers, (B, K, D), torch.float32),
            A.dev("mu", mu, (B, D), torch.float32), int(sign),
            A.dev("out", out, (B, K, D), torch.float32))
    A.done()
    _check(f, lib().fkm_shift_centroids(B, K, D, *args, _stream(stream)))
    return out


def fkm_selftest_wait_timeout(timeout_ns, ws, stream=None):
    """Launch a kernel whose bounded wait runs out after timeout_ns (see fkm.h)."""
    A = _Args("fkm_selftest_wait_timeout", stream, ws)
    wp, wn = A.ws(ws)
    _check("fkm_selftest_wait_timeout",
           lib().fkm_selftest_wait_timeout(int(timeout_ns), wp, wn, _stream(stream)))


def fkm_segsum_stats(ws, n_rows, reset=False, stream=None):
    """(fp64 element atomics the segment sums made into ws's cluster sums since
    the last reset, sorted rows per segment-sum range for n_rows points)."""
    A = _Args("fkm_segsum_stats", stream, ws)
    wp, wn = A.ws(ws)
    cnt = ctypes.c_ulonglong(0)
    rng = ctypes.c_int(0)
    _check("fkm_segsum_stats", lib().fkm_segsum_stats(wp, wn, int(n_rows), 1 if reset else 0,
                                                      ctypes.byref(cnt), ctypes.byref(rng),
                                                      _stream(stream)))
    return cnt.value, rng.value


def fkm_sync_status(ws, stream=None):
    A = _Args("fkm_sync_status", stream, ws)
    wp, wn = A.ws(ws)
    _check("fkm_sync_status", lib().fkm_sync_status(wp, wn, _stream(stream)))


def fkm_set_verbose(level) -> None:
    """Per-iteration progress lines of fkm_lloyd on stderr (level > 0)."""
    _check("fkm_set_verbose", lib().fkm_set_verbose(int(level)))


def fkm_profile(enable: bool) -> None:
    _check("fkm_profile", lib().fkm_profile(1 if enable else 0))


STAGES = ("assign", "argsort", "segsum", "finalize", "iteration")


def fkm_profile_read(reset: bool = False) -> dict:
    """Accumulated stage milliseconds of profiled fkm_lloyd calls, and iterations."""
    ms = (ctypes.c_double * 5)()
    it = ctypes.c_longlong(0)
    _check("fkm_profile_read", lib().fkm_profile_read(ms, ctypes.byref(it), 1 if reset else 0))
    out = {s: ms[i] for i, s in enumerate(STAGES)}
    out["iterations"] = it.value
    return out


def fkm_kernel_launches() -> int:
    return int(lib().fkm_kernel_launches())


def fkm_version() -> str:
    return lib().fkm_version().decode()


# ---------------------------------------------------------------- wrapper
def batch_kmeans(x: torch.Tensor, n_clusters: int, max_iters: int = 100, tol: float = 0.0,
                 init_centroids: torch.Tensor | None = None, seed: int = 0,
                 metric: str = "euclid", verbose: bool = False):
    """Exact batched Lloyd k-means under metric 'euclid', 'dot' or 'cosine'
    (fkm.h, fkm_metric).  x: [B, N, D] (or [N, D]) CUDA tensor in float32 /
    float16 / bfloat16.  Returns (cluster_ids int32 [B, N], centers float32
    [B, K, D], n_iter).  Default initial centroids: per batch, the points at
    the first K positions of a seeded random permutation.  verbose prints one
    progress line per iteration (fkm_set_verbose)."""
    squeeze = x.dim() == 2
    if squeeze:
        x = x.unsqueeze(0)
    x = x.contiguous()
    B, N, D = x.shape
    K = int(n_clusters)
    dev = x.device
    if init_centroids is None:
        g = torch.Generator(device="cpu").manual_seed(seed)
        idx = torch.stack([torch.randperm(N, generator=g)[:K] for _ in range(B)]).to(dev)
        init = torch.gather(x, 1, idx.unsqueeze(-1).expand(B, K, D)).float().contiguous()
    else:
        init = init_centroids.reshape(B, K, D).to(device=dev, dtype=torch.float32).contiguous()
    ids = torch.empty(B, N, dtype=torch.int32, device=dev)
    centers = torch.empty(B, K, D, dtype=torch.float32, device=dev)
    counts = torch.empty(B, K, dtype=torch.int32, device=dev)
    if verbose:
        fkm_set_verbose(1)
    try:
        if _metric(metric) == METRICS["euclid"]:
            n_iter = fkm_lloyd(x, init, max_iters, tol, ids, centers, counts)
        else:
            n_iter = fkm_lloyd_metric(x, init, max_iters, tol, ids, centers, counts, metric)
    finally:
        if verbose:
            fkm_set_verbose(0)
    if squeeze:
        return ids[0], centers[0], n_iter
    return ids, centers, n_iter


def batch_kmeans_Euclid(x: torch.Tensor, n_clusters: int, max_iters: int = 100, tol: float = 0.0,
                        init_centroids: torch.Tensor | None = None, seed: int = 0,
                        verbose: bool = False):
    """Exact batched Lloyd k-means (Euclidean), the README's call shape; see
    batch_kmeans."""
    return batch_kmeans(x, n_clusters, max_iters, tol, init_centroids, seed, "euclid", verbose)


# ---------------------------------------------------------------- class API
class FlashKMeans:
    """Exact Lloyd k-means with the class-style calls of the "Flash-KMeans"
    GitHub README (section "Usage"): fit, predict, fit_predict, and train for
    data held in host memory.

    d, k       point dimension and number of clusters
    niter      maximum Lloyd iterations; tol: stop once every batch's squared
               centroid shift is below it (0 runs all niter iterations)
    dtype      storage type the points are clustered in (bf16, fp16 or fp32;
               None keeps the input's)
    centre     subtract the per-batch mean of the points first and add it back
               to the centroids (README, "Centre your data"); costs one extra
               copy of x
    chunk_rows rows per streamed chunk when the points are in host memory

    device     the GPU to run on.  None: the current CUDA device, or, when a
               torch.distributed process group of two or more ranks is
               initialised (one process per GPU, e.g. under torchrun), every
               rank clusters its contiguous shard of the points on its own
               GPU and the ranks combine their partial sums with one
               all-reduce per iteration (README "Multi-GPU Support");
               labels_ then holds every point's label on every rank
    group      the process group for that case (None: the default group)

    Points are [N, D] or [B, N, D] (B independent problems).  After fit:
    centroids [B, K, D] float32 (or [K, D]), labels_ int32 [B, N] (or [N]),
    n_iter, inertia [B] (the objective of the last assignment).
    """

    def __init__(self, d, k, niter=100, tol=0.0, dtype=None, centre=False, seed=0,
                 chunk_rows=1 << 23, device=None, group=None):
        self.d, self.k, self.niter, self.tol = int(d), int(k), int(niter), float(tol)
        self.dtype, self.centre, self.seed = dtype, bool(centre), int(seed)
        self.chunk_rows = int(chunk_rows)
        self.group = group
        self._sharded = device is None and _group_size(group) > 1
        self.device = torch.device(device) if device is not None else torch.device("cuda")
        self.centroids = None
        self.labels_ = None
        self.n_iter = 0
        self.inertia = None
        self._squeeze = False

    def _shape(self, x):
        if x.dim() == 2:
            x = x.unsqueeze(0)
        if x.dim() != 3 or x.shape[-1] != self.d:
            raise ValueError(f"points must be [N, {self.d}] or [B, N, {self.d}], got {tuple(x.shape)}")
        if self.dtype is not None and x.dtype != self.dtype:
            x = x.to(self.dtype)
        return x.contiguous()

    def _init(self, x, init_centroids):
        B, N, D = x.shape
        if init_centroids is not None:
            return init_centroids.reshape(B, self.k, D).to(self.device, torch.float32).contiguous()
        if N < self.k:
            raise ValueError(f"k = {self.k} clusters need at least as many points, got {N}")
        g = torch.Generator(device="cpu").manual_seed(self.seed)
        idx = torch.stack([torch.randperm(N, generator=g)[:self.k] for _ in range(B)])
        rows = torch.gather(x, 1, idx.to(x.device).unsqueeze(-1).expand(B, self.k, D))
        return rows.to(self.device, torch.float32).contiguous()

    def fit(self, x, init_centroids=None):
        self._squeeze = x.dim() == 2
        x = self._shape(x)
        if self._sharded:
            return self._fit_sharded(x, init_centroids)
        if not x.is_cuda:
            return self._fit_host(x, init_centroids)
        B, N, D = x.shape
        mu = None
        if self.centre:
            x, mu = fkm_centre(x)
            if init_centroids is not None:
                c = init_centroids.reshape(B, self.k, D).to(x.device, torch.float32).contiguous()
                init_centroids = fkm_shift_centroids(c, mu, -1)
        init = self._init(x, init_centroids)
        ids = torch.empty(B, N, dtype=torch.int32, device=x.device)
        centers = torch.empty(B, self.k, D, dtype=torch.float32, device=x.device)
        counts = torch.empty(B, self.k, dtype=torch.int32, device=x.device)
        inertia = torch.empty(B, dtype=torch.float64, device=x.device)
        self.n_iter = fkm_lloyd(x, init, self.niter, self.tol, ids, centers, counts, inertia)
        if mu is not None:
            fkm_shift_centroids(centers, mu, +1, out=centers)
        self._store(ids, centers, inertia)
        return self

    def _fit_host(self, x, init_centroids):
        B, N, D = x.shape
        if self.centre:
            raise ValueError("centre=True needs the points on the GPU (one extra device copy)")
        xh = x if x.is_pinned() else x.pin_memory()
        init = self._init(xh, init_centroids)
        ids = torch.empty(B, N, dtype=torch.int32, device=self.device)
        centers = torch.empty(B, self.k, D, dtype=torch.float32, device=self.device)
        counts = torch.empty(B, self.k, dtype=torch.int32, device=self.device)
        inertia = torch.empty(B, dtype=torch.float64, device=self.device)
        self.n_iter = fkm_lloyd_host(xh, init, self.niter, self.tol, self.chunk_rows, ids, centers,
                                     counts, inertia)
        self._store(ids, centers, inertia)
        return self

    def _fit_sharded(self, x, init_centroids):
        """One shard of the points per rank: rows shard_rows(N, rank, world)
        of every problem, in pinned host memory (streamed) when x is on the
        host, else on this rank's GPU."""
        import torch.distributed as dist
        if self.centre:
            raise ValueError("centre=True is not supported with sharded fitting")
        rank, world = dist.get_rank(self.group), dist.get_world_size(self.group)
        dev = torch.device("cuda", torch.cuda.current_device())
        B, N, D = x.shape
        r0, r1 = shard_rows(N, rank, world)
        shard = x[:, r0:r1].contiguous()
        if shard.is_cuda:
            shard = shard.to(dev)
        elif not shard.is_pinned():
            shard = shard.pin_memory()
        init = self._init(x, init_centroids).to(dev)   # the same seed on every rank
        ids, centers, _, inertia, self.n_iter = lloyd_sharded(
            shard, init, self.niter, self.tol, self.group,
            chunk_rows=None if shard.is_cuda else self.chunk_rows)
        self._store(gather_shard_ids(ids, N, self.group), centers, inertia)
        return self

    def _store(self, ids, centers, inertia):
        self.labels_ = ids[0] if self._squeeze else ids
        self.centroids = centers[0] if self._squeeze else centers
        self.inertia = inertia

    def train(self, data, init_centroids=None):
        """fit, under the README's name for training on large data (host
        tensors are streamed to the GPU in chunks)."""
        return self.fit(data, init_centroids)

    def predict(self, x):
        """Nearest-centroid ids of the points x (on the GPU) for the fitted centroids."""
        if self.centroids is None:
            raise RuntimeError("predict before fit")
        squeeze = x.dim() == 2
        x = self._shape(x).to(self.device)
        B, N, D = x.shape
        c = self.centroids.reshape(-1, self.k, D)
        if c.shape[0] != B:
            raise ValueError("predict needs as many batches as fit")
        ids = torch.empty(B, N, dtype=torch.int32, device=x.device)
        fkm_assign(x, c.contiguous(), ids)
        return ids[0] if squeeze else ids

    def fit_predict(self, x, init_centroids=None):
        return self.fit(x, init_centroids).labels_
