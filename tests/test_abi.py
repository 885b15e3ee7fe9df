"""The C ABI library: it builds, loads without a GPU, exports every entry point
include/fkm.h declares, and its host-only paths (sizes, validation, status
strings) behave as documented.  No compute call is made here."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fkm.h")


@pytest.fixture(scope="module")
def fkm():
    from exact_means_clustering_b200 import build
    build.build()
    import exact_means_clustering_b200 as m
    return m


def declared_functions():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"FKM_API\s+[\w\s\*]+?\b(fkm_\w+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("fkm_assign", "fkm_update", "fkm_lloyd", "fkm_lloyd_host",
                     "fkm_workspace_size", "fkm_argsort", "fkm_sync_status", "fkm_last_error"):
        assert required in names


def test_library_exports_every_declared_symbol(fkm):
    lib = ctypes.CDLL(fkm.LIB_PATH)
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, f"not exported: {missing}"
    # and the binding wraps each of them under the same name
    for n in declared_functions():
        assert n in fkm._SIG


def test_library_hides_internal_symbols(fkm):
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", fkm.LIB_PATH], capture_output=True,
                         text=True).stdout
    exported = {l.split()[-1] for l in out.splitlines() if " T " in l}
    ours = {s for s in exported if s.startswith("fkm")}
    assert ours == set(declared_functions())


def test_workspace_size_is_independent_of_n_times_k(fkm):
    a = fkm.fkm_workspace_size(1, 65536, 256, 128, 2)
    b = fkm.fkm_workspace_size(1, 65536, 8192, 128, 2)
    # growing K 32x grows only K-sized buffers, far below an N*K distance matrix
    assert b - a < 65536 * (8192 - 256) * 4 / 100
    c2 = fkm.fkm_workspace_size(32, 65536, 1024, 128, 2)
    assert c2 < 32 * 65536 * 1024 * 4 / 50


@pytest.mark.parametrize("shape,code", [
    ((0, 10, 4, 64, 2), 1),        # B < 1
    ((1, 10, 0, 64, 2), 1),        # K < 1
    ((1, 10, 4, 64, 9), 1),        # bad dtype
    ((1, 10, 4, 12, 2), 2),        # 24-byte rows: not a multiple of 16
    ((1, 10, 4, 6, 0), 2),         # 24-byte fp32 rows
    ((1, 10, 4, 4104, 2), 2),      # D too large for 16-bit points
    ((1, 10, 4, 4100, 0), 2),      # D too large for fp32 points
    ((2, 1 << 30, 4, 64, 2), 2),   # B*N >= 2^31
])
def test_invalid_shapes_are_rejected(fkm, shape, code):
    with pytest.raises(fkm.FkmError) as e:
        fkm.fkm_workspace_size(*shape)
    assert e.value.code == code
    assert fkm.lib().fkm_last_error().decode()


def test_null_pointers_rejected_before_any_launch(fkm):
    L = fkm.lib()
    ws = ctypes.create_string_buffer(1 << 20)
    addr = (ctypes.addressof(ws) + 15) & ~15
    rc = L.fkm_assign(1, 16, 4, 64, 2, None, addr, addr, None, addr, 1 << 19, None)
    assert rc == 1
    rc = L.fkm_update(1, 16, 4, 64, 2, addr, addr, addr, addr, addr, None, None, None, 0, None)
    assert rc == 1
    # workspace too small is its own status
    rc = L.fkm_assign(1, 16, 4, 64, 2, addr, addr, addr, None, addr, 64, None)
    assert rc == 4


def test_shard_calls_validate_before_any_launch(fkm):
    L = fkm.lib()
    ws = ctypes.create_string_buffer(1 << 20)
    a = (ctypes.addressof(ws) + 15) & ~15
    # fkm_partial_update: x is required
    assert L.fkm_partial_update(1, 16, 4, 64, 2, None, a, a, a, a, None, a, 1 << 19, None) == 1
    # fkm_finalize_sums: centers may not alias prev; the scratch must hold 256 + 8*B*K bytes
    assert L.fkm_finalize_sums(1, 4, 64, a, a + 4096, a + 8192, a + 8192, None, None, a + 16384,
                               1024, None) == 1
    assert L.fkm_finalize_sums(1, 4, 64, a, a + 4096, a + 8192, a + 12288, None, None, a + 16384,
                               200, None) == 4
    # fkm_partial_update_host: sums are required and 16-byte aligned; the host workspace
    # is sized by fkm_host_workspace_size
    assert L.fkm_partial_update_host(1, 16, 4, 64, 2, a, a, 16, a, None, a, None, 0, a, 1 << 19,
                                     None) == 1
    assert L.fkm_partial_update_host(1, 16, 4, 64, 2, a, a, 16, a, a + 8, a, None, 0, a, 1 << 19,
                                     None) == 1
    assert L.fkm_partial_update_host(1, 16, 4, 64, 2, a, a, 16, a, a, a, None, 0, a, 64,
                                     None) == 4
    # unknown flags
    assert L.fkm_partial_update_host(1, 16, 4, 64, 2, a, a, 16, a, a, a, None, 6, a, 1 << 19,
                                     None) == 1


def test_metric_calls_reject_unknown_metric(fkm):
    L = fkm.lib()
    ws = ctypes.create_string_buffer(1 << 20)
    a = (ctypes.addressof(ws) + 15) & ~15
    assert L.fkm_assign_metric(1, 16, 4, 64, 2, 3, a, a, a, a, 1 << 19, None) == 1
    assert L.fkm_assign_metric(1, 16, 4, 64, 2, -1, a, a, a, a, 1 << 19, None) == 1
    assert b"metric" in L.fkm_last_error()
    # a known metric still validates its pointers first
    assert L.fkm_assign_metric(1, 16, 4, 64, 2, 2, None, a, a, a, 1 << 19, None) == 1
    n = ctypes.c_int(0)
    assert L.fkm_lloyd_host_metric(1, 16, 4, 64, 2, 3, a, a, 1, 0.0, 16, a, a, a, None,
                                   ctypes.byref(n), a, 1 << 19, None) == 1
    assert b"metric" in L.fkm_last_error()
    assert L.fkm_lloyd_host_metric(1, 16, 4, 64, 2, 1, None, a, 1, 0.0, 16, a, a, a, None,
                                   ctypes.byref(n), a, 1 << 19, None) == 1


def test_status_strings_and_version(fkm):
    L = fkm.lib()
    assert L.fkm_status_string(0) == b"ok"
    assert b"workspace" in L.fkm_status_string(4)
    assert L.fkm_version().startswith(b"fkm")


def test_argsort_workspace_size(fkm):
    a = fkm.fkm_argsort_workspace_size(6, 4)
    b = fkm.fkm_argsort_workspace_size(1 << 20, 4)
    assert 0 < a < b
    with pytest.raises(fkm.FkmError):
        fkm.fkm_argsort_workspace_size(-1, 4)


def test_binding_refuses_strided_views_and_wrong_dtypes(fkm):
    """The C calls read dense row-major arrays of fixed types, so the binding
    refuses a strided view or a wrong dtype before any call."""
    import torch
    x = torch.zeros(2, 64, 16, dtype=torch.bfloat16)
    c = torch.zeros(2, 4, 16)
    ids = torch.zeros(2, 64, dtype=torch.int32)
    ws = torch.zeros(1 << 20, dtype=torch.uint8)
    with pytest.raises(ValueError, match="contiguous"):
        fkm.fkm_assign(x[:, ::2], c, ids[:, ::2], ws=ws)
    with pytest.raises(TypeError, match="float32"):
        fkm.fkm_assign(x, c.double(), ids, ws=ws)
    with pytest.raises(TypeError, match="int32"):
        fkm.fkm_assign(x, c, ids.long(), ws=ws)
    with pytest.raises(TypeError, match="float64"):
        fkm.fkm_partial_update(x, ids, c, torch.zeros(2, 4, 16), torch.zeros(2, 4, dtype=torch.int32),
                               ws=ws)


def test_binding_refuses_wrong_sizes_and_host_tensors(fkm):
    """Every tensor must hold the elements its role needs and sit on the GPU
    (host memory only for the streamed points): checked before any C call,
    so a mis-sized or host tensor never reaches a kernel."""
    import torch
    x = torch.zeros(2, 64, 16, dtype=torch.bfloat16)
    c = torch.zeros(2, 4, 16)
    ids = torch.zeros(2, 64, dtype=torch.int32)
    ws = torch.zeros(1 << 20, dtype=torch.uint8)
    with pytest.raises(ValueError, match="ids has shape"):
        fkm.fkm_assign(x, c, ids[:, :32].contiguous(), ws=ws)
    with pytest.raises(ValueError, match="inertia has shape"):
        fkm.fkm_assign(x, c, ids, torch.zeros(3, dtype=torch.float64), ws=ws)
    with pytest.raises(ValueError, match="centers has shape"):
        fkm.fkm_update(x, ids, c, torch.zeros(2, 5, 16), torch.zeros(2, 4, dtype=torch.int32),
                       ws=ws)
    with pytest.raises(ValueError, match="counts has shape"):
        fkm.fkm_lloyd(x, c, 3, 0.0, ids, torch.zeros(2, 4, 16), torch.zeros(2, 5, dtype=torch.int32),
                      ws=ws)
    with pytest.raises(ValueError, match="must be 3-D"):
        fkm.fkm_assign(x, c[0], ids, ws=ws)
    # sizes right, but host tensors where device memory is required
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        fkm.fkm_assign(x, c, ids, ws=ws)
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        fkm.fkm_assign_noalloc(x, c, ids)
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        fkm.fkm_lloyd_host(x, c, 3, 0.0, 16, ids, torch.zeros(2, 4, 16),
                           torch.zeros(2, 4, dtype=torch.int32), ws=ws)
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        fkm.fkm_lloyd_host_metric(x, c, 3, 0.0, 16, ids, torch.zeros(2, 4, 16),
                                  torch.zeros(2, 4, dtype=torch.int32), "cosine", ws=ws)
    with pytest.raises(ValueError, match="objective has shape"):
        fkm.fkm_lloyd_host_metric(x, c, 3, 0.0, 16, ids, torch.zeros(2, 4, 16),
                                  torch.zeros(2, 4, dtype=torch.int32), "dot",
                                  torch.zeros(3, dtype=torch.float64), ws=ws)
    with pytest.raises(ValueError, match="sums has shape"):
        fkm.fkm_finalize_sums(torch.zeros(2, 4, 8, dtype=torch.float64),
                              torch.zeros(2, 4, dtype=torch.float64), c, torch.zeros(2, 4, 16),
                              ws=ws)
    with pytest.raises(ValueError, match="idx has shape"):
        fkm.fkm_argsort(torch.zeros(10, dtype=torch.int32), 4, torch.zeros(9, dtype=torch.int32),
                        ws=ws)


def test_noalloc_size_limit_matches_the_header(fkm):
    """The header's limit, 256 + B*(4D + Kp*(2D + 32)) bytes with each part
    rounded up to 256, against FKM_NOALLOC_SCRATCH_BYTES: the first K past
    the limit is refused as unsupported before any device work.  (The shape
    just inside is not called here: it would go on to launch.)"""
    src = open(HEADER).read()
    assert "Kp*(2*D + 32)" in src
    L = fkm.lib()
    limit = 16 << 20
    D = 128

    def need(B, K):
        Kp = -(-K // 256) * 256
        r = lambda v: -(-v // 256) * 256
        return 256 + r(B * D * 4) + r(B * Kp * D * 2) + r(B * Kp * 32)

    K_in = 256 * ((limit - 256 - 512) // (256 * (2 * D + 32)))
    assert need(1, K_in) <= limit < need(1, K_in + 256)
    a = 1 << 12   # a 16-byte-aligned non-null stand-in; validation runs before any access
    rc_out = L.fkm_assign_noalloc(1, 128, K_in + 256, D, 2, a, a, a, None)
    assert rc_out == 2 and b"static scratch" in L.fkm_last_error()


def test_batch_per_grid_row_paths_reject_more_than_65535_batches(fkm):
    """fkm_assign's objective and fkm_centre run one grid row per batch: more
    than 65535 batches are refused before any launch (no CUDA call here)."""
    L = fkm.lib()
    buf = ctypes.create_string_buffer(1 << 12)
    a = (ctypes.addressof(buf) + 15) & ~15
    huge = 1 << 40   # a size check only: nothing is read or written
    B = 70000
    assert L.fkm_assign(B, 1, 1, 8, 2, a, a, a, a, a, huge, None) == 2
    assert b"65535" in L.fkm_last_error()
    assert L.fkm_centre(B, 1, 8, 2, a, a, a, a, huge, None) == 2
    assert b"65535" in L.fkm_last_error()
