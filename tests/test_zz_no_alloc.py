"""fkm_assign_noalloc, the assign entry point for callers that cannot allocate
device memory (code whose device memory belongs to a framework allocator that
must not be bypassed, services with all memory reserved up front, plugins
handed only inputs and outputs).  It must give exactly what fkm_assign gives,
call after call, while its scratch lives in one static device array that
every call reuses, and it must allocate nothing.

This file is collected last so that a run stopping at the first failure has
run every other test first; it also passes alone in a fresh process."""
import numpy as np
import pytest
import torch

import datagen
from parity import check_assign, problem

pytestmark = pytest.mark.gpu

fkm = pytest.importorskip("exact_means_clustering_b200")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _call_c_abi(x, c, ids, K):
    """Call the entry point through the C ABI directly (no binding helper)."""
    L = fkm.lib()
    B, N, D = x.shape
    dtype = {torch.bfloat16: 2, torch.float16: 1}[x.dtype]
    rc = L.fkm_assign_noalloc(B, N, K, D, dtype, x.data_ptr(), c.data_ptr(), ids.data_ptr(),
                              torch.cuda.current_stream().cuda_stream)
    assert rc == 0, L.fkm_last_error().decode()


def _status():
    L = fkm.lib()
    rc = L.fkm_assign_noalloc_status(torch.cuda.current_stream().cuda_stream)
    assert rc == 0, L.fkm_last_error().decode()


def _free_bytes():
    torch.cuda.synchronize()
    return torch.cuda.mem_get_info()[0]


@pytest.mark.parametrize("wid,scale", [(2, dict(B=3, N=5000, K=700)),
                                       (3, dict(B=2, N=7560, K=1000))])
def test_noalloc_matches_workspace_assign_twice(wid, scale):
    w = datagen.CONFIGS[wid].scaled(**scale)
    x, xt, c0 = problem(w)
    rng = np.random.default_rng(wid)
    # two calls in a row with different centroids: no state may leak between them
    for call in range(2):
        cn = c0 + 0.05 * call * rng.standard_normal(c0.shape).astype(np.float32)
        c = torch.from_numpy(cn).cuda()
        ref = torch.empty(w.B, w.N, dtype=torch.int32, device="cuda")
        fkm.fkm_assign(xt, c, ref)
        got = torch.full((w.B, w.N), -1, dtype=torch.int32, device="cuda")
        _call_c_abi(xt, c, got, w.K)
        _status()
        assert torch.equal(got, ref), f"call {call}: {(got != ref).sum().item()} ids differ"
        # and against the fp64 oracle, with the criteria every assign test uses
        check_assign(x, w.dtype, cn, got.cpu().numpy())


def test_noalloc_allocates_nothing():
    """After a first call on the device (which looks up the array and loads
    the kernels), further calls change neither torch's allocations nor the
    device's free memory."""
    w = datagen.CONFIGS[2].scaled(B=2, N=3000, K=300)
    x, xt, c0 = problem(w)
    c = torch.from_numpy(c0).cuda()
    ids = torch.empty(w.B, w.N, dtype=torch.int32, device="cuda")
    _call_c_abi(xt, c, ids, w.K)
    _status()
    torch.cuda.synchronize()
    alloc0, free0 = torch.cuda.memory_allocated(), _free_bytes()
    for _ in range(3):
        _call_c_abi(xt, c, ids, w.K)
    _status()
    assert torch.cuda.memory_allocated() == alloc0
    assert _free_bytes() == free0


def test_noalloc_at_the_size_limit():
    """The largest K the static scratch holds at D = 128 (the header's limit,
    256 + B*(4D + Kp*(2D + 32)) bytes, each part rounded to 256) runs and
    matches fkm_assign; one centroid tile more is refused."""
    D, N = 128, 1024
    K = 256 * (((16 << 20) - 768) // (256 * (2 * D + 32)))
    rng = np.random.default_rng(5)
    xt = torch.from_numpy(rng.standard_normal((1, N, D)).astype(np.float32)).to(torch.bfloat16).cuda()
    c = torch.from_numpy(rng.standard_normal((1, K, D)).astype(np.float32)).cuda()
    ref = torch.empty(1, N, dtype=torch.int32, device="cuda")
    fkm.fkm_assign(xt, c, ref)
    got = torch.full((1, N), -1, dtype=torch.int32, device="cuda")
    _call_c_abi(xt, c, got, K)
    _status()
    assert torch.equal(got, ref)
    L = fkm.lib()
    c2 = torch.zeros(1, K + 256, D, device="cuda")
    rc = L.fkm_assign_noalloc(1, N, K + 256, D, 2, xt.data_ptr(), c2.data_ptr(), got.data_ptr(),
                              None)
    assert rc == 2 and b"static scratch" in L.fkm_last_error()


def test_noalloc_rejects_oversized_and_fp32():
    L = fkm.lib()
    x = torch.zeros(1, 128, 128, dtype=torch.bfloat16, device="cuda")
    c = torch.zeros(1, 65536, 128, device="cuda")
    ids = torch.empty(1, 128, dtype=torch.int32, device="cuda")
    # 65536 centroids x 128 dims x 2 bytes = 16 MiB of operands: over the limit
    rc = L.fkm_assign_noalloc(1, 128, 65536, 128, 2, x.data_ptr(), c.data_ptr(), ids.data_ptr(),
                              None)
    assert rc == 2 and b"static scratch" in L.fkm_last_error()
    xf = torch.zeros(1, 128, 128, device="cuda")
    rc = L.fkm_assign_noalloc(1, 128, 4, 128, 0, xf.data_ptr(), c.data_ptr(), ids.data_ptr(),
                              None)
    assert rc == 2
