"""fkm_assign_noalloc, the assign entry point for callers that cannot allocate
device memory (code inside an allocation-free stream capture, services with
all memory reserved up front, plugins handed only inputs and outputs).  It
must give exactly what fkm_assign gives, call after call, while its scratch
lives in one static device array that every call reuses.

This file is collected last so that a run stopping at the first failure has
run every other test first; it also passes alone in a fresh process."""
import ctypes

import numpy as np
import pytest
import torch

import datagen
from parity import problem

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


@pytest.mark.parametrize("wid,scale", [(2, dict(B=3, N=5000, K=700)),
                                       (3, dict(B=2, N=7560, K=1000))])
def test_noalloc_matches_workspace_assign_twice(wid, scale):
    w = datagen.CONFIGS[wid].scaled(**scale)
    x, xt, c0 = problem(w)
    rng = np.random.default_rng(wid)
    # two calls in a row with different centroids: no state may leak between them
    for call in range(2):
        c = torch.from_numpy(c0 + 0.05 * call * rng.standard_normal(c0.shape).astype(np.float32))
        c = c.cuda()
        ref = torch.empty(w.B, w.N, dtype=torch.int32, device="cuda")
        fkm.fkm_assign(xt, c, ref)
        got = torch.full((w.B, w.N), -1, dtype=torch.int32, device="cuda")
        _call_c_abi(xt, c, got, w.K)
        torch.cuda.synchronize()
        assert torch.equal(got, ref), f"call {call}: {(got != ref).sum().item()} ids differ"


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
