"""The main paths of the library on odd shapes, run in the process that
loads the checked build (FKM_LIB_VARIANT=checked; tests/test_gpu_checked.py
starts it): every call is followed by a read of its workspace's status word,
so an out-of-range gather or scatter index raises, and the results are held
to the oracle.  Exits 0 when every path is clean."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
sys.path.insert(0, os.path.join(ROOT, "tests"))

import numpy as np  # noqa: E402
import torch  # noqa: E402

import datagen  # noqa: E402
import exact_means_clustering_b200 as fkm  # noqa: E402
from parity import check_assign, check_update, problem  # noqa: E402


def run_case(dtype, B, N, K, D, iters=3):
    w = datagen.Workload("checked", B, N, D, K, dtype, K, sigma=0.5, iters=iters, seed=B + N + K)
    x, xt, c0 = problem(w)
    c0t = torch.from_numpy(c0).cuda()
    ws = fkm.workspace(fkm.fkm_workspace_size(B, N, K, D, xt.dtype))
    ids = torch.empty(B, N, dtype=torch.int32, device="cuda")
    fkm.fkm_assign(xt, c0t, ids, ws=ws)
    fkm.fkm_sync_status(ws)
    g = ids.cpu().numpy()
    check_assign(x, dtype, c0, g)
    cen = torch.empty_like(c0t)
    cnt = torch.empty(B, K, dtype=torch.int32, device="cuda")
    fkm.fkm_update(xt, ids, c0t, cen, cnt, ws=ws)
    fkm.fkm_sync_status(ws)
    check_update(x, dtype, g, c0, cen.cpu().numpy(), cnt.cpu().numpy())
    for tol in (0.0, 1e-9):
        fkm.fkm_lloyd(xt, c0t, iters, tol, ids, cen, cnt, ws=ws)   # reads the status itself
    buf, sums, counts, obj = fkm.partial_buffers(B, K, D, "cuda")
    fkm.fkm_partial_update(xt, ids, c0t, sums, counts, obj, ws=ws)
    fkm.fkm_sync_status(ws)
    if dtype != "f32":
        fkm.fkm_assign_noalloc(xt, c0t, ids)
        fkm.fkm_assign_noalloc_status()
    hws = fkm.workspace(fkm.fkm_host_workspace_size(B, N, K, D, xt.dtype, 1000))
    fkm.fkm_lloyd_host(xt.cpu().pin_memory(), c0t, 2, 0.0, 1000, ids, cen, cnt, ws=hws)
    return True


def main():
    assert "checked build" in fkm.fkm_version(), fkm.fkm_version()
    cases = [("bf16", 3, 1000, 300, 64), ("f16", 2, 4097, 257, 32), ("f32", 1, 3001, 70, 132),
             ("bf16", 1, 9000, 2500, 128), ("bf16", 2, 777, 33, 264), ("bf16", 1, 40000, 3000, 64),
             ("f16", 8, 4096, 2048, 64), ("bf16", 1, 1, 1, 8)]
    for c in cases:
        run_case(*c)
        print("clean:", c, flush=True)
    keys = torch.from_numpy(np.random.default_rng(1).integers(0, 70000, 100003).astype(np.int32))
    keys = keys.cuda()
    idx = torch.empty_like(keys)
    ws = fkm.workspace(fkm.fkm_argsort_workspace_size(keys.numel(), 70000))
    fkm.fkm_argsort(keys, 70000, idx, ws=ws)
    fkm.fkm_sync_status(ws)
    print("all paths clean in the checked build")


if __name__ == "__main__":
    main()
