"""The allocation-free H reduction, nm_hessian_diag_noalloc.

Some callers cannot allocate device memory (a plugin inside a framework that
owns all device memory, or a loop that must not pay for cudaMalloc's possible
device synchronisation).  For them the library keeps the partial sums of the
H reduction in a static device array.  These tests call that entry point
through the C ABI and compare it with nm_hessian_diag, which takes a caller
workspace: the two must give bit-identical H (the tolerance of every H test),
on calls in a row of different sizes, since the shared array keeps the
previous call's contents.  Its argument checks (sizes beyond what it takes
return NM_ERR_SHAPE before any CUDA call) are tested on the CPU in
test_abi.py.  This file is collected last on purpose.
"""
import numpy as np
import pytest
import torch

import datagen
import oracle
from nm_testutil import to_dev

pytestmark = pytest.mark.gpu

MAX_PAIRS = 131072   # NM_HESSIAN_NOALLOC_MAX_PAIRS: (s, c) fp64 pairs, 2 MiB


def _reference_H(lib, Xd, T, K, ld):
    H = torch.empty(K, dtype=torch.float64, device="cuda")
    need = lib.nm_hessian_workspace_bytes(T, K)
    ws = torch.empty(max(need, 16), dtype=torch.uint8, device="cuda")
    st = lib.nm_hessian_diag(Xd.data_ptr(), T, K, ld, H.data_ptr(), ws.data_ptr(), need,
                             torch.cuda.current_stream().cuda_stream)
    assert st == 0
    return H


# a large first call, then smaller ones: stale pairs of an earlier call remain
# in the shared array and must not leak into a later result.  8192 x 16384
# uses the most pairs of these (two token ranges x 16384 columns); 1000 x 517
# is ragged in both dimensions; 100 x 70000 needs no scratch (one range).
@pytest.mark.parametrize("calls", [((8192, 16384, 16384, 1), (4096, 8192, 8192, 2), (1000, 517, 520, 3)),
                                   ((100, 70000, 70000, 4), (2048, 4096, 4096, 5))])
def test_noalloc_matches_workspace_entry_point_calls_in_a_row(calls):
    import semi_structured_sparse_diag_b200 as nm
    lib = nm.load()
    stream = torch.cuda.current_stream().cuda_stream
    for (T, K, ld, seed) in calls:
        assert lib.nm_hessian_workspace_bytes(T, K) <= MAX_PAIRS * 16
        X = datagen.make_activations(T, K, seed=seed, n_outliers=3)
        Xd = to_dev(X, ld)
        H = torch.full((K,), float("nan"), dtype=torch.float64, device="cuda")
        st = lib.nm_hessian_diag_noalloc(Xd.data_ptr(), T, K, ld, H.data_ptr(), stream)
        assert st == 0, lib.nm_status_string(st)
        Href = _reference_H(lib, Xd, T, K, ld)
        torch.cuda.synchronize()
        nm.check_device_error()
        assert torch.equal(H, Href)
        if T * K <= 1000 * 520:
            assert np.array_equal(H.cpu().numpy(), oracle.hessian_diag(X))
