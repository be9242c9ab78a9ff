"""The allocation-free H reduction, nm_hessian_diag_noalloc.

Some callers cannot allocate device memory (a plugin inside a framework that
owns all device memory, or a loop that must not pay for cudaMalloc's possible
device synchronisation).  For them the library keeps the chunk partials of the
H reduction in a static device array.  These tests call that entry point
through the C ABI and compare it with nm_hessian_diag, which takes a caller
workspace: the two must give bit-identical H (the tolerance of every H test),
on two calls in a row, since the shared array keeps the previous call's
contents.  This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

import datagen
from nm_testutil import to_dev

pytestmark = pytest.mark.gpu

NM_ERR_TOO_LARGE = 9
MAX_PARTIALS = 1048576


def _reference_H(lib, Xd, T, K, ld):
    H = torch.empty(K, dtype=torch.float64, device="cuda")
    need = lib.nm_hessian_workspace_bytes(T, K)
    ws = torch.empty(max(need, 1), dtype=torch.uint8, device="cuda")
    st = lib.nm_hessian_diag(Xd.data_ptr(), T, K, ld, H.data_ptr(), ws.data_ptr(), need,
                             torch.cuda.current_stream().cuda_stream)
    assert st == 0
    return H


def test_noalloc_matches_workspace_entry_point_two_calls_in_a_row():
    import semi_structured_sparse_diag_b200 as nm
    lib = nm.load()
    stream = torch.cuda.current_stream().cuda_stream
    # the second call is smaller than the first: stale partials of the first
    # call remain in the shared array and must not leak into the result
    for (T, K, ld, seed) in ((4096, 8192, 8192, 1), (1000, 517, 520, 2)):
        X = datagen.make_activations(T, K, seed=seed, n_outliers=3)
        Xd = to_dev(X, ld)
        H = torch.full((K,), float("nan"), dtype=torch.float64, device="cuda")
        st = lib.nm_hessian_diag_noalloc(Xd.data_ptr(), T, K, ld, H.data_ptr(), stream)
        assert st == 0, lib.nm_status_string(st)
        Href = _reference_H(lib, Xd, T, K, ld)
        torch.cuda.synchronize()
        nm.check_device_error()
        assert torch.equal(H, Href)


def test_noalloc_rejects_sizes_beyond_its_scratch():
    import semi_structured_sparse_diag_b200 as nm
    lib = nm.load()
    Xd = torch.zeros((8, 8), dtype=torch.bfloat16, device="cuda")
    H = torch.zeros(8, dtype=torch.float64, device="cuda")
    # 8192 tokens -> 64 chunks; 64 * 16392 > 1048576 partials
    st = lib.nm_hessian_diag_noalloc(Xd.data_ptr(), 8192, 16392, 16392, H.data_ptr(), None)
    assert st == NM_ERR_TOO_LARGE
    assert b"static scratch" in lib.nm_status_string(st)
    # a single chunk of tokens needs no scratch at all: no limit applies
    st = lib.nm_hessian_diag_noalloc(Xd.data_ptr(), 8, 8, 8, H.data_ptr(), None)
    assert st == 0
    torch.cuda.synchronize()
