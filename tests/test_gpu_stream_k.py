"""GPU parity of the stream-K schedule of the CTA-pair GEMMs.

Stream-K splits the K' blocks of all output tiles evenly over the CTA pairs; a
split tile's first pair adds the fp32 partial sums the later pairs left in the
workspace.  These tests force that schedule (and small pair counts, so that
tiles are split at many places, and large ones, so that some pairs get no
work) and check the products against the fp64 oracle, against the whole-tile
schedule, and for run-to-run determinism.
"""
import numpy as np
import pytest
import torch

import datagen
import oracle
from nm_testutil import bf16_to_f64, rel_err, to_dev, to_host_u16

pytestmark = pytest.mark.gpu

GEMM_TOL = 1e-2


@pytest.fixture(scope="module")
def nm():
    import semi_structured_sparse_diag_b200 as nm
    nm.load()
    yield nm
    nm.set_gemm_schedule(0, 0)


@pytest.fixture
def schedule(nm):
    def set_(policy, clusters=0):
        nm.set_gemm_schedule(policy, clusters)
    yield set_
    nm.set_gemm_schedule(0, 0)


def _sync_ok(nm):
    torch.cuda.synchronize()
    nm.check_device_error()


def _layer(R, K, T, m, seed):
    X = datagen.make_activations(T, K, seed=seed, n_outliers=2)
    W = datagen.make_weight(R, K, 0.02, seed=seed + 1)
    return X, W, oracle.run_layer(X, W, m - 2, m)


def _packed(nm, res, R, K, m):
    wm = res["meta24"] if m == 4 else res["wmeta"]
    return nm.sparse_prepare(to_dev(res["vals"]), torch.from_numpy(wm).cuda(), R, K, m)


def _y(t):
    return bf16_to_f64(to_host_u16(t))


# (m, R, K, T, pairs): 0 pairs = all that fit on the device
SPARSE_CASES = [
    (4, 256, 512, 128, 0),      # 8 K' blocks over every pair: most pairs idle
    (4, 512, 4096, 300, 3),     # 4 tiles over 3 pairs: splits inside tiles 1 and 2
    (4, 256, 4096, 256, 0),     # one tile split over 32 pairs
    (4, 4096, 4096, 16, 0),     # decode-sized T: one valid 32-token chunk
    (4, 1000, 768, 1100, 7),    # ragged rows and tokens
    (8, 520, 2056, 700, 5),     # 6:8, raw and middle-window blocks split
    (8, 4096, 4096, 128, 0),
    (6, 131, 1003, 77, 0),      # 4:6 via the lifted 2:4 GEMM
    (10, 260, 2010, 300, 7),    # 8:10
]


@pytest.mark.parametrize("m,R,K,T,pairs", SPARSE_CASES)
def test_sparse_stream_k_vs_oracle(nm, schedule, m, R, K, T, pairs):
    X, W, res = _layer(R, K, T, m, seed=R + K + T + m)
    packed = _packed(nm, res, R, K, m)
    Xd = to_dev(X, (K + 7) // 8 * 8)
    schedule(2, pairs)
    Ysk = nm.sparse_gemm(Xd, packed, R, m)
    Ysk2 = nm.sparse_gemm(Xd, packed, R, m)
    schedule(1, pairs)
    Yt = nm.sparse_gemm(Xd, packed, R, m)
    _sync_ok(nm)
    Y64 = oracle.gemm_masked(X, res["mask"], W, m)
    a, b, t = _y(Ysk), _y(Ysk2), _y(Yt)
    assert rel_err(a, Y64) <= GEMM_TOL
    assert rel_err(t, Y64) <= GEMM_TOL
    assert np.array_equal(a, b)               # fixed summation order: deterministic
    assert rel_err(a, t) <= 2 ** -7           # differs from whole tiles by rounding only


DENSE_CASES = [
    (384, 4096, 384, 0),
    (130, 1030, 200, 3),
    (4096, 4096, 16, 0),
    (1000, 768, 1100, 5),
]


@pytest.mark.parametrize("R,K,T,pairs", DENSE_CASES)
def test_dense_stream_k_vs_oracle(nm, schedule, R, K, T, pairs):
    X, W, res = _layer(R, K, T, 4, seed=3 * R + T)
    Wd = oracle.dense_masked(res["mask"], W, K)
    ld = (K + 7) // 8 * 8
    Xd, Wdd = to_dev(X, ld), to_dev(Wd, ld)
    schedule(2, pairs)
    Ysk = _y(nm.dense_gemm(Xd, Wdd))
    Ysk2 = _y(nm.dense_gemm(Xd, Wdd))
    schedule(1, pairs)
    Yt = _y(nm.dense_gemm(Xd, Wdd))
    _sync_ok(nm)
    Y64 = oracle.gemm_dense(X, Wd)
    assert rel_err(Ysk, Y64) <= GEMM_TOL
    assert np.array_equal(Ysk, Ysk2)
    assert rel_err(Ysk, Yt) <= 2 ** -7


def test_stream_k_workspace_reuse(nm, schedule):
    # one workspace for consecutive launches on different inputs: each launch's
    # flags carry its own sequence number, so no stale partial is ever used
    R, K, T, m = 512, 2048, 200, 4
    lib = nm.load()
    ws = torch.empty(lib.nm_sparse_gemm_workspace_bytes(T, K, m), dtype=torch.uint8, device="cuda")
    schedule(2, 4)
    outs = []
    for seed in (1, 2, 3):
        X, W, res = _layer(R, K, T, m, seed=seed)
        packed = _packed(nm, res, R, K, m)
        Y = nm.sparse_gemm(to_dev(X), packed, R, m, ws=ws)
        outs.append((Y, X, W, res))
    _sync_ok(nm)
    for Y, X, W, res in outs:
        assert rel_err(_y(Y), oracle.gemm_masked(X, res["mask"], W, m)) <= GEMM_TOL


def test_small_workspace_falls_back_to_whole_tiles(nm, schedule):
    # a workspace holding only the staged activations still gives the product
    R, K, T, m = 256, 1024, 100, 8
    X, W, res = _layer(R, K, T, m, seed=11)
    packed = _packed(nm, res, R, K, m)
    G = (K + m - 1) // m
    ws = torch.empty(T * ((G * 4 + 7) // 8 * 8) * 2, dtype=torch.uint8, device="cuda")
    schedule(2, 0)
    Y = nm.sparse_gemm(to_dev(X), packed, R, m, ws=ws)
    _sync_ok(nm)
    assert rel_err(_y(Y), oracle.gemm_masked(X, res["mask"], W, m)) <= GEMM_TOL


def test_owner_gives_up_on_a_withheld_flag_and_the_next_launch_is_correct(nm, schedule):
    # Failure detection without a GPU fault: one tile of 2:4 (R = 256, K' = 32
    # blocks) cut into four stream-K ranges, so pairs 1..3 hand partial sums to
    # pair 0.  Pair 2 withholds its flag and the wait limit is 10 ms: pair 0's
    # bounded poll gives up, records NM_ERR_TIMEOUT and the kernel finishes
    # (it releases tensor memory and exits as on a normal run; only global
    # memory polling is involved, no copy is in flight).  The error word
    # reports it once; a following launch with the controls back is correct.
    lib = nm.load()
    R, K, T, m = 256, 4096, 64, 4
    X, W, res = _layer(R, K, T, m, seed=77)
    packed = _packed(nm, res, R, K, m)
    Xd = to_dev(X)
    Y64 = oracle.gemm_masked(X, res["mask"], W, m)
    schedule(2, 4)
    try:
        assert lib.nm_test_set_wait_limit_ns(10_000_000) == 0
        assert lib.nm_test_withhold_stream_k_flag(2) == 0
        nm.sparse_gemm(Xd, packed, R, m)
        torch.cuda.synchronize()
        with pytest.raises(nm.NMError, match="NM_ERR_TIMEOUT"):
            nm.check_device_error()
    finally:
        assert lib.nm_test_withhold_stream_k_flag(-1) == 0
        assert lib.nm_test_set_wait_limit_ns(0) == 0
    nm.check_device_error()                    # reported once, then cleared
    Y = nm.sparse_gemm(Xd, packed, R, m)       # same schedule, flags published
    _sync_ok(nm)
    assert rel_err(_y(Y), Y64) <= GEMM_TOL
    assert lib.nm_test_set_wait_limit_ns(2_000_000_000) == 2   # above one second: refused
