"""GPU parity of the FP8 (E4M3) path: per-token quantisation fused with the
lift, the FP8 weight operand, and the kind::f8f6f4 sparse GEMM (SlideSparse
sec. 2B / 2C).

Codes and scales are bit-exact against the oracle (both sides multiply by
fp32(1 / scale) and round to the nearest E4M3 code, ties to even,
saturating).  The GEMM is
bit-exact where every code is exact and the scales are 1 (integer products
below 2^24 in fp32, one bf16 rounding), and within the GEMM bar
max|Y - Y64| / max|Y64| <= 1e-2 of the oracle's fp64 product of the same
codes elsewhere.
"""
import numpy as np
import pytest
import torch

import datagen
import oracle
from nm_testutil import bf16_to_f64, rel_err, to_dev, to_host, to_host_u16

pytestmark = pytest.mark.gpu

GEMM_TOL = 1e-2


@pytest.fixture(scope="module")
def nm():
    import semi_structured_sparse_diag_b200 as nm
    nm.load()
    return nm


def _sync_ok(nm):
    torch.cuda.synchronize()
    nm.check_device_error()


def _u8(t):
    return t.contiguous().cpu().numpy()


def _wmeta(res, m):
    return res["meta24"] if m == 4 else res["wmeta"]


# (T, K, m, ldq extra): one token, ragged K, every pattern, a padded ld, and
# rows wider than the 48 K columns staged in shared memory (read from global)
@pytest.mark.parametrize("T,K,m,extra", [(1, 7, 4, 0), (33, 1030, 8, 16), (300, 4096, 6, 0),
                                         (5, 2010, 10, 32), (129, 512, 4, 0), (64, 4096, 8, 0),
                                         (3, 50001, 8, 0)])
def test_quant_lift_f8_bitexact(nm, T, K, m, extra):
    X = datagen.make_activations(T, K, seed=T + K + m, n_outliers=min(2, K))
    X[0, : min(K, 5)] = 0                                  # some exact zeros
    if T > 3:
        X[3] = 0                                           # an all-zero token (scale 1)
    ldq = oracle.lifted_cols_f8(K, m) + extra
    Xq, xs = nm.quant_lift_f8(to_dev(X, (K + 7) // 8 * 8), m, ldq=ldq)
    _sync_ok(nm)
    Q, s = oracle.quant_lift_f8(X, m, ldq=ldq)
    assert np.array_equal(_u8(Xq), Q)
    assert np.array_equal(to_host(xs), s)


def _expected_meta_blocks(wmeta, R, K, m):
    G = (K + m - 1) // m
    nwin = G * (m // 2 - 1)
    KLf = oracle.lifted_cols_f8(K, m)
    nkb, Rpad = KLf // 256, (R + 127) // 128 * 128
    wbytes = (nwin + 1) // 2
    out = np.zeros((Rpad // 128) * nkb * 4096, dtype=np.uint8)
    for r in range(Rpad):
        mt, lane = divmod(r, 128)
        for kb in range(nkb):
            for a in range(2):
                for i in range(16):
                    w0 = 64 * kb + 32 * a + 2 * i
                    lo = hi = 0x4
                    if r < R:
                        byte = int(wmeta[r, w0 // 2]) if w0 // 2 < wbytes else 0x44
                        lo = byte & 0xF if w0 < nwin else 0x4
                        hi = byte >> 4 if w0 + 1 < nwin else 0x4
                    out[((mt * nkb + kb) * 2 + a) * 2048 + lane * 16 + i] = lo | (hi << 4)
    return out


@pytest.mark.parametrize("R,K,m", [(130, 520, 8), (64, 1003, 6), (200, 256, 4), (3, 90, 10)])
def test_prepare_f8_layout(nm, R, K, m):
    X = datagen.make_activations(40, K, seed=R, n_outliers=2)
    W = datagen.make_weight(R, K, 0.02, seed=R + 1)
    res = oracle.run_layer(X, W, m - 2, m)
    wm = _wmeta(res, m)
    packed = _u8(nm.sparse_prepare_f8(to_dev(res["vals"]), torch.from_numpy(wm).cuda(), R, K, m))
    _sync_ok(nm)
    KLf, Rpad = oracle.lifted_cols_f8(K, m), (R + 127) // 128 * 128
    L = res["vals"].shape[1]
    codes = packed[: Rpad * KLf // 2].reshape(Rpad, KLf // 2)
    meta = packed[Rpad * KLf // 2: Rpad * KLf // 2 + (Rpad // 128) * (KLf // 256) * 4096]
    scales = packed[Rpad * KLf // 2 + len(meta):].view(np.float32)
    Wq, ws = oracle.quant_rows_f8(res["vals"])
    assert np.array_equal(codes[:R, :L], Wq) and not codes[:R, L:].any() and not codes[R:].any()
    assert np.array_equal(scales[:R], ws) and np.all(scales[R:] == 1.0)
    assert np.array_equal(meta, _expected_meta_blocks(wm, R, K, m))


def _exact_layer(T, R, K, m, seed):
    # integer values with one +-448 per token / weight row: exact codes, scale 1
    g = np.random.default_rng(seed)
    X = datagen.f32_to_bf16_bits(g.integers(-8, 9, size=(T, K)).astype(np.float32))
    X[:, 1] = datagen.f32_to_bf16_bits(np.full(T, 448.0, np.float32))
    W = datagen.f32_to_bf16_bits(g.integers(-8, 9, size=(R, K)).astype(np.float32))
    W[:, 2] = datagen.f32_to_bf16_bits(np.full(R, -448.0, np.float32))
    return X, W, oracle.run_layer(X, W, m - 2, m, score="magnitude")


# exact codes, scale 1: the product is exact in fp32, so Y is the bf16 rounding
# of the exact integer result; every pattern, ragged T, R and K, several tiles
@pytest.mark.parametrize("T,R,K,m", [(1, 1, 8, 4), (130, 200, 520, 4), (77, 131, 1003, 6),
                                     (256, 256, 1024, 8), (33, 129, 2010, 10), (300, 64, 4096, 8)])
def test_gemm_f8_exact(nm, T, R, K, m):
    X, W, res = _exact_layer(T, R, K, m, seed=T + R + K)
    packed = nm.sparse_prepare_f8(to_dev(res["vals"]), torch.from_numpy(_wmeta(res, m)).cuda(), R, K, m)
    Xq, xs = nm.quant_lift_f8(to_dev(X, (K + 7) // 8 * 8), m)
    Y = nm.sparse_gemm_f8(Xq, xs, packed, R, K, m)
    _sync_ok(nm)
    assert np.all(to_host(xs) == 1.0)
    exact = oracle.gemm_masked(X, res["mask"], W, m)
    expect = np.array([[oracle.f64_to_bf16(v) for v in row] for row in exact], dtype=np.uint16)
    assert np.array_equal(to_host_u16(Y), expect)


# realistic layers: against the oracle's fp64 product of the same codes
@pytest.mark.parametrize("T,R,K,m", [(300, 520, 2056, 8), (128, 256, 4096, 4), (77, 131, 1003, 6),
                                     (2048, 4096, 4096, 8)])
def test_gemm_f8_vs_oracle(nm, T, R, K, m):
    X = datagen.make_activations(T, K, seed=T + m, n_outliers=2)
    W = datagen.make_weight(R, K, 0.02, seed=R + K)
    res = oracle.run_layer(X, W, m - 2, m)
    packed = nm.sparse_prepare_f8(to_dev(res["vals"]), torch.from_numpy(_wmeta(res, m)).cuda(), R, K, m)
    Xq, xs = nm.quant_lift_f8(to_dev(X, (K + 7) // 8 * 8), m)
    Y = nm.sparse_gemm_f8(Xq, xs, packed, R, K, m)
    _sync_ok(nm)
    Xq4, xs4 = oracle.quant_lift_f8(X, 4)
    Wq, ws = oracle.quant_rows_f8(res["vals"])
    rows = None if T <= 512 else np.random.default_rng(1).choice(T, 256, replace=False)
    Y64 = oracle.gemm_f8(Xq4, xs4, res["mask"], Wq, ws, K, m, rows=rows)
    y = bf16_to_f64(to_host_u16(Y))
    assert rel_err(y if rows is None else y[rows], Y64) <= GEMM_TOL
    # and the FP8 layer stays close to the bf16 one (E4M3 keeps 3 mantissa bits)
    Yb = oracle.gemm_masked(X, res["mask"], W, m, rows=rows)
    assert rel_err(y if rows is None else y[rows], Yb) <= 0.1
