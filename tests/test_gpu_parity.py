"""GPU parity: every C-ABI call of libnmsparse against the fp64 CPU oracle.

Bit-exact for H, S, masks, values, metadata, window metadata, the lifted
activations and the packed GEMM operand; GEMM outputs within
max|Y - Y64| / max|Y64| <= 1e-2 of the oracle's fp64 product.
"""
import numpy as np
import pytest
import torch

import datagen
import oracle
from nm_testutil import (bf16_to_f64, decode_packed, packed_geometry, rel_err, to_dev, to_host,
                         to_host_u16, wmeta_nibbles)

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


# ---------------------------------------------------------------- a1 / a2
@pytest.fixture(params=["clusters", "workspace"])
def h_path(request, nm):
    # nm_hessian_diag combines a strip's token ranges inside a thread-block
    # cluster when the clusters fit on the device, else through the workspace
    # pairs and a second kernel; both paths must give the same H
    lib = nm.load()
    assert lib.nm_test_hessian_clusters(1 if request.param == "clusters" else 0) == 0
    yield request.param
    assert lib.nm_test_hessian_clusters(1) == 0


# one chunk; ragged runs; one column; a block with several chunks in its
# three-tile pipeline (K = 40000: more column blocks than SMs, so one split);
# 65 chunks over the SM-sized split of a 4096-column layer
@pytest.mark.parametrize("T,K,ld", [(128, 512, 512), (1000, 520, 520), (1, 7, 8), (129, 3, 8),
                                    (2048, 4096, 4096), (300, 517, 528), (257, 96, 104),
                                    (1000, 40000, 40000), (8292, 4096, 4104)])
def test_hessian_bitexact(nm, h_path, T, K, ld):
    X = datagen.make_activations(T, K, seed=T + K, n_outliers=min(4, K))
    H = nm.hessian_diag(to_dev(X, ld))
    _sync_ok(nm)
    assert np.array_equal(to_host(H), oracle.hessian_diag(X))


def test_hessian_launch_count(nm):
    # the launch accounting of the bench: one kernel for one token range or
    # for ranges combined inside clusters (they fit on a B200), two on the
    # workspace path
    lib = nm.load()
    assert lib.nm_hessian_launch_count(128, 4096) == 1
    assert lib.nm_hessian_launch_count(8192, 4096) == 1
    assert lib.nm_test_hessian_clusters(0) == 0
    try:
        assert lib.nm_hessian_launch_count(8192, 4096) == 2
        assert lib.nm_hessian_launch_count(128, 4096) == 1
    finally:
        assert lib.nm_test_hessian_clusters(1) == 0


def test_hessian_special_values_bitexact(nm, h_path):
    # zeros of both signs, bf16 subnormals, the smallest and largest normals
    # and infinities, in even and odd columns: every class of value whose
    # square the reduction must form exactly, against the oracle's fp64
    T, K = 300, 64
    X = datagen.make_activations(T, K, seed=5)
    special = np.array([0x0000, 0x8000, 0x0001, 0x807F, 0x0040, 0x0080, 0x8080, 0x7F7F, 0xFF7F,
                        0x1F80, 0x2000], dtype=np.uint16)
    g = np.random.default_rng(5)
    for j in range(2, 40):                       # a few special values in most columns
        rows = g.choice(T, size=int(g.integers(1, 6)), replace=False)
        X[rows, j] = g.choice(special, size=rows.size)
    X[:, 40] = 0x0001                            # a whole column of subnormals
    X[:, 41] = 0x8003
    X[:, 42] = 0x0000                            # and one of zeros
    X[7, 50] = 0x7F80                            # +inf and -inf
    X[9, 51] = 0xFF80
    X[11, 52] = 0x7FC1                           # NaN, and NaN beside an infinity
    X[12, 53] = 0xFFC0
    X[13, 53] = 0x7F80
    H = nm.hessian_diag(to_dev(X))
    _sync_ok(nm)
    h, ref = to_host(H), oracle.hessian_diag(X)
    assert np.isinf(ref[50]) and np.isinf(ref[51]) and ref[42] == 0.0 and 0.0 < ref[40] < 1e-70
    assert np.isnan(ref[52]) and np.isnan(ref[53])
    assert np.array_equal(h, ref, equal_nan=True)


@pytest.mark.parametrize("T", [300, 5000])
def test_hessian_exact_rounding_paths(nm, h_path, T):
    # columns that need each path of the exact sum, against the oracle:
    #  0: the tie 2^52 + 2^52 + 1 (rounds to even) and 1: the same broken up by
    #     the square of the smallest subnormal (the integer path);
    #  2: a 16-token run holding 2^20 and 2^-12 among ordinary values (its
    #     check fails; summed again in two parts, each exact);
    #  3: 2^60 and 2^-60 in two runs of one block (each run exact, the block's
    #     chain too wide: the integer path); 4: the same in different blocks
    #     (the finish adds the blocks' exact pairs);
    #  5: a run of 2^-64 values among ordinary ones; the rest Gaussian
    K = 40
    X = datagen.make_activations(T, K, seed=T, n_outliers=4)
    X[:, :6] = 0
    X[0, 0], X[1, 0], X[2, 0] = 0x4C80, 0x4C80, 0x3F80
    X[0, 1], X[1, 1], X[2, 1], X[T - 1, 1] = 0x4C80, 0x4C80, 0x3F80, 0x0001
    X[:, 2] = datagen.make_activations(T, 1, seed=1)[:, 0]
    X[17, 2], X[20, 2] = 0x3980, 0x4980                    # 2^-12, 2^20
    X[5, 3], X[40, 3] = 0x5D80, 0x2180                     # 2^60, 2^-60
    X[5, 4], X[T - 3, 4] = 0x5D80, 0x2180
    X[:, 5] = datagen.make_activations(T, 1, seed=2)[:, 0]
    X[32:48, 5] = 0x1F80                                   # 2^-64
    H = nm.hessian_diag(to_dev(X, 40))
    _sync_ok(nm)
    ref = oracle.hessian_diag(X)
    assert ref[0] == 2.0 ** 53 / T and ref[1] == (2.0 ** 53 + 2) / T
    assert np.array_equal(to_host(H), ref)


@pytest.mark.parametrize("R,K,ld", [(256, 512, 512), (33, 1030, 1032), (5, 13, 16), (64, 4096, 4096)])
def test_score_bitexact(nm, R, K, ld):
    X = datagen.make_activations(77, K, seed=R, n_outliers=2)
    W = datagen.make_weight(R, K, 0.02, seed=R + 1)
    H, S = nm.score(to_dev(X, ld), to_dev(W, ld), eps=1e-8)
    _, Sm = nm.score(None, to_dev(W, ld))
    _sync_ok(nm)
    Ho = oracle.hessian_diag(X)
    assert np.array_equal(to_host(H), Ho)
    assert np.array_equal(to_host(S), oracle.score_hessian(Ho, W, 1e-8))
    assert np.array_equal(to_host(Sm), oracle.score_magnitude(W))


@pytest.mark.parametrize("K", [1, 517, 4096])
def test_hessian_rescale_bitexact(nm, K):
    # the O(d_in) refresh, and for power-of-two scales the proxy recomputed from
    # the rescaled activations on the GPU
    X = datagen.make_activations(300, K, seed=K, n_outliers=min(2, K))
    H = nm.hessian_diag(to_dev(X, (K + 7) // 8 * 8))
    g = np.random.default_rng(K).uniform(0.3, 3.0, size=K)
    out = nm.hessian_rescale(H, torch.from_numpy(g).cuda())
    p2 = np.array([2.0 ** ((j % 7) - 3) for j in range(K)])
    out2 = nm.hessian_rescale(H, torch.from_numpy(p2).cuda())
    X2 = datagen.f32_to_bf16_bits(bf16_to_f64(X).astype(np.float32) / p2[None, :].astype(np.float32))
    H2 = nm.hessian_diag(to_dev(X2, (K + 7) // 8 * 8))
    _sync_ok(nm)
    assert np.array_equal(to_host(out), oracle.hessian_rescale(oracle.hessian_diag(X), g))
    assert np.array_equal(to_host(out2), to_host(H2))


def _zbits_dev(zb):
    return torch.from_numpy(np.ascontiguousarray(zb).view(np.int32)).cuda()


def _signs(zb, K):
    S = zb.shape[0]
    k = np.arange(K)
    return np.where((zb[:, k // 32] >> (k % 32).astype(np.uint32)) & 1, -1, 1).astype(np.int64)  # [S x K]


def _hutch_exact(Xbits, zb):
    # integer-valued X: D_k = N_k / (S T) with N_k = sum_s z_s[k] (X^T X z_s)[k]
    # an exact integer, then one correctly rounded division
    Xi = bf16_to_f64(Xbits).astype(np.int64)
    T, K = Xi.shape
    Z = _signs(zb, K)
    N = ((Xi.T @ (Xi @ Z.T)) * Z.T).sum(axis=1)
    return N.astype(np.float64) / float(zb.shape[0] * T)


def _hutch_scale(X, zb):
    # per column, (1/(S T)) sum_t |x_tk| sum_s |u_ts| with u = X z_s: the size of
    # the terms the kernels round in fp32 (an error scale, not the estimate)
    Xf = bf16_to_f64(X)
    Z = _signs(zb, X.shape[1]).astype(np.float64)
    U = np.abs(Xf @ Z.T).sum(axis=1)
    return (np.abs(Xf) * U[:, None]).sum(axis=0) / (zb.shape[0] * X.shape[0])


# integer-valued activations in [-4, 4] with S * K <= 2^15: every fp32 sum on
# the tensor-core path (u, the pieces of u, P, 32-token runs of x * P) stays an
# integer below 2^24, so the GPU estimate is the exact value up to the final
# scaling by 1/(S T): within 2^-51 relative.  One token / one column, ragged
# 128-token and 64-column tiles, S across 16-row and 64-column paddings, the
# largest S.
@pytest.mark.parametrize("T,K,S", [(1, 1, 1), (7, 33, 3), (300, 1000, 32), (129, 2048, 16),
                                   (1100, 128, 256), (2000, 517, 48), (4100, 64, 22)])
def test_hutchinson_integer_inputs_exact(nm, T, K, S):
    X = datagen.small_int_bf16((T, K), seed=T + K, tensor_id=3)
    zb = datagen.rademacher_bits(S, K, seed=S)
    D = nm.hutchinson_diag(to_dev(X, (K + 7) // 8 * 8), _zbits_dev(zb))
    _sync_ok(nm)
    d, exact = to_host(D), _hutch_exact(X, zb)
    assert np.all(np.abs(d - exact) <= 2.0 ** -51 * np.abs(exact))


# realistic activations (outlier channels x20): the fp64 oracle within 1e-5 of
# the fp32 rounding scale per column, and bit-identical repeated runs.  The
# last case is a full Llama-7B gate-projection input (8192 x 4096).
@pytest.mark.parametrize("T,K,S", [(1, 1, 1), (7, 33, 3), (300, 1000, 7), (129, 4096, 64),
                                   (1100, 517, 256), (8192, 4096, 16)])
def test_hutchinson_vs_oracle(nm, T, K, S):
    X = datagen.make_activations(T, K, seed=T + S, n_outliers=min(2, K))
    zb = datagen.rademacher_bits(S, K, seed=K + S)
    Xd, zd = to_dev(X, (K + 7) // 8 * 8), _zbits_dev(zb)
    D = nm.hutchinson_diag(Xd, zd)
    D2 = nm.hutchinson_diag(Xd, zd)
    _sync_ok(nm)
    d, d2 = to_host(D), to_host(D2)
    ref = oracle.hutchinson_diag(X, zb)
    assert np.array_equal(d, d2)                       # fixed summation order
    assert np.all(np.abs(d - ref) <= 1e-5 * _hutch_scale(X, zb) + 1e-300)


def test_hutchinson_hadamard_signs_give_h(nm):
    # K orthogonal sign vectors (Sylvester-Hadamard rows) make the estimate
    # exact: with integer activations the GPU estimate equals the GPU's H
    K, T = 64, 500
    Hd = np.array([[1.0]])
    while Hd.shape[0] < K:
        Hd = np.block([[Hd, Hd], [Hd, -Hd]])
    zb = np.zeros((K, 2), dtype=np.uint32)
    for k in range(K):
        zb[:, k // 32] |= (Hd[:, k] < 0).astype(np.uint32) << np.uint32(k % 32)
    X = datagen.small_int_bf16((T, K), seed=41, tensor_id=3)
    Xd = to_dev(X)
    D = nm.hutchinson_diag(Xd, _zbits_dev(zb))
    H = nm.hessian_diag(Xd)
    _sync_ok(nm)
    assert np.all(np.abs(to_host(D) - to_host(H)) <= 2.0 ** -51 * to_host(H))


def test_hutchinson_caller_workspace(nm):
    # a caller-owned workspace reused across calls of different shapes
    lib = nm.load()
    ws = torch.empty(lib.nm_hutchinson_workspace_bytes(1000, 1000, 32), dtype=torch.uint8, device="cuda")
    for (T, K, S) in ((1000, 1000, 32), (999, 520, 31), (1, 1000, 1)):
        assert lib.nm_hutchinson_workspace_bytes(T, K, S) <= ws.numel()
        X = datagen.small_int_bf16((T, K), seed=K, tensor_id=3)
        zb = datagen.rademacher_bits(S, K, seed=S)
        D = nm.hutchinson_diag(to_dev(X), _zbits_dev(zb), ws=ws)
        _sync_ok(nm)
        exact = _hutch_exact(X, zb)
        assert np.all(np.abs(to_host(D) - exact) <= 2.0 ** -51 * np.abs(exact))


# ---------------------------------------------------------------- a3
@pytest.mark.parametrize("n,m,R,K", [(2, 4, 64, 512), (6, 8, 33, 1030), (4, 6, 17, 1003),
                                     (8, 10, 9, 207), (2, 4, 3, 9), (1, 4, 8, 64), (3, 4, 8, 60),
                                     (2, 8, 5, 100), (5, 16, 4, 99), (1, 3, 6, 10), (6, 8, 128, 4096)])
@pytest.mark.parametrize("kind", ["gauss", "ties"])
def test_prune_bitexact(nm, n, m, R, K, kind):
    W = datagen.make_weight(R, K, 0.02, seed=K + m)
    if kind == "gauss":
        S = oracle.score_magnitude(W)
    else:
        S = datagen.tie_heavy_scores(R, K, seed=n + m, levels=3)
        S[:, ::7] = -0.0  # signed zeros tie with +0
    ld = (K + 7) // 8 * 8
    Sd = torch.from_numpy(np.pad(S, ((0, 0), (0, ld - K)))).cuda()[:, :K]
    mask, vals, meta = nm.prune_compress(Sd, to_dev(W, ld), n, m)
    _sync_ok(nm)
    om, ov, ometa = oracle.prune(np.abs(S) if kind == "ties" else S, W, n, m)
    assert np.array_equal(to_host(mask).view(np.uint32), om)
    assert np.array_equal(to_host_u16(vals), ov)
    if ometa is not None:
        assert np.array_equal(to_host(meta), ometa)


# ---------------------------------------------------------------- a4 / a5
# a2 + a3 fused (scores in registers, never written): the oracle's mask, values
# and 2:4 metadata, and bit-identical to the two-call path on the GPU
@pytest.mark.parametrize("n,m,R,K", [(2, 4, 64, 512), (2, 4, 33, 1030), (6, 8, 33, 1030), (4, 6, 17, 1003),
                                     (8, 10, 9, 207), (2, 4, 3, 9), (1, 4, 8, 64), (3, 4, 8, 60),
                                     (2, 8, 5, 100), (5, 16, 4, 99), (6, 8, 128, 4096)])
@pytest.mark.parametrize("mode", ["hessian", "magnitude", "ternary_values", "ties"])
def test_score_prune_fused_bitexact(nm, n, m, R, K, mode):
    ld = (K + 7) // 8 * 8
    X = datagen.make_activations(77, K, seed=R + K, n_outliers=2)
    if mode == "ties":
        # small integers: many equal |w| and equal products
        W = datagen.small_int_bf16((R, K), seed=R, tensor_id=5)
    else:
        W = datagen.make_weight(R, K, 0.02, seed=R + 1)
    score = "magnitude" if mode in ("magnitude", "ternary_values") else "hessian"
    ref = oracle.run_layer(X, W, n, m, eps=1e-8, score=score, ternary_values=(mode == "ternary_values"))
    Wd = to_dev(W, ld)
    Vd = to_dev(ref["V"], ld) if mode == "ternary_values" else None
    H = nm.hessian_diag(to_dev(X, ld)) if score == "hessian" else None
    mask, vals, meta = nm.score_prune_compress(H, Wd, n, m, V=Vd, eps=1e-8)
    # the two-call path on the same device inputs
    _, S = nm.score(to_dev(X, ld) if score == "hessian" else None, Wd, eps=1e-8)
    Sp = torch.zeros((R, ld), dtype=torch.float32, device="cuda")
    Sp[:, :K] = S                                   # prune wants a row stride % 8 == 0
    mask2, vals2, meta2 = nm.prune_compress(Sp[:, :K], Vd if Vd is not None else Wd, n, m)
    _sync_ok(nm)
    assert np.array_equal(to_host(mask).view(np.uint32), ref["mask"])
    assert np.array_equal(to_host_u16(vals), ref["vals"])
    assert np.array_equal(to_host(mask), to_host(mask2))
    assert np.array_equal(to_host_u16(vals), to_host_u16(vals2))
    if m == 4 and n == 2:
        assert np.array_equal(to_host(meta), ref["meta24"])
        assert np.array_equal(to_host(meta), to_host(meta2))


# the widths of the layers the bench runs and ragged ones: several 4096-column
# slices of the fused 2:4 kernel (H staged per slice), a ragged last slice,
# ragged row blocks (R = 9 against four rows per block), every (2N-2):2N
# pattern; Hessian scores, ternary values under magnitude scores, and
# small-integer weights (ties) under Hessian scores
@pytest.mark.parametrize("K", [4097, 8195, 11008, 28672])
@pytest.mark.parametrize("n,m", [(2, 4), (4, 6), (6, 8), (8, 10)])
@pytest.mark.parametrize("mode", ["hessian", "ternary_values", "ties"])
def test_score_prune_fused_wide_k(nm, n, m, K, mode):
    R = 9
    ld = (K + 7) // 8 * 8
    X = datagen.make_activations(77, K, seed=K + m, n_outliers=3)
    if mode == "ties":
        W = datagen.small_int_bf16((R, K), seed=K, tensor_id=5)
    else:
        W = datagen.make_weight(R, K, 0.02, seed=K + n)
    score = "magnitude" if mode == "ternary_values" else "hessian"
    ref = oracle.run_layer(X, W, n, m, eps=1e-8, score=score, ternary_values=(mode == "ternary_values"))
    Wd = to_dev(W, ld)
    Vd = to_dev(ref["V"], ld) if mode == "ternary_values" else None
    H = nm.hessian_diag(to_dev(X, ld)) if score == "hessian" else None
    mask, vals, meta = nm.score_prune_compress(H, Wd, n, m, V=Vd, eps=1e-8)
    _sync_ok(nm)
    if H is not None:
        assert np.array_equal(to_host(H), ref["H"])
    assert np.array_equal(to_host(mask).view(np.uint32), ref["mask"])
    assert np.array_equal(to_host_u16(vals), ref["vals"])
    if m == 4:
        assert np.array_equal(to_host(meta), ref["meta24"])


@pytest.mark.parametrize("m,R,K", [(4, 64, 512), (6, 20, 1003), (8, 33, 1030), (10, 9, 207),
                                   (8, 4, 8), (6, 128, 4096), (10, 7, 8195)])
def test_slide_pack_bitexact(nm, m, R, K):
    W = datagen.make_weight(R, K, 0.02, seed=m * K)
    S = oracle.score_magnitude(W)
    om, ov, _ = oracle.prune(S, W, m - 2, m)
    wm = nm.slide_pack(torch.from_numpy(om.view(np.int32)).cuda(), K, m)
    _sync_ok(nm)
    assert np.array_equal(to_host(wm), oracle.slide_pack(om, K, m))


def test_slide_pack_flags_bad_mask(nm):
    # a 5:8 mask is not (m-2):m: the kernel records NM_ERR_DEVICE, nothing hangs
    S = np.zeros((1, 8), dtype=np.float32)
    S[0, :5] = 1
    om, _, _ = oracle.prune(S, datagen.f32_to_bf16_bits(np.ones((1, 8), np.float32)), 5, 8)
    nm.slide_pack(torch.from_numpy(om.view(np.int32)).cuda(), 8, 8)
    torch.cuda.synchronize()
    with pytest.raises(nm.NMError, match="NM_ERR_DEVICE"):
        nm.check_device_error()
    nm.check_device_error()  # cleared


@pytest.mark.parametrize("m,T,K", [(4, 16, 64), (6, 33, 1003), (8, 17, 1030), (10, 5, 207),
                                   (8, 128, 4096), (6, 3, 9)])
def test_lift_bitexact(nm, m, T, K):
    X = datagen.make_activations(T, K, seed=T * m)
    ld = (K + 7) // 8 * 8
    XL = nm.lift_activations(to_dev(X, ld), m)
    _sync_ok(nm)
    assert np.array_equal(to_host_u16(XL), oracle.lift(X, m))


# ---------------------------------------------------------------- a6
@pytest.mark.parametrize("m,R,K", [(4, 256, 512), (8, 130, 1030), (6, 64, 1003), (10, 200, 2050),
                                   (4, 1, 9), (8, 300, 8195), (6, 257, 4100), (10, 129, 4096), (4, 390, 1034)])
def test_prepare_layout_bitexact(nm, m, R, K):
    # from the window metadata, and from the mask (the window pack fused in):
    # both decode to the oracle's values and window index pairs, byte for byte
    W = datagen.make_weight(R, K, 0.02, seed=R * m)
    res = oracle.run_layer(None, W, m - 2, m, score="magnitude")
    wm = res["meta24"] if m == 4 else res["wmeta"]
    packed = nm.sparse_prepare(to_dev(res["vals"]), torch.from_numpy(wm).cuda(), R, K, m)
    packed_m = nm.sparse_prepare_from_mask(to_dev(res["vals"]), torch.from_numpy(res["mask"].view(np.int32)).cuda(),
                                           R, K, m)
    _sync_ok(nm)
    g = packed_geometry(R, K, m)
    assert packed.numel() == g["vals_bytes"] + g["meta_bytes"]
    vals, nib, pad_ok = decode_packed(to_host(packed), R, K, m)
    assert pad_ok
    assert np.array_equal(vals, res["vals"])
    assert np.array_equal(nib, wmeta_nibbles(wm, g["nwin"]))
    assert np.array_equal(to_host(packed_m), to_host(packed))


def test_prepare_from_mask_flags_bad_mask(nm):
    # a 5:8 mask is not (m-2):m: NM_ERR_DEVICE in the error word, nothing hangs
    S = np.zeros((3, 16), dtype=np.float32)
    S[:, :5] = 1
    S[:, 8:14] = 1
    W = datagen.f32_to_bf16_bits(np.ones((3, 16), np.float32))
    om, ov, _ = oracle.prune(S, W, 5, 8)
    vals = to_dev(np.zeros((3, 12), dtype=np.uint16))
    nm.sparse_prepare_from_mask(vals, torch.from_numpy(om.view(np.int32)).cuda(), 3, 16, 8)
    torch.cuda.synchronize()
    with pytest.raises(nm.NMError, match="NM_ERR_DEVICE"):
        nm.check_device_error()
    nm.check_device_error()


# ---------------------------------------------------------------- a7 / a8
def _layer(R, K, T, n, m, seed, outliers=0):
    X = datagen.make_activations(T, K, seed=seed, n_outliers=outliers)
    W = datagen.make_weight(R, K, 0.02, seed=seed + 1)
    res = oracle.run_layer(X, W, n, m)
    return X, W, res


def _gemm_sparse(nm, X, res, R, K, m, ldx=None):
    wm = res["meta24"] if m == 4 else res["wmeta"]
    packed = nm.sparse_prepare(to_dev(res["vals"]), torch.from_numpy(wm).cuda(), R, K, m)
    Y = nm.sparse_gemm(to_dev(X, ldx), packed, R, m)
    _sync_ok(nm)
    return bf16_to_f64(to_host_u16(Y))


@pytest.mark.parametrize("m,R,K,T", [(4, 256, 512, 128), (4, 130, 1030, 200), (4, 128, 128, 1),
                                     (6, 256, 1536, 128), (8, 256, 1024, 128), (10, 256, 1280, 128),
                                     (6, 131, 1003, 77), (8, 200, 1030, 257), (10, 129, 2050, 16),
                                     (8, 384, 4096, 384), (4, 1000, 768, 1100), (8, 520, 2056, 700),
                                     (6, 300, 1206, 513), (10, 260, 2010, 300)])
def test_sparse_gemm_vs_oracle(nm, m, R, K, T):
    X, W, res = _layer(R, K, T, m - 2, m, seed=R + K + T, outliers=2)
    Y = _gemm_sparse(nm, X, res, R, K, m, ldx=(K + 7) // 8 * 8)
    Y64 = oracle.gemm_masked(X, res["mask"], W, m)
    assert rel_err(Y, Y64) <= GEMM_TOL


# tokens per wide tile: T <= 240 gives one tile of T rounded up to 16 (the
# last store of 16 tokens when T % 32 lands in (0, 16]); larger T splits into
# near-equal tiles of at most 240 (their count chosen against the resident CTA
# pairs' waves)
@pytest.mark.parametrize("T", [1, 16, 33, 48, 240, 241, 496, 721])
@pytest.mark.parametrize("m,R", [(4, 700), (8, 512)])
def test_sparse_gemm_token_tiling(nm, m, R, T):
    K = 512
    X, W, res = _layer(R, K, T, m - 2, m, seed=R + T + m)
    Y = _gemm_sparse(nm, X, res, R, K, m)
    Y64 = oracle.gemm_masked(X, res["mask"], W, m)
    assert rel_err(Y, Y64) <= GEMM_TOL


@pytest.mark.parametrize("m,R,K,T", [(4, 256, 512, 128), (4, 1000, 768, 1100), (8, 520, 2056, 700),
                                     (6, 131, 1003, 77), (10, 260, 2010, 300)])
def test_tile256_ablation_vs_oracle(nm, m, R, K, T):
    # the 256 x 256 pair-tile GEMM (ablation entry point) gives the same product
    X, W, res = _layer(R, K, T, m - 2, m, seed=R + K + T + 2)
    wm = res["meta24"] if m == 4 else res["wmeta"]
    packed = nm.sparse_prepare(to_dev(res["vals"]), torch.from_numpy(wm).cuda(), R, K, m)
    Y = nm.sparse_gemm(to_dev(X, (K + 7) // 8 * 8), packed, R, m, tile256=True)
    _sync_ok(nm)
    Y64 = oracle.gemm_masked(X, res["mask"], W, m)
    assert rel_err(bf16_to_f64(to_host_u16(Y)), Y64) <= GEMM_TOL


@pytest.mark.parametrize("m,R,K,T", [(6, 256, 1536, 128), (8, 256, 1024, 128), (10, 256, 1280, 128),
                                     (8, 200, 1030, 257), (6, 131, 1003, 77), (10, 129, 2050, 16),
                                     (4, 130, 1030, 200)])
def test_in_kernel_lift_ablation_vs_oracle(nm, m, R, K, T):
    # the ablation entry point lifts inside the GEMM (no workspace)
    X, W, res = _layer(R, K, T, m - 2, m, seed=R + K + T + 1, outliers=2)
    wm = res["meta24"] if m == 4 else res["wmeta"]
    packed = nm.sparse_prepare(to_dev(res["vals"]), torch.from_numpy(wm).cuda(), R, K, m)
    Y = nm.sparse_gemm(to_dev(X, (K + 7) // 8 * 8), packed, R, m, fused=True)
    _sync_ok(nm)
    Y64 = oracle.gemm_masked(X, res["mask"], W, m)
    assert rel_err(bf16_to_f64(to_host_u16(Y)), Y64) <= GEMM_TOL


@pytest.mark.parametrize("m", [6, 8, 10])
def test_fused_lift_equals_two_pass(nm, m):
    # lift_activations + a 2:4 GEMM of width K' versus the fused kernel.  For
    # 4:6 and 8:10 both use the natural K' order and the same tiles, so the fp32
    # tensor-core sums are identical bits; 6:8 packs K' in another order (raw
    # tiles of X first), and the library kernel visits its blocks in yet
    # another (every raw block before every middle-window block), so those
    # agree within rounding.
    # (whole-tile schedule throughout: the fused kernel has no stream-K form,
    # and splitting K' would change the fp32 summation order)
    R, K, T = 256, 1030, 130
    X, W, res = _layer(R, K, T, m - 2, m, seed=m)
    wm = res["wmeta"]
    packed = nm.sparse_prepare(to_dev(res["vals"]), torch.from_numpy(wm).cuda(), R, K, m)
    nm.set_gemm_schedule(1)
    try:
        Yf = bf16_to_f64(to_host_u16(nm.sparse_gemm(to_dev(X, 1032), packed, R, m, fused=True)))
        Yl = bf16_to_f64(to_host_u16(nm.sparse_gemm(to_dev(X, 1032), packed, R, m)))
        XL = nm.lift_activations(to_dev(X, 1032), m)
        KL = XL.shape[1]
        packed24 = nm.sparse_prepare(to_dev(res["vals"]), torch.from_numpy(res["wmeta"]).cuda(), R, KL, 4)
        Y2 = bf16_to_f64(to_host_u16(nm.sparse_gemm(XL, packed24, R, 4)))
        _sync_ok(nm)
    finally:
        nm.set_gemm_schedule(0)
    Y64 = oracle.gemm_masked(X, res["mask"], W, m)
    assert rel_err(Y2, Y64) <= GEMM_TOL
    assert rel_err(Yl, Y64) <= GEMM_TOL
    if m == 8:
        assert rel_err(Yf, Y2) <= 2 ** -7
        assert rel_err(Yl, Yf) <= 2 ** -7
    else:
        assert np.array_equal(Y2, Yf)
        assert np.array_equal(Yl, Yf)


@pytest.mark.parametrize("R,K,T", [(256, 512, 128), (384, 4096, 384)])
def test_single_cta_ablation_gemms(nm, R, K, T):
    # the 1-CTA baseline kernels (ablation entry point) give the same products
    X, W, res = _layer(R, K, T, 2, 4, seed=R + T)
    lib = nm.load()
    s = torch.cuda.current_stream().cuda_stream
    Xd = to_dev(X)
    packed = nm.sparse_prepare(to_dev(res["vals"]), torch.from_numpy(res["meta24"]).cuda(), R, K, 4)
    Wd = oracle.dense_masked(res["mask"], W, K)
    Ys = torch.empty((T, R), dtype=torch.bfloat16, device="cuda")
    Yd = torch.empty((T, R), dtype=torch.bfloat16, device="cuda")
    assert lib.nm_gemm_1cta(1, Xd.data_ptr(), T, K, K, packed.data_ptr(), R, 0, Ys.data_ptr(), R, s) == 0
    Wdd = to_dev(Wd)
    assert lib.nm_gemm_1cta(0, Xd.data_ptr(), T, K, K, Wdd.data_ptr(), R, K, Yd.data_ptr(), R, s) == 0
    _sync_ok(nm)
    Y64 = oracle.gemm_masked(X, res["mask"], W, 4)
    assert rel_err(bf16_to_f64(to_host_u16(Ys)), Y64) <= GEMM_TOL
    assert rel_err(bf16_to_f64(to_host_u16(Yd)), Y64) <= GEMM_TOL


@pytest.mark.parametrize("R,K,T", [(256, 512, 128), (130, 1030, 200), (128, 64, 1), (384, 4096, 384),
                                   (1000, 768, 1100)])
def test_dense_gemm_vs_oracle_and_torch(nm, R, K, T):
    X, W, res = _layer(R, K, T, 2, 4, seed=R * 3 + T)
    Wd = oracle.dense_masked(res["mask"], W, K)
    ld = (K + 7) // 8 * 8
    Yd = nm.dense_gemm(to_dev(X, ld), to_dev(Wd, ld))
    _sync_ok(nm)
    Y = bf16_to_f64(to_host_u16(Yd))
    Y64 = oracle.gemm_dense(X, Wd)
    assert rel_err(Y, Y64) <= GEMM_TOL
    Yt = (to_dev(X).float() @ to_dev(Wd).float().T).double().cpu().numpy()
    assert rel_err(Y, Yt) <= GEMM_TOL


# ---------------------------------------------------------------- ternary
def test_ternary_gamma_exact_rounding_and_specials(nm):
    # gamma is the correctly rounded sum / (R K): a tie to even, the tie
    # broken by a subnormal (integer path), a row of subnormals only; an
    # infinity or a NaN in W is reported, not returned
    rows = np.zeros((4, 8), dtype=np.uint16)
    rows[0, :2] = (0x5A00, 0x3F80)                 # 2^53 + 1: a tie, to even
    rows[1, 0] = 0x0001                            # breaks it upwards
    rows[2, :] = (0x0001, 0x0003, 0x807F, 0x0040, 0, 0x8001, 0x0002, 0)
    W = datagen.make_weight(40, 8, 0.02, seed=3)
    W[:4] = rows
    Wq, gamma = nm.ternary_quantize(to_dev(W))
    _sync_ok(nm)
    g, oWq = oracle.ternary(W)
    assert to_host(gamma)[0] == g
    assert np.array_equal(to_host_u16(Wq), oWq)
    for bad in (0x7F80, 0xFFC1):
        Wb = W.copy()
        Wb[7, 5] = bad
        nm.ternary_quantize(to_dev(Wb))
        torch.cuda.synchronize()
        with pytest.raises(nm.NMError, match="NM_ERR_DEVICE"):
            nm.check_device_error()


def test_ternary_threshold_at_the_tie(nm):
    # gamma = mean |w| = 1 exactly: ones everywhere but six values whose
    # magnitudes also sum to six.  |w| = 0.5 is the tie (rint(0.5) = 0), the
    # bf16 just below gives 0 and the one just above gives +-bf16(gamma)
    def bf(v):
        return np.frombuffer(np.float32(v).tobytes(), dtype=np.uint16)[1]
    W = np.full((16, 64), bf(1.0), dtype=np.uint16)
    W[::2, 1::3] |= 0x8000                                   # signs play no part in gamma
    specials = [(0.5, (3, 5)), (0.498046875, (4, 6)), (0.50390625, (5, 7)),
                (2.5, (6, 8)), (1.5, (7, 9)), (0.498046875, (8, 10))]
    for v, (i, j) in specials:
        W[i, j] = bf(v) | (W[i, j] & 0x8000)
    Wq, gamma = nm.ternary_quantize(to_dev(W))
    _sync_ok(nm)
    assert to_host(gamma)[0] == 1.0
    q = to_host_u16(Wq)
    g, oWq = oracle.ternary(W)
    assert g == 1.0 and np.array_equal(q, oWq)
    assert q[3, 5] == 0 and q[4, 6] == 0 and q[8, 10] == 0   # 0.5 ties to 0; below
    assert q[5, 7] & 0x7FFF == bf(1.0)                       # just above the tie
    assert np.count_nonzero(q) == W.size - 3


@pytest.mark.parametrize("R,K", [(64, 256), (11008 // 8, 4096 // 4), (3, 13)])
def test_ternary_bitexact(nm, R, K):
    W = datagen.make_weight(R, K, 0.02, seed=R)
    ld = (K + 7) // 8 * 8
    Wq, gamma = nm.ternary_quantize(to_dev(W, ld))
    _sync_ok(nm)
    g, oWq = oracle.ternary(W)
    assert to_host(gamma)[0] == g
    assert np.array_equal(to_host_u16(Wq), oWq)


# ---------------------------------------------------------------- whole path
def _device_pipeline(nm, X, W, n, m, eps=1e-8, score="hessian", ternary=False):
    # the calls the bench's step makes: H, the fused score + prune, the window
    # pack fused into the operand preparation, and the sparse GEMM
    Xd, Wd = to_dev(X), to_dev(W)
    V = Wd
    if ternary:
        V, _ = nm.ternary_quantize(Wd)
    H = nm.hessian_diag(Xd) if score == "hessian" else None
    mask, vals, meta = nm.score_prune_compress(H, Wd, n, m, V=V, eps=eps)
    if m == 4:
        packed = nm.sparse_prepare(vals, meta, W.shape[0], W.shape[1], m)
    else:
        packed = nm.sparse_prepare_from_mask(vals, mask, W.shape[0], W.shape[1], m)
    Y = nm.sparse_gemm(Xd, packed, W.shape[0], m)
    wm = meta if m == 4 else nm.slide_pack(mask, W.shape[1], m)   # the standalone pack, checked too
    _sync_ok(nm)
    return dict(H=H, mask=mask, vals=vals, wm=wm, Y=Y, V=V)


def _check_pipeline(nm, layer, n_rows=512):
    X, W = datagen.layer_inputs(layer)
    out = _device_pipeline(nm, X, W, layer.n, layer.m, layer.eps, layer.score, layer.ternary)
    ref = oracle.run_layer(X, W, layer.n, layer.m, layer.eps, layer.score, layer.ternary)
    if ref["H"] is not None:
        assert np.array_equal(to_host(out["H"]), ref["H"])
    assert np.array_equal(to_host(out["mask"]).view(np.uint32), ref["mask"])
    assert np.array_equal(to_host_u16(out["vals"]), ref["vals"])
    wm_ref = ref["meta24"] if layer.m == 4 else ref["wmeta"]
    assert np.array_equal(to_host(out["wm"]), wm_ref)
    rows = np.sort(np.random.default_rng(layer.T).choice(layer.T, size=min(n_rows, layer.T), replace=False))
    Y = bf16_to_f64(to_host_u16(out["Y"][torch.from_numpy(rows).cuda()]))
    Y64 = oracle.gemm_masked(X, ref["mask"], ref["V"], layer.m, rows=rows)
    assert rel_err(Y, Y64) <= GEMM_TOL
    # every output row is finite and the unsampled rows are not left unwritten
    Yall = out["Y"].float()
    assert torch.isfinite(Yall).all()


# every workload family; 512 sampled token rows of Y (all of them when T is
# smaller) against the oracle's fp64 product, the rest checked finite (outputs
# are poisoned with NaN before each call)
@pytest.mark.parametrize("name", ["small_2of4", "slide_6of8_4096", "ternary_6of8_gate",
                                  "llama7b_q_T8192", "llama7b_gate_T8192", "llama7b_down_T8192",
                                  "llama7b_gate_T2048", "llama7b_down_T128", "llama7b_q_T16"])
def test_workload_pipeline(nm, name):
    _check_pipeline(nm, datagen.WORKLOADS[name])


@pytest.mark.parametrize("name", [f"llama70b_{p}_{nm_}" for p in ("up", "down")
                                  for nm_ in ("2of4", "4of6", "6of8", "8of10")])
def test_workload_pipeline_70b(nm, name):
    _check_pipeline(nm, datagen.WORKLOADS[name])
