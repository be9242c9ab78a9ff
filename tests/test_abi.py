"""Host-side checks of the C ABI (no GPU needed): the library builds for
sm_100a, loads, exports every function include/nmsparse.h declares, and its
argument validation rejects bad calls before launching anything."""
import ctypes
import os
import re

import pytest

import semi_structured_sparse_diag_b200 as nm
from nm_testutil import packed_geometry

INCLUDE = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include")


def declared_functions():
    src = "\n".join(open(os.path.join(INCLUDE, f)).read() for f in sorted(os.listdir(INCLUDE))
                    if f.endswith(".h"))
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b([A-Za-z_]\w*)\s*\(", src, flags=re.M)
    return sorted(set(n for n in names if n not in ("if", "defined")))


def test_header_matches_exports():
    lib = nm.load()
    decl = declared_functions()
    assert len(decl) >= 14
    assert sorted(nm.EXPORTED) == decl
    for name in decl:
        assert getattr(lib, name) is not None


def test_status_strings_and_version():
    lib = nm.load()
    assert lib.nm_status_string(0) == b"NM_OK"
    for code in range(1, 10):
        assert lib.nm_status_string(code).startswith(b"NM_ERR_")
    assert lib.nm_status_string(99) == b"unknown nm_status"
    assert lib.nm_version() >> 16 == 1


def test_size_queries():
    lib = nm.load()
    # H: one (s, c) pair of fp64 per column and token range; the ranges of
    # 128-token chunks fill one wave of 2 * 148 blocks of 128 columns, and a
    # single range needs no workspace
    def h_ws(T, K):
        cb, chunks = (K + 127) // 128, (T + 127) // 128
        split = max(1, min(296 // cb, chunks))
        return split * K * 16 if split > 1 else 0
    assert lib.nm_hessian_workspace_bytes(128, 512) == 0
    assert lib.nm_hessian_workspace_bytes(129, 512) == 2 * 512 * 16
    assert lib.nm_hessian_workspace_bytes(8192, 4096) == 9 * 4096 * 16
    for (T, K) in ((300, 4), (2048, 4096), (8192, 11008), (4096, 28672), (1, 100000), (10 ** 6, 56832)):
        assert lib.nm_hessian_workspace_bytes(T, K) == h_ws(T, K)
        # every size fits the allocation-free variant's 2 MiB of pairs
        assert lib.nm_hessian_workspace_bytes(T, K) <= 131072 * 16
    assert lib.nm_hessian_workspace_bytes(8192, 40000) == 0
    for (R, K, m) in ((256, 512, 4), (4096, 4096, 8), (131, 1003, 6), (28672, 8192, 10), (1, 1, 4)):
        g = packed_geometry(R, K, m)
        assert lib.nm_sparse_prepare_bytes(R, K, m) == g["vals_bytes"] + g["meta_bytes"]
    assert lib.nm_sparse_prepare_bytes(256, 512, 5) == 0
    assert lib.nm_sparse_prepare_bytes(0, 512, 4) == 0
    assert lib.nm_ternary_workspace_bytes(100) == 100 * 16 + 16
    # staged activations (rounded up to 256 bytes), then the stream-K region:
    # per CTA pair 2 x 8 slots of 32 x 240 fp32 and 2 x 8 flags of 8 bytes
    sk = 96 * 2 * 8 * (32 * 240 * 4 + 8)
    up = lambda b: (b + 255) // 256 * 256
    assert lib.nm_sparse_gemm_workspace_bytes(2048, 4096, 4) == sk
    assert lib.nm_sparse_gemm_workspace_bytes(2048, 4096, 8) == 2048 * 2048 * 2 + sk      # T x K/2
    assert lib.nm_sparse_gemm_workspace_bytes(7, 1003, 6) == up(7 * 1344 * 2) + sk       # T x K'
    assert lib.nm_sparse_gemm_workspace_bytes(16, 8195, 10) == up(16 * 13120 * 2) + sk
    assert lib.nm_sparse_gemm_workspace_bytes(0, 4096, 4) == 0
    assert lib.nm_sparse_gemm_workspace_bytes(16, 4096, 5) == 0
    assert lib.nm_dense_gemm_workspace_bytes(16, 4096, 4096) == sk
    assert lib.nm_dense_gemm_workspace_bytes(16, 0, 4096) == 0
    # Z [S16 x ldz], [Z^T Z^T Z^T] [K x C3], U partials [nsplit x T x S16] fp32,
    # U pieces [T x C3] bf16, D partials [T/128 x K] fp64, each padded to 1 KiB
    k1 = lambda b: (b + 1023) // 1024 * 1024

    def hq(T, K, S):
        S16, C3, ldz, tt = (S + 15) // 16 * 16, (3 * S + 63) // 64 * 64, (K + 7) // 8 * 8, (T + 127) // 128
        ns = max(1, min(8, (K + 63) // 64, (148 + tt - 1) // tt))
        return (k1(S16 * ldz * 2) + k1(K * C3 * 2) + k1(ns * T * S16 * 4) + k1(T * C3 * 2)
                + k1(tt * K * 8))
    assert lib.nm_hutchinson_workspace_bytes(300, 1000, 7) == hq(300, 1000, 7)
    assert lib.nm_hutchinson_workspace_bytes(8192, 4096, 16) == hq(8192, 4096, 16)
    assert lib.nm_hutchinson_workspace_bytes(1, 1, 256) == hq(1, 1, 256)
    assert lib.nm_hutchinson_workspace_bytes(0, 64, 1) == 0
    # FP8: lifted width rounded up to 256; packed = codes [Rpad x KLf/2] +
    # 4 KB of metadata per (128 rows, 256 lifted columns) + fp32 row scales
    assert lib.nm_lifted_cols_f8(4096, 4) == 4096 and lib.nm_lifted_cols_f8(4096, 8) == 6144
    assert lib.nm_lifted_cols_f8(1003, 6) == 1536 and lib.nm_lifted_cols_f8(7, 10) == 256
    assert lib.nm_lifted_cols_f8(64, 5) == 0 and lib.nm_lifted_cols_f8(64, 12) == 0
    for (R, K, m) in ((4096, 4096, 8), (131, 1003, 6), (1, 1, 4)):
        KLf, Rpad = lib.nm_lifted_cols_f8(K, m), (R + 127) // 128 * 128
        assert lib.nm_sparse_prepare_f8_bytes(R, K, m) == Rpad * KLf // 2 + Rpad // 128 * KLf // 256 * 4096 + Rpad * 4
    assert lib.nm_sparse_prepare_f8_bytes(0, 8, 4) == 0
    assert lib.nm_hutchinson_workspace_bytes(64, 64, 257) == 0


# fake but 16-byte aligned device addresses: validation fails before any use
A = 0x10000
MIS = 0x10002


@pytest.mark.parametrize("call,expect", [
    (lambda l: l.nm_hessian_diag(None, 4, 4, 8, A, None, 0, None), 1),
    (lambda l: l.nm_hessian_diag(A, 0, 4, 8, A, None, 0, None), 2),
    (lambda l: l.nm_hessian_diag(A, 4, 9, 8, A, None, 0, None), 2),
    (lambda l: l.nm_hessian_diag(MIS, 4, 4, 8, A, None, 0, None), 3),
    (lambda l: l.nm_hessian_diag(A, 4, 4, 12, A, None, 0, None), 3),
    (lambda l: l.nm_hessian_diag(A, 300, 4, 8, A, None, 0, None), 5),
    (lambda l: l.nm_hessian_diag(A, 300, 4, 8, A, A + 8, 1 << 20, None), 3),
    (lambda l: l.nm_hessian_diag(A, 4, 4, 8, A + 4, None, 0, None), 3),
    (lambda l: l.nm_hessian_diag(A, 1 << 31, 4, 8, A, A, 1 << 40, None), 2),
    # the allocation-free variant: the same checks, before any CUDA call
    (lambda l: l.nm_hessian_diag_noalloc(None, 4, 4, 8, A, None), 1),
    (lambda l: l.nm_hessian_diag_noalloc(A, 4, 4, 8, None, None), 1),
    (lambda l: l.nm_hessian_diag_noalloc(A, 0, 4, 8, A, None), 2),
    (lambda l: l.nm_hessian_diag_noalloc(A, 4, 9, 8, A, None), 2),
    (lambda l: l.nm_hessian_diag_noalloc(A, 1 << 31, 4, 8, A, None), 2),
    (lambda l: l.nm_hessian_diag_noalloc(A, (1 << 62) + 5, 16392, 16392, A, None), 2),
    (lambda l: l.nm_hessian_diag_noalloc(MIS, 4, 4, 8, A, None), 3),
    (lambda l: l.nm_hessian_diag_noalloc(A, 4, 4, 12, A, None), 3),
    (lambda l: l.nm_prune_compress(A, 8, A, 8, 4, 8, 2, 17, A, A, A, None), 4),
    (lambda l: l.nm_prune_compress(A, 8, A, 8, 4, 8, 4, 4, A, A, A, None), 4),
    (lambda l: l.nm_prune_compress(A, 8, A, 8, 4, 8, 2, 4, A, A, None, None), 1),
    (lambda l: l.nm_prune_compress(A, 8, MIS, 8, 4, 8, 2, 4, A, A, A, None), 3),
    (lambda l: l.nm_score_prune_compress(None, 0.0, None, 8, A, 8, 4, 8, 2, 4, A, A, A, None), 1),
    (lambda l: l.nm_score_prune_compress(None, 0.0, A, 8, A, 8, 4, 8, 2, 4, A, A, None, None), 1),
    (lambda l: l.nm_score_prune_compress(None, 0.0, A, 8, A, 8, 4, 8, 2, 17, A, A, A, None), 4),
    (lambda l: l.nm_score_prune_compress(None, 0.0, A, 4, A, 8, 4, 8, 2, 4, A, A, A, None), 2),
    (lambda l: l.nm_score_prune_compress(None, 0.0, MIS, 8, A, 8, 4, 8, 2, 4, A, A, A, None), 3),
    (lambda l: l.nm_score_prune_compress(A + 4, 0.0, A, 8, A, 8, 4, 8, 2, 4, A, A, A, None), 3),
    (lambda l: l.nm_hessian_rescale(None, A, 8, A, None), 1),
    (lambda l: l.nm_hessian_rescale(A, A, 0, A, None), 2),
    (lambda l: l.nm_hessian_rescale(A, A + 4, 8, A, None), 3),
    (lambda l: l.nm_hutchinson_diag(None, 4, 8, 8, A, 2, A, A, 1 << 20, None), 1),
    (lambda l: l.nm_hutchinson_diag(A, 4, 8, 8, A, 2, A, None, 1 << 20, None), 1),
    (lambda l: l.nm_hutchinson_diag(A, 4, 8, 4, A, 2, A, A, 1 << 20, None), 2),
    (lambda l: l.nm_hutchinson_diag(A, 4, 8, 8, A, 0, A, A, 1 << 20, None), 2),
    (lambda l: l.nm_hutchinson_diag(A, 4, 8, 8, A, 257, A, A, 1 << 20, None), 2),
    (lambda l: l.nm_hutchinson_diag(A, 4, 8, 12, A, 2, A, A, 1 << 20, None), 3),
    (lambda l: l.nm_hutchinson_diag(A, 4, 8, 8, A + 2, 2, A, A, 1 << 20, None), 3),
    (lambda l: l.nm_hutchinson_diag(A, 4, 8, 8, A, 2, A + 4, A, 1 << 20, None), 3),
    (lambda l: l.nm_hutchinson_diag(A, 4, 8, 8, A, 2, A, A, 16, None), 5),
    (lambda l: l.nm_hutchinson_diag(A, 4, 1 << 31, 1 << 31, A, 2, A, A, 1 << 62, None), 2),
    (lambda l: l.nm_hutchinson_diag(A, 1 << 31, 8, 8, A, 2, A, A, 1 << 62, None), 2),
    (lambda l: l.nm_quant_lift_f8(None, 4, 8, 8, 4, A, 256, A, None), 1),
    (lambda l: l.nm_quant_lift_f8(A, 4, 8, 8, 5, A, 256, A, None), 4),
    (lambda l: l.nm_quant_lift_f8(A, 4, 8, 8, 4, A, 128, A, None), 2),
    (lambda l: l.nm_quant_lift_f8(A, 4, 8, 8, 4, A, 264, A, None), 3),
    (lambda l: l.nm_quant_lift_f8(A, 4, 8, 8, 4, MIS, 256, A, None), 3),
    (lambda l: l.nm_sparse_prepare_f8(A, None, 4, 8, 8, A, 1 << 20, None), 1),
    (lambda l: l.nm_sparse_prepare_f8(A, A, 4, 8, 12, A, 1 << 20, None), 4),
    (lambda l: l.nm_sparse_prepare_f8(A, A, 4, 8, 8, A, 16, None), 5),
    (lambda l: l.nm_sparse_gemm_f8(A, 4, 8, 256, None, A, 4, 8, A, 8, None), 1),
    (lambda l: l.nm_sparse_gemm_f8(A, 4, 8, 128, A, A, 4, 8, A, 8, None), 2),
    (lambda l: l.nm_sparse_gemm_f8(A, 4, 8, 256, A, A, 4, 8, A, 12, None), 3),
    (lambda l: l.nm_sparse_gemm_f8(A, 4, 8, 256, A, A, 4, 3, A, 8, None), 4),
    (lambda l: l.slide_pack(A, 4, 8, 7, A, None), 4),
    (lambda l: l.slide_pack(A, 4, 8, 12, A, None), 4),
    (lambda l: l.lift_activations(A, 4, 8, 8, 5, A, 8, None), 4),
    (lambda l: l.lift_activations(A, 4, 8, 8, 8, A, 8, None), 2),
    (lambda l: l.nm_sparse_prepare(A, A, 4, 8, 4, A, 1, None), 5),
    (lambda l: l.nm_sparse_prepare(A, A, 4, 8, 4, MIS, 1 << 20, None), 3),
    (lambda l: l.nm_sparse_prepare(A + 2, A, 4, 8, 4, A, 1 << 20, None), 3),
    (lambda l: l.nm_sparse_prepare_from_mask(A, None, 4, 8, 4, A, 1 << 20, None), 1),
    (lambda l: l.nm_sparse_prepare_from_mask(A, A, 4, 8, 5, A, 1 << 20, None), 4),
    (lambda l: l.nm_sparse_prepare_from_mask(A, A, 4, 8, 8, A, 1, None), 5),
    (lambda l: l.nm_sparse_prepare_from_mask(A, A + 2, 4, 8, 8, A, 1 << 20, None), 3),
    (lambda l: l.nm_sparse_prepare_from_mask(A, A, 0, 8, 8, A, 1 << 20, None), 2),
    (lambda l: l.nm_sparse_gemm(A, 4, 8, 8, A, 4, 9, A, 8, None, 0, None), 4),
    (lambda l: l.nm_sparse_gemm(A, 4, 8, 8, A, 4, 4, A, 12, None, 0, None), 3),
    (lambda l: l.nm_sparse_gemm(A, 4, 8, 4, A, 4, 4, A, 8, None, 0, None), 2),
    (lambda l: l.nm_sparse_gemm(A, 4, 16, 16, A, 4, 8, A, 8, None, 0, None), 5),
    (lambda l: l.nm_sparse_gemm(A, 4, 16, 16, A, 4, 8, A, 8, MIS, 1 << 20, None), 3),
    (lambda l: l.nm_sparse_gemm_fused(A, 4, 8, 8, A, 4, 9, A, 8, None), 4),
    (lambda l: l.nm_dense_gemm(A, 4, 8, 8, None, 4, 8, A, 8, None, 0, None), 1),
    (lambda l: l.nm_dense_gemm(A, 4, 8, 8, A, 4, 8, MIS, 8, None, 0, None), 3),
    (lambda l: l.nm_dense_gemm(A, 4, 8, 8, A, 4, 8, A, 8, MIS, 1 << 20, None), 3),
    (lambda l: l.nm_dense_gemm(A, 4, 8, 4, A, 4, 8, A, 8, None, 0, None), 2),
    (lambda l: l.nm_gemm_set_schedule(3, 0), 2),
    (lambda l: l.nm_gemm_set_schedule(-1, 0), 2),
    (lambda l: l.nm_gemm_set_schedule(0, -1), 2),
    (lambda l: l.nm_gemm_set_schedule(0, 0), 0),
    (lambda l: l.nm_ternary_quantize(A, 4, 8, 8, A, A, A, 1, None), 5),
])
def test_argument_validation(call, expect):
    assert call(nm.load()) == expect


def test_binding_rejects_host_tensors_and_bad_patterns():
    # the binding marshals device tensors only: host tensors and unsupported
    # patterns are refused before any call reaches the library
    import torch
    X = torch.zeros((4, 64), dtype=torch.bfloat16)
    zb = torch.zeros((2, 2), dtype=torch.int32)
    for call in (lambda: nm.hutchinson_diag(X, zb), lambda: nm.quant_lift_f8(X, 8),
                 lambda: nm.hessian_rescale(torch.zeros(8, dtype=torch.float64), torch.ones(8, dtype=torch.float64)),
                 lambda: nm.sparse_gemm_f8(torch.zeros((4, 256), dtype=torch.uint8), torch.ones(4), X, 4, 64, 4)):
        with pytest.raises(nm.NMError):
            call()
    lib = nm.load()
    assert lib.nm_lifted_cols_f8(64, 7) == 0 and lib.nm_sparse_prepare_f8_bytes(8, 64, 12) == 0
