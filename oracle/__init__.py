"""fp64 CPU oracle for the N:M-pruned linear layer -- TEST INFRASTRUCTURE ONLY.

Only the tests, the smoke check and the CPU-baseline leg of the benchmark may
import this package.  It shares no code with the CUDA library and never
imports it.  The arithmetic lives in ``nm_oracle.c`` (plain loops, fp64,
compiled without FMA contraction or fast-math); this module only builds that
file, marshals numpy arrays into it and shapes the outputs.

Function -> passage it follows (page title, section):
  hessian_diag     Sparsity Induction (2602.21652) sec. 2C, diagonal GN proxy
  hessian_rescale  Sparsity Induction sec. 2C, O(d_in) refresh under equivalent scaling
  hutchinson_diag  Hutchinson estimate of diag(X^T X / T) from given sign vectors
  score_hessian    SparseForge (2605.06402), Hessian-aware importance s=(H+eps)W^2
  score_magnitude  Sparse-BitNet (2603.05168) sec. 2, mask from latent magnitudes
  prune            SparseForge "Mistura Progressiva" (top-N per group);
                   Sparse-BitNet sec. 1 (N of every M consecutive weights)
  slide_pack       SlideSparse (2603.05232) sec. 2A, sliding-window decomposition
  slide_unpack     inverse of slide_pack (used for the reconstruction pin)
  lift             SlideSparse sec. 2B, activation lifting
  gemm_*           Y = X * W_sparse^T in fp64
  ternary          Sparse-BitNet sec. 1, ternary absmean quantisation
  e4m3_*, quant_lift_f8, quant_rows_f8, gemm_f8
                   SlideSparse sec. 2B / 2C: per-token FP8 quantisation fused
                   with the lift, FP8 weights, the GEMM on dequantised codes

Every function here has a pin in tests/test_oracle_pins.py; none is unpinned.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "nm_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile nm_oracle.c into liboracle.so (gcc, OpenMP, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
               "-fPIC", "-shared", _SRC, "-o", tmp, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            P, I64, I, D = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_double
            sig = {
                "oracle_hessian_diag": (None, [P, I64, I64, I64, P]),
                "oracle_hessian_rescale": (None, [P, P, I64, P]),
                "oracle_e4m3_value": (D, [ctypes.c_uint8]),
                "oracle_e4m3_encode": (ctypes.c_uint8, [ctypes.c_float]),
                "oracle_quant_lift_f8": (I, [P, I64, I64, I64, I, I64, P, P]),
                "oracle_quant_rows_f8": (None, [P, I64, I64, P, P]),
                "oracle_hutchinson_diag": (None, [P, I64, I64, I64, P, I64, P]),
                "oracle_hessian_diag_naive": (None, [P, I64, I64, I64, P]),
                "oracle_score_hessian": (None, [P, D, P, I64, I64, I64, P]),
                "oracle_score_magnitude": (None, [P, I64, I64, I64, P]),
                "oracle_prune": (I, [P, I64, P, I64, I64, I64, I, I, P, P, P]),
                "oracle_slide_pack": (I, [P, I64, I64, I, P]),
                "oracle_slide_unpack": (I, [P, P, I64, I64, I, P]),
                "oracle_lift": (I, [P, I64, I64, I64, I, P]),
                "oracle_gemm_masked": (None, [P, I64, I64, I64, P, I, P, I64, I64, P, I64, P]),
                "oracle_gemm_dense": (None, [P, I64, I64, I64, P, I64, I64, P, I64, P]),
                "oracle_gemm_lifted": (None, [P, I64, I64, P, P, I64, I64, I, P, I64, P]),
                "oracle_ternary": (D, [P, I64, I64, I64, P]),
                "oracle_f64_to_bf16": (ctypes.c_uint16, [D]),
            }
            for name, (res, args) in sig.items():
                fn = getattr(lib, name)
                fn.restype = res
                fn.argtypes = args
            _lib = lib
    return _lib


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def n_groups(K: int, m: int) -> int:
    return (K + m - 1) // m


def mask_words(K: int, m: int) -> int:
    return (n_groups(K, m) * m + 31) // 32


def lifted_cols(K: int, m: int) -> int:
    return n_groups(K, m) * (m // 2 - 1) * 4


def hessian_diag(X: np.ndarray, naive: bool = False) -> np.ndarray:
    """H [K] fp64 from X [T x K] bf16 bits: the exact column sums of squares
    rounded once to fp64, divided by T (naive: one sequential fp64 sum instead,
    a diagnostic)."""
    X = _c(X, np.uint16)
    T, K = X.shape
    H = np.empty(K, dtype=np.float64)
    fn = _load().oracle_hessian_diag_naive if naive else _load().oracle_hessian_diag
    fn(_p(X), T, K, K, _p(H))
    return H


def hessian_rescale(H: np.ndarray, s: np.ndarray) -> np.ndarray:
    """H_j / (s_j * s_j): the proxy of X diag(1/s) (Sparsity Induction sec. 2C)."""
    H = _c(H, np.float64)
    s = _c(s, np.float64)
    out = np.empty_like(H)
    _load().oracle_hessian_rescale(_p(H), _p(s), H.shape[0], _p(out))
    return out


def hutchinson_diag(X: np.ndarray, zbits: np.ndarray) -> np.ndarray:
    """(1/S) sum_s z_s * (X^T X z_s) / T in fp64, z_s = -1 where a bit is set."""
    X = _c(X, np.uint16)
    zbits = _c(zbits, np.uint32)
    T, K = X.shape
    D = np.empty(K, dtype=np.float64)
    _load().oracle_hutchinson_diag(_p(X), T, K, K, _p(zbits), zbits.shape[0], _p(D))
    return D


def score_hessian(H: np.ndarray, W: np.ndarray, eps: float) -> np.ndarray:
    H = _c(H, np.float64)
    W = _c(W, np.uint16)
    R, K = W.shape
    S = np.empty((R, K), dtype=np.float32)
    _load().oracle_score_hessian(_p(H), float(eps), _p(W), R, K, K, _p(S))
    return S


def score_magnitude(W: np.ndarray) -> np.ndarray:
    W = _c(W, np.uint16)
    R, K = W.shape
    S = np.empty((R, K), dtype=np.float32)
    _load().oracle_score_magnitude(_p(W), R, K, K, _p(S))
    return S


def prune(S: np.ndarray, V: np.ndarray, n: int, m: int):
    """Returns (mask u32 [R x words], vals bf16 [R x G*n], meta24 u8 [R x ceil(G/2)] or None)."""
    S = _c(S, np.float32)
    V = _c(V, np.uint16)
    R, K = S.shape
    G = n_groups(K, m)
    mask = np.empty((R, mask_words(K, m)), dtype=np.uint32)
    vals = np.empty((R, G * n), dtype=np.uint16)
    meta = np.empty((R, (G + 1) // 2), dtype=np.uint8) if (m == 4 and n == 2) else None
    rc = _load().oracle_prune(_p(S), K, _p(V), K, R, K, n, m, _p(mask), _p(vals),
                              _p(meta) if meta is not None else None)
    if rc != 0:
        raise ValueError("oracle_prune: unsupported n:m or invalid scores")
    return mask, vals, meta


def slide_pack(mask: np.ndarray, K: int, m: int) -> np.ndarray:
    mask = _c(mask, np.uint32)
    R = mask.shape[0]
    nw = n_groups(K, m) * (m // 2 - 1)
    wmeta = np.empty((R, (nw + 1) // 2), dtype=np.uint8)
    if _load().oracle_slide_pack(_p(mask), R, K, m, _p(wmeta)) != 0:
        raise ValueError("oracle_slide_pack: mask is not (m-2):m or window index out of range")
    return wmeta


def slide_unpack(vals: np.ndarray, wmeta: np.ndarray, K: int, m: int) -> np.ndarray:
    vals = _c(vals, np.uint16)
    wmeta = _c(wmeta, np.uint8)
    R = vals.shape[0]
    Wd = np.empty((R, K), dtype=np.uint16)
    if _load().oracle_slide_unpack(_p(vals), _p(wmeta), R, K, m, _p(Wd)) != 0:
        raise ValueError("oracle_slide_unpack: invalid window metadata")
    return Wd


def lift(X: np.ndarray, m: int) -> np.ndarray:
    X = _c(X, np.uint16)
    T, K = X.shape
    XL = np.empty((T, lifted_cols(K, m)), dtype=np.uint16)
    if _load().oracle_lift(_p(X), T, K, K, m, _p(XL)) != 0:
        raise ValueError("oracle_lift: unsupported m")
    return XL


def _rows(rows, T):
    if rows is None:
        return None, T
    rows = _c(rows, np.int64)
    return rows, rows.size


def gemm_masked(X, mask, V, m, rows=None) -> np.ndarray:
    X = _c(X, np.uint16)
    mask = _c(mask, np.uint32)
    V = _c(V, np.uint16)
    T, K = X.shape
    R = V.shape[0]
    rows, nr = _rows(rows, T)
    Y = np.empty((nr, R), dtype=np.float64)
    _load().oracle_gemm_masked(_p(X), T, K, K, _p(mask), m, _p(V), K, R,
                               _p(rows) if rows is not None else None, nr, _p(Y))
    return Y


def gemm_dense(X, Wd, rows=None) -> np.ndarray:
    X = _c(X, np.uint16)
    Wd = _c(Wd, np.uint16)
    T, K = X.shape
    R = Wd.shape[0]
    rows, nr = _rows(rows, T)
    Y = np.empty((nr, R), dtype=np.float64)
    _load().oracle_gemm_dense(_p(X), T, K, K, _p(Wd), K, R,
                              _p(rows) if rows is not None else None, nr, _p(Y))
    return Y


def gemm_lifted(XL, vals, wmeta, K, m, rows=None) -> np.ndarray:
    XL = _c(XL, np.uint16)
    vals = _c(vals, np.uint16)
    wmeta = _c(wmeta, np.uint8)
    T, KL = XL.shape
    R = vals.shape[0]
    rows, nr = _rows(rows, T)
    Y = np.empty((nr, R), dtype=np.float64)
    _load().oracle_gemm_lifted(_p(XL), T, KL, _p(vals), _p(wmeta), R, K, m,
                               _p(rows) if rows is not None else None, nr, _p(Y))
    return Y


def ternary(W: np.ndarray):
    """Returns (gamma fp64, W_q [R x K] bf16 bits)."""
    W = _c(W, np.uint16)
    R, K = W.shape
    Wq = np.empty((R, K), dtype=np.uint16)
    g = _load().oracle_ternary(_p(W), R, K, K, _p(Wq))
    if g < 0:
        raise ValueError("oracle_ternary: gamma out of bf16 normal range")
    return g, Wq


def f64_to_bf16(v: float) -> int:
    return int(_load().oracle_f64_to_bf16(float(v)))


def dense_masked(mask: np.ndarray, V: np.ndarray, K: int) -> np.ndarray:
    """mask (.) V as a dense [R x K] bf16-bit matrix (pure bit selection)."""
    R = V.shape[0]
    words = _c(mask, np.uint32)
    bits = ((words[:, :, None] >> np.arange(32, dtype=np.uint32)) & 1).reshape(R, -1)[:, :K]
    return np.where(bits.astype(bool), V[:, :K], np.uint16(0)).astype(np.uint16)


def run_layer(X, W, n, m, eps=1e-8, score="hessian", ternary_values=False):
    """Whole oracle path for one layer: H, S, mask, vals, meta, wmeta, V used."""
    H = None
    V = W
    if ternary_values:
        _, V = ternary(W)
    if score == "hessian":
        H = hessian_diag(X)
        S = score_hessian(H, W, eps)
    else:
        S = score_magnitude(W)
    mask, vals, meta = prune(S, V, n, m)
    wmeta = slide_pack(mask, W.shape[1], m) if (m % 2 == 0 and n == m - 2) else None
    return dict(H=H, S=S, mask=mask, vals=vals, meta24=meta, wmeta=wmeta, V=V)


def e4m3_value(code: int) -> float:
    return _load().oracle_e4m3_value(code)


def e4m3_encode(x: float) -> int:
    return _load().oracle_e4m3_encode(x)


def e4m3_table() -> np.ndarray:
    """fp64 value of each of the 256 codes (NaN for 0x7F and 0xFF)."""
    t = np.array([e4m3_value(c) for c in range(256)])
    t[0x7F] = t[0xFF] = np.nan
    return t


def lifted_cols_f8(K: int, m: int) -> int:
    """Lifted width rounded up to the FP8 GEMM's 256-column K' block."""
    return (lifted_cols(K, m) + 255) // 256 * 256


def quant_lift_f8(X: np.ndarray, m: int, ldq: int | None = None):
    """Per-token E4M3 codes of the lifted activations and the fp32 scales."""
    X = _c(X, np.uint16)
    T, K = X.shape
    ldq = lifted_cols_f8(K, m) if ldq is None else ldq
    Q = np.empty((T, ldq), dtype=np.uint8)
    sc = np.empty(T, dtype=np.float32)
    if _load().oracle_quant_lift_f8(_p(X), T, K, K, m, ldq, _p(Q), _p(sc)) != 0:
        raise ValueError("oracle_quant_lift_f8: unsupported m or ldq")
    return Q, sc


def quant_rows_f8(V: np.ndarray):
    """Per-row E4M3 codes of kept weight values [R x L] and the fp32 scales."""
    V = _c(V, np.uint16)
    R, L = V.shape
    Q = np.empty((R, L), dtype=np.uint8)
    sc = np.empty(R, dtype=np.float32)
    _load().oracle_quant_rows_f8(_p(V), R, L, _p(Q), _p(sc))
    return Q, sc


def gemm_f8(Xq, xs, mask, Wq, ws, K, m, rows=None) -> np.ndarray:
    """Y64[t, r] = xs[t] ws[r] sum over kept k of e4m3(Xq[t, k]) e4m3(Wq[r, j(k)])
    in fp64, Xq being the per-token codes of X in its own column order (the
    lift only duplicates columns, so each lifted code equals one of these)."""
    tab = e4m3_table()
    T = Xq.shape[0]
    sel = np.arange(T) if rows is None else np.asarray(rows)
    Xd = tab[Xq[sel, :K]]
    R = Wq.shape[0]
    words = _c(mask, np.uint32)
    bits = ((words[:, :, None] >> np.arange(32, dtype=np.uint32)) & 1).reshape(R, -1)[:, :K].astype(bool)
    Wd = np.zeros((R, K))
    for r in range(R):
        Wd[r, bits[r]] = tab[Wq[r, : bits[r].sum()]]
    return (Xd @ Wd.T) * xs[sel, None].astype(np.float64) * ws[None, :].astype(np.float64)
