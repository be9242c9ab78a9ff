"""B200 (sm_100a) N:M-pruned linear layer: Python binding of libnmsparse.so.

Argument marshalling only.  Every step of the path runs in the CUDA kernels of
``libnmsparse.so`` (declared in ``include/nmsparse.h``); PyTorch supplies device
memory and the current stream.  There is no CPU fallback: if the library is
missing and cannot be built, importing the functions below raises.

bf16 tensors may be given as ``torch.bfloat16`` or as ``torch.uint16`` /
``torch.int16`` bit patterns; outputs are ``torch.bfloat16``.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

from . import build as _build

__all__ = [
    "NMError", "load", "hessian_diag", "score", "score_from_hessian", "prune_compress",
    "score_prune_compress", "hessian_rescale", "hutchinson_diag", "quant_lift_f8", "sparse_prepare_f8",
    "sparse_gemm_f8", "slide_pack", "lift_activations", "sparse_prepare", "sparse_prepare_from_mask",
    "sparse_gemm", "dense_gemm",
    "ternary_quantize", "check_device_error", "set_gemm_schedule", "set_poison", "EXPORTED",
]

EXPORTED = (
    "nm_status_string", "nm_check_device_error", "nm_version",
    "nm_hessian_workspace_bytes", "nm_hessian_diag", "nm_score", "nm_score_from_hessian",
    "nm_prune_compress", "slide_pack", "lift_activations", "nm_sparse_prepare_bytes",
    "nm_sparse_prepare", "nm_sparse_gemm", "nm_dense_gemm", "nm_ternary_workspace_bytes",
    "nm_ternary_quantize", "nm_hessian_diag_noalloc", "nm_probe_mma", "nm_probe_copy", "nm_gemm_1cta", "nm_sparse_gemm_workspace_bytes",
    "nm_sparse_gemm_fused", "nm_dense_gemm_workspace_bytes", "nm_gemm_set_schedule",
    "nm_sparse_gemm_tile256", "nm_score_prune_compress", "nm_hessian_rescale",
    "nm_hutchinson_workspace_bytes", "nm_hutchinson_diag", "nm_lifted_cols_f8", "nm_sparse_prepare_f8_bytes",
    "nm_quant_lift_f8", "nm_sparse_prepare_f8", "nm_sparse_gemm_f8", "nm_test_set_wait_limit_ns",
    "nm_test_withhold_stream_k_flag", "nm_test_hessian_clusters", "nm_hessian_launch_count", "nm_sparse_prepare_from_mask",
)

_P, _I64, _I, _D, _SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_double, ctypes.c_size_t
_SIGS = {
    "nm_status_string": (ctypes.c_char_p, [_I]),
    "nm_check_device_error": (_I, [_P]),
    "nm_version": (_I, []),
    "nm_hessian_workspace_bytes": (_SZ, [_I64, _I64]),
    "nm_hessian_diag": (_I, [_P, _I64, _I64, _I64, _P, _P, _SZ, _P]),
    "nm_score": (_I, [_P, _I64, _I64, _P, _I64, _I64, _I64, _D, _P, _P, _P, _SZ, _P]),
    "nm_score_from_hessian": (_I, [_P, _D, _P, _I64, _I64, _I64, _P, _P]),
    "nm_prune_compress": (_I, [_P, _I64, _P, _I64, _I64, _I64, _I, _I, _P, _P, _P, _P]),
    "nm_hessian_rescale": (_I, [_P, _P, _I64, _P, _P]),
    "nm_hutchinson_workspace_bytes": (_SZ, [_I64, _I64, _I64]),
    "nm_hutchinson_diag": (_I, [_P, _I64, _I64, _I64, _P, _I64, _P, _P, _SZ, _P]),
    "nm_lifted_cols_f8": (_I64, [_I64, _I]),
    "nm_sparse_prepare_f8_bytes": (_SZ, [_I64, _I64, _I]),
    "nm_quant_lift_f8": (_I, [_P, _I64, _I64, _I64, _I, _P, _I64, _P, _P]),
    "nm_sparse_prepare_f8": (_I, [_P, _P, _I64, _I64, _I, _P, _SZ, _P]),
    "nm_sparse_gemm_f8": (_I, [_P, _I64, _I64, _I64, _P, _P, _I64, _I, _P, _I64, _P]),
    "nm_score_prune_compress": (_I, [_P, _D, _P, _I64, _P, _I64, _I64, _I64, _I, _I, _P, _P, _P, _P]),
    "slide_pack": (_I, [_P, _I64, _I64, _I, _P, _P]),
    "lift_activations": (_I, [_P, _I64, _I64, _I64, _I, _P, _I64, _P]),
    "nm_sparse_prepare_bytes": (_SZ, [_I64, _I64, _I]),
    "nm_sparse_prepare": (_I, [_P, _P, _I64, _I64, _I, _P, _SZ, _P]),
    "nm_sparse_gemm": (_I, [_P, _I64, _I64, _I64, _P, _I64, _I, _P, _I64, _P, _SZ, _P]),
    "nm_sparse_gemm_workspace_bytes": (_SZ, [_I64, _I64, _I]),
    "nm_sparse_gemm_fused": (_I, [_P, _I64, _I64, _I64, _P, _I64, _I, _P, _I64, _P]),
    "nm_sparse_gemm_tile256": (_I, [_P, _I64, _I64, _I64, _P, _I64, _I, _P, _I64, _P, _SZ, _P]),
    "nm_dense_gemm": (_I, [_P, _I64, _I64, _I64, _P, _I64, _I64, _P, _I64, _P, _SZ, _P]),
    "nm_dense_gemm_workspace_bytes": (_SZ, [_I64, _I64, _I64]),
    "nm_gemm_set_schedule": (_I, [_I, _I]),
    "nm_ternary_workspace_bytes": (_SZ, [_I64]),
    "nm_ternary_quantize": (_I, [_P, _I64, _I64, _I64, _P, _P, _P, _SZ, _P]),
    "nm_hessian_diag_noalloc": (_I, [_P, _I64, _I64, _I64, _P, _P]),
    "nm_probe_mma": (_I, [_I, _I, _I, _I, _P, _P, _P]),
    "nm_probe_copy": (_I, [_P, _P, _SZ, _I, _P]),
    "nm_gemm_1cta": (_I, [_I, _P, _I64, _I64, _I64, _P, _I64, _I64, _P, _I64, _P]),
    "nm_test_set_wait_limit_ns": (_I, [ctypes.c_ulonglong]),
    "nm_sparse_prepare_from_mask": (_I, [_P, _P, _I64, _I64, _I, _P, _SZ, _P]),
    "nm_test_withhold_stream_k_flag": (_I, [_I]),
    "nm_test_hessian_clusters": (_I, [_I]),
    "nm_hessian_launch_count": (_I, [_I64, _I64]),
}

_lock = threading.Lock()
_lib = None


class NMError(RuntimeError):
    pass


def load() -> ctypes.CDLL:
    """Load (building first if missing or stale) the CUDA library."""
    global _lib
    with _lock:
        if _lib is None:
            path = _build.build()
            if not os.path.exists(path):
                raise NMError(f"CUDA library not found at {path}")
            lib = ctypes.CDLL(path)
            for name, (res, args) in _SIGS.items():
                fn = getattr(lib, name)
                fn.restype = res
                fn.argtypes = args
            _lib = lib
    return _lib


def _check(status: int, what: str):
    if status != 0:
        msg = load().nm_status_string(status).decode()
        raise NMError(f"{what}: {msg}")


def _stream(stream=None) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


_POISON = False


def set_poison(on: bool = True) -> None:
    """Fill every output and workspace this binding allocates with 0xFF bytes
    (NaN for fp32 / fp64 / bf16, all-ones for integers) before the call, so
    that an element a kernel fails to write cannot pass a comparison by
    holding the bytes of an earlier, identical call.  For tests."""
    global _POISON
    _POISON = bool(on)


def _out(*shape, dtype, device) -> torch.Tensor:
    t = torch.empty(*shape, dtype=dtype, device=device)
    if _POISON and t.numel():
        t.view(torch.uint8).fill_(0xFF)
    return t


def _ptr(t: torch.Tensor | None):
    return None if t is None else t.data_ptr()


def _dev(t: torch.Tensor, name: str):
    if not t.is_cuda:
        raise NMError(f"{name} must be a CUDA tensor")
    return t


def _bf16(t: torch.Tensor, name: str) -> torch.Tensor:
    _dev(t, name)
    if t.dtype not in (torch.bfloat16, torch.uint16, torch.int16):
        raise NMError(f"{name} must be bf16 (or 16-bit bit patterns), got {t.dtype}")
    if t.stride(-1) != 1:
        raise NMError(f"{name} must have unit stride in its last dimension")
    return t


def _ld(t: torch.Tensor) -> int:
    return t.stride(0) if t.dim() == 2 else t.shape[-1]


def check_device_error(stream=None):
    """Synchronise and raise if a kernel recorded a timeout or a device check."""
    _check(load().nm_check_device_error(_stream(stream)), "device error word")


def hessian_diag(X, H=None, ws=None, stream=None):
    X = _bf16(X, "X")
    T, K = X.shape
    lib = load()
    if H is None:
        H = _out(K, dtype=torch.float64, device=X.device)
    need = lib.nm_hessian_workspace_bytes(T, K)
    if ws is None and need:
        ws = _out(need, dtype=torch.uint8, device=X.device)
    _check(lib.nm_hessian_diag(_ptr(X), T, K, _ld(X), _ptr(H), _ptr(ws),
                               ws.numel() * ws.element_size() if ws is not None else 0,
                               _stream(stream)), "nm_hessian_diag")
    return H


def score_from_hessian(H, W, eps, S=None, stream=None):
    W = _bf16(W, "W")
    R, K = W.shape
    if S is None:
        S = _out((R, K), dtype=torch.float32, device=W.device)
    _check(load().nm_score_from_hessian(_ptr(H), float(eps), _ptr(W), R, K, _ld(W), _ptr(S),
                                        _stream(stream)), "nm_score_from_hessian")
    return S


def score(X, W, eps=1e-8, H=None, S=None, ws=None, stream=None):
    """Hessian-aware score (X given) or latent-magnitude score (X is None).
    Returns (H or None, S)."""
    W = _bf16(W, "W")
    R, K = W.shape
    lib = load()
    if S is None:
        S = _out((R, K), dtype=torch.float32, device=W.device)
    if X is None:
        _check(lib.nm_score(None, 0, 0, _ptr(W), R, K, _ld(W), 0.0, None, _ptr(S), None, 0,
                            _stream(stream)), "nm_score")
        return None, S
    X = _bf16(X, "X")
    T = X.shape[0]
    if X.shape[1] != K:
        raise NMError("X and W disagree on K")
    if H is None:
        H = _out(K, dtype=torch.float64, device=W.device)
    need = lib.nm_hessian_workspace_bytes(T, K)
    if ws is None and need:
        ws = _out(need, dtype=torch.uint8, device=W.device)
    _check(lib.nm_score(_ptr(X), T, _ld(X), _ptr(W), R, K, _ld(W), float(eps), _ptr(H), _ptr(S),
                        _ptr(ws), ws.numel() if ws is not None else 0, _stream(stream)), "nm_score")
    return H, S


def n_groups(K, m):
    return (K + m - 1) // m


def prune_compress(S, V, n, m, K=None, stream=None):
    """Returns (mask int32 [R x words], vals bf16 [R x G*n], meta24 uint8 or None)."""
    _dev(S, "S")
    V = _bf16(V, "V")
    R, K = V.shape
    G = n_groups(K, m)
    dev = V.device
    mask = _out((R, (G * m + 31) // 32), dtype=torch.int32, device=dev)
    vals = _out((R, G * n), dtype=torch.bfloat16, device=dev)
    meta = _out((R, (G + 1) // 2), dtype=torch.uint8, device=dev) if (m == 4 and n == 2) else None
    _check(load().nm_prune_compress(_ptr(S), S.stride(0), _ptr(V), _ld(V), R, K, n, m, _ptr(mask),
                                    _ptr(vals), _ptr(meta), _stream(stream)), "nm_prune_compress")
    return mask, vals, meta


def hessian_rescale(H, s, out=None, stream=None):
    """H / s^2 per channel (fp64), the O(d_in) refresh under equivalent scaling."""
    _dev(H, "H")
    _dev(s, "s")
    out = torch.empty_like(H) if out is None else out
    _check(load().nm_hessian_rescale(_ptr(H), _ptr(s), H.shape[0], _ptr(out), _stream(stream)),
           "nm_hessian_rescale")
    return out


def hutchinson_diag(X, zbits, D=None, ws=None, stream=None):
    """Hutchinson estimate of diag(X^T X / T): X bf16 [T x K], zbits int32 /
    uint32 [S x ceil(K/32)] sign bits (set = -1).  Returns fp64 [K]."""
    X = _bf16(X, "X")
    _dev(zbits, "zbits")
    T, K = X.shape
    S = zbits.shape[0]
    if zbits.dim() != 2 or zbits.shape[1] != (K + 31) // 32 or zbits.element_size() != 4 \
            or not zbits.is_contiguous():
        raise NMError(f"zbits must be contiguous 32-bit words [S x {(K + 31) // 32}]")
    lib = load()
    need = lib.nm_hutchinson_workspace_bytes(T, K, S)
    if ws is None:
        ws = _out(max(need, 16), dtype=torch.uint8, device=X.device)
    if D is None:
        D = _out(K, dtype=torch.float64, device=X.device)
    _check(lib.nm_hutchinson_diag(_ptr(X), T, K, _ld(X), _ptr(zbits), S, _ptr(D), _ptr(ws),
                                  ws.numel() * ws.element_size(), _stream(stream)), "nm_hutchinson_diag")
    return D


def quant_lift_f8(X, m, ldq=None, stream=None):
    """Per-token E4M3 codes of the lifted activations: (Xq uint8 [T x ldq],
    xscale fp32 [T]); ldq defaults to nm_lifted_cols_f8(K, m)."""
    X = _bf16(X, "X")
    T, K = X.shape
    lib = load()
    KLf = lib.nm_lifted_cols_f8(K, m)
    if KLf == 0:
        raise NMError(f"unsupported pattern m={m} for the FP8 path")
    ldq = KLf if ldq is None else ldq
    Xq = _out((T, ldq), dtype=torch.uint8, device=X.device)
    xs = _out(T, dtype=torch.float32, device=X.device)
    _check(lib.nm_quant_lift_f8(_ptr(X), T, K, _ld(X), m, _ptr(Xq), ldq, _ptr(xs), _stream(stream)),
           "nm_quant_lift_f8")
    return Xq, xs


def sparse_prepare_f8(vals, wmeta, R, K, m, stream=None):
    """FP8 GEMM operand from the kept values and window metadata (meta24 for
    2:4): codes, kind::f8f6f4 metadata blocks and row scales in one buffer."""
    _dev(vals, "vals")
    _dev(wmeta, "wmeta")
    lib = load()
    nbytes = lib.nm_sparse_prepare_f8_bytes(R, K, m)
    if nbytes == 0:
        raise NMError(f"unsupported shape or pattern for the FP8 path (R={R}, K={K}, m={m})")
    packed = _out(nbytes, dtype=torch.uint8, device=vals.device)
    _check(lib.nm_sparse_prepare_f8(_ptr(vals), _ptr(wmeta), R, K, m, _ptr(packed), nbytes, _stream(stream)),
           "nm_sparse_prepare_f8")
    return packed


def sparse_gemm_f8(Xq, xscale, packed, R, K, m, Y=None, stream=None):
    """Y = (xscale ws) * (E4M3 lifted activations x E4M3 packed weights^T), bf16."""
    _dev(Xq, "Xq")
    T, ldq = Xq.shape
    if Y is None:
        Y = _out((T, (R + 7) // 8 * 8), dtype=torch.bfloat16, device=Xq.device)[:, :R]
    _check(load().nm_sparse_gemm_f8(_ptr(Xq), T, K, ldq, _ptr(xscale), _ptr(packed), R, m, _ptr(Y), _ld(Y),
                                    _stream(stream)), "nm_sparse_gemm_f8")
    return Y


def score_prune_compress(H, W, n, m, V=None, eps=1e-8, stream=None):
    """a2 + a3 in one pass (scores never written): H fp64 [K] or None (|W|
    scores); V defaults to W.  Returns (mask, vals, meta24 or None) exactly as
    prune_compress(score(...), V) would."""
    W = _bf16(W, "W")
    V = W if V is None else _bf16(V, "V")
    if H is not None:
        _dev(H, "H")
    R, K = W.shape
    G = n_groups(K, m)
    dev = W.device
    mask = _out((R, (G * m + 31) // 32), dtype=torch.int32, device=dev)
    vals = _out((R, G * n), dtype=torch.bfloat16, device=dev)
    meta = _out((R, (G + 1) // 2), dtype=torch.uint8, device=dev) if (m == 4 and n == 2) else None
    _check(load().nm_score_prune_compress(_ptr(H), eps, _ptr(W), _ld(W), _ptr(V), _ld(V), R, K, n, m,
                                          _ptr(mask), _ptr(vals), _ptr(meta), _stream(stream)),
           "nm_score_prune_compress")
    return mask, vals, meta


def slide_pack(mask, K, m, stream=None):
    _dev(mask, "mask")
    R = mask.shape[0]
    nw = n_groups(K, m) * (m // 2 - 1)
    wmeta = _out((R, (nw + 1) // 2), dtype=torch.uint8, device=mask.device)
    _check(load().slide_pack(_ptr(mask), R, K, m, _ptr(wmeta), _stream(stream)), "slide_pack")
    return wmeta


def lifted_cols(K, m):
    return n_groups(K, m) * (m // 2 - 1) * 4


def lift_activations(X, m, XL=None, stream=None):
    X = _bf16(X, "X")
    T, K = X.shape
    KL = lifted_cols(K, m)
    if XL is None:
        XL = _out((T, (KL + 7) // 8 * 8), dtype=torch.bfloat16, device=X.device)[:, :KL]
    _check(load().lift_activations(_ptr(X), T, K, _ld(X), m, _ptr(XL), _ld(XL), _stream(stream)),
           "lift_activations")
    return XL


def sparse_prepare(vals, wmeta, R, K, m, packed=None, stream=None):
    lib = load()
    need = lib.nm_sparse_prepare_bytes(R, K, m)
    if need == 0:
        raise NMError("nm_sparse_prepare_bytes: unsupported shape or pattern")
    if packed is None:
        packed = _out(need, dtype=torch.uint8, device=vals.device)
    _check(lib.nm_sparse_prepare(_ptr(vals), _ptr(wmeta), R, K, m, _ptr(packed),
                                 packed.numel() * packed.element_size(), _stream(stream)),
           "nm_sparse_prepare")
    return packed


def sparse_prepare_from_mask(vals, mask, R, K, m, packed=None, stream=None):
    """The GEMM operand straight from the kept values and the mask: the
    sliding-window pack and the operand preparation in one pass."""
    _dev(vals, "vals")
    _dev(mask, "mask")
    lib = load()
    need = lib.nm_sparse_prepare_bytes(R, K, m)
    if need == 0:
        raise NMError("nm_sparse_prepare_bytes: unsupported shape or pattern")
    if packed is None:
        packed = _out(need, dtype=torch.uint8, device=vals.device)
    _check(lib.nm_sparse_prepare_from_mask(_ptr(vals), _ptr(mask), R, K, m, _ptr(packed),
                                           packed.numel() * packed.element_size(), _stream(stream)),
           "nm_sparse_prepare_from_mask")
    return packed


def sparse_gemm(X, packed, R, m, Y=None, ws=None, stream=None, fused=False, tile256=False):
    """Y = X * W_sparse^T.  Ablation variants: fused=True lifts inside the GEMM,
    tile256=True uses the 256 x 256 CTA-pair tile."""
    X = _bf16(X, "X")
    T, K = X.shape
    lib = load()
    if Y is None:
        Y = _out((T, (R + 7) // 8 * 8), dtype=torch.bfloat16, device=X.device)[:, :R]
    if fused:
        _check(lib.nm_sparse_gemm_fused(_ptr(X), T, K, _ld(X), _ptr(packed), R, m, _ptr(Y),
                                        _ld(Y), _stream(stream)), "nm_sparse_gemm_fused")
        return Y
    need = lib.nm_sparse_gemm_workspace_bytes(T, K, m)
    if ws is None and need:
        ws = _out(need, dtype=torch.uint8, device=X.device)
    fn = lib.nm_sparse_gemm_tile256 if tile256 else lib.nm_sparse_gemm
    _check(fn(_ptr(X), T, K, _ld(X), _ptr(packed), R, m, _ptr(Y), _ld(Y),
              _ptr(ws), ws.numel() if ws is not None else 0, _stream(stream)),
           "nm_sparse_gemm")
    return Y


def dense_gemm(X, W, Y=None, ws=None, stream=None):
    X = _bf16(X, "X")
    W = _bf16(W, "W")
    T, K = X.shape
    R = W.shape[0]
    lib = load()
    if Y is None:
        Y = _out((T, (R + 7) // 8 * 8), dtype=torch.bfloat16, device=X.device)[:, :R]
    if ws is None:
        ws = _out(lib.nm_dense_gemm_workspace_bytes(T, K, R), dtype=torch.uint8, device=X.device)
    _check(lib.nm_dense_gemm(_ptr(X), T, K, _ld(X), _ptr(W), R, _ld(W), _ptr(Y), _ld(Y),
                             _ptr(ws), ws.numel(), _stream(stream)), "nm_dense_gemm")
    return Y


def set_gemm_schedule(policy: int = 0, clusters: int = 0) -> None:
    """GEMM schedule for this process: policy 0 automatic, 1 whole tiles only,
    2 stream-K whenever the workspace allows; clusters 0 = all that fit."""
    _check(load().nm_gemm_set_schedule(policy, clusters), "nm_gemm_set_schedule")


def ternary_quantize(W, stream=None):
    """Returns (W_q bf16 [R x K], gamma fp64 device scalar)."""
    W = _bf16(W, "W")
    R, K = W.shape
    lib = load()
    Wq = _out((R, K), dtype=torch.bfloat16, device=W.device)
    gamma = _out(1, dtype=torch.float64, device=W.device)
    ws = _out(lib.nm_ternary_workspace_bytes(R), dtype=torch.uint8, device=W.device)
    _check(lib.nm_ternary_quantize(_ptr(W), R, K, _ld(W), _ptr(Wq), _ptr(gamma), _ptr(ws),
                                   ws.numel(), _stream(stream)), "nm_ternary_quantize")
    return Wq, gamma
