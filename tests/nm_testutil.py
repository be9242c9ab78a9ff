"""Helpers shared by the tests: host <-> device marshalling of bf16 bit patterns
and a host-side decoder of the packed GEMM operand (written from the layout
documented in the library's header and source, independently of its kernels)."""
from __future__ import annotations

import numpy as np
import torch


def to_dev(a: np.ndarray, ld: int | None = None) -> torch.Tensor:
    """uint16 [rows x cols] -> CUDA bf16 tensor, optionally with a padded leading dim."""
    a = np.ascontiguousarray(a, dtype=np.uint16)
    if ld is None or ld == a.shape[1]:
        return torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)
    buf = np.zeros((a.shape[0], ld), dtype=np.uint16)
    buf[:, : a.shape[1]] = a
    t = torch.from_numpy(buf.view(np.int16)).cuda().view(torch.bfloat16)
    return t[:, : a.shape[1]]


def to_host_u16(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def to_host(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.bfloat16:
        return to_host_u16(t)
    return t.contiguous().cpu().numpy()


def bf16_to_f64(u: np.ndarray) -> np.ndarray:
    return (np.asarray(u, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def rel_err(Y: np.ndarray, Y64: np.ndarray) -> float:
    """max |Y - Y64| / max |Y64| (the error metric of the GEMM outputs)."""
    denom = np.max(np.abs(Y64))
    return float(np.max(np.abs(Y - Y64)) / (denom if denom > 0 else 1.0))


def packed_geometry(R: int, K: int, m: int):
    G = (K + m - 1) // m
    nwin = G * (m // 2 - 1)
    KL = nwin * 4
    KLpad = (KL + 127) // 128 * 128
    Rpad = (R + 127) // 128 * 128
    return dict(G=G, nwin=nwin, KL=KL, KLpad=KLpad, Rpad=Rpad, nkb=KLpad // 128,
                vals_bytes=Rpad * KLpad, meta_bytes=Rpad * KLpad // 8)


def decode_packed(packed: np.ndarray, R: int, K: int, m: int):
    """Undo the GEMM operand layout: returns (vals [R x nwin*2] uint16,
    window nibbles [R x nwin] uint8, padding_ok bool).

    Metadata block b of row tile mt and K' block kb (2048 bytes): byte j holds
    the index pairs of two adjacent windows of one row; with L = j // 16 and
    w = j % 16: row = (L % 8) + 8 * ((w // 2) % 2) + 16 * (L // 16) and first
    lifted column = 8 * (w % 2) + 16 * ((L // 8) % 2) + 32 * (w // 4).
    """
    g = packed_geometry(R, K, m)
    KLh = g["KLpad"] // 2
    vals_all = packed[: g["vals_bytes"]].view(np.uint16).reshape(g["Rpad"], KLh)
    meta = packed[g["vals_bytes"]: g["vals_bytes"] + g["meta_bytes"]]
    nib = np.zeros((g["Rpad"], g["KLpad"] // 4), dtype=np.uint8)
    j = np.arange(2048)
    L, w = j // 16, j % 16
    rows = (L % 8) + 8 * ((w // 2) % 2) + 16 * (L // 16)
    cols = 8 * (w % 2) + 16 * ((L // 8) % 2) + 32 * (w // 4)
    blocks = meta.reshape(g["Rpad"] // 128, g["nkb"], 2048)
    for mt in range(g["Rpad"] // 128):
        for kb in range(g["nkb"]):
            b = blocks[mt, kb]
            win = kb * 32 + cols // 4
            nib[mt * 128 + rows, win] = b & 0xF
            nib[mt * 128 + rows, win + 1] = b >> 4
    nw = g["nwin"]
    pad_ok = bool(np.all(vals_all[R:] == 0) and np.all(vals_all[:, nw * 2:] == 0)
                  and np.all(nib[R:] == 4) and np.all(nib[:, nw:] == 4))
    return vals_all[:R, : nw * 2], nib[:R, :nw], pad_ok


def wmeta_nibbles(wmeta: np.ndarray, nwin: int) -> np.ndarray:
    lo = wmeta & 0xF
    hi = wmeta >> 4
    out = np.stack([lo, hi], axis=2).reshape(wmeta.shape[0], -1)
    return out[:, :nwin]
