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
    nkb = 3 * ((G + 31) // 32) if m == 8 else (KL + 127) // 128
    KLpad = nkb * 128
    Rpad = (R + 255) // 256 * 256
    return dict(G=G, nwin=nwin, KL=KL, KLpad=KLpad, Rpad=Rpad, nkb=nkb,
                vals_bytes=Rpad * KLpad, meta_bytes=Rpad * KLpad // 8)


def slot_windows(m: int, nkb: int):
    """(group, window) of every slot (4 lifted columns) of the packed K' order:
    natural for m in (4, 6, 10); for m = 8, per 32 groups: two blocks holding
    windows 0 and 2 of groups 0-15 and 16-31 (X's own column order), then one
    block holding window 1 of groups 0-31."""
    g = np.empty(nkb * 32, dtype=np.int64)
    w = np.empty(nkb * 32, dtype=np.int64)
    nwin = m // 2 - 1
    for kb in range(nkb):
        for s in range(32):
            if m == 8:
                j, typ = divmod(kb, 3)
                if typ < 2:
                    gg, ww = 32 * j + 16 * typ + s // 2, 2 * (s % 2)
                else:
                    gg, ww = 32 * j + s, 1
            else:
                gg, ww = divmod(32 * kb + s, nwin)
            g[kb * 32 + s], w[kb * 32 + s] = gg, ww
    return g, w


def decode_packed(packed: np.ndarray, R: int, K: int, m: int):
    """Undo the GEMM operand layout: returns (vals [R x nwin*2] uint16 and
    window nibbles [R x nwin] uint8, both in (group, window) order, and
    padding_ok: every padded row or slot holds value 0 and the pair (0,1)).

    Metadata block of row tile mt and K' block kb (2048 bytes): byte j holds
    the index pairs of two adjacent slots of one row; with L = j // 16 and
    w = j % 16: row = (L % 8) + 8 * ((w // 2) % 2) + 16 * (L // 16) and first
    lifted column = 8 * (w % 2) + 16 * ((L // 8) % 2) + 32 * (w // 4).
    """
    geo = packed_geometry(R, K, m)
    KLh = geo["KLpad"] // 2
    vals_all = packed[: geo["vals_bytes"]].view(np.uint16).reshape(geo["Rpad"], KLh)
    meta = packed[geo["vals_bytes"]: geo["vals_bytes"] + geo["meta_bytes"]]
    nslots = geo["KLpad"] // 4
    nib = np.zeros((geo["Rpad"], nslots), dtype=np.uint8)
    j = np.arange(2048)
    L, w = j // 16, j % 16
    rows = (L % 8) + 8 * ((w // 2) % 2) + 16 * (L // 16)
    cols = 8 * (w % 2) + 16 * ((L // 8) % 2) + 32 * (w // 4)
    blocks = meta.reshape(geo["Rpad"] // 128, geo["nkb"], 2048)
    for mt in range(geo["Rpad"] // 128):
        for kb in range(geo["nkb"]):
            b = blocks[mt, kb]
            slot = kb * 32 + cols // 4
            nib[mt * 128 + rows, slot] = b & 0xF
            nib[mt * 128 + rows, slot + 1] = b >> 4
    sg, sw = slot_windows(m, geo["nkb"])
    nwin_g = m // 2 - 1
    real = sg < geo["G"]
    wi = sg[real] * nwin_g + sw[real]
    order = np.argsort(wi)
    assert np.array_equal(wi[order], np.arange(geo["nwin"]))
    slot_idx = np.nonzero(real)[0][order]          # slot of window wi, in wi order
    vals = np.empty((R, geo["nwin"] * 2), dtype=np.uint16)
    vals[:, 0::2] = vals_all[:R, 2 * slot_idx]
    vals[:, 1::2] = vals_all[:R, 2 * slot_idx + 1]
    nibs = nib[:R, slot_idx]
    pad_slots = np.nonzero(~real)[0]
    pad_ok = bool(np.all(vals_all[R:] == 0) and np.all(nib[R:] == 4)
                  and np.all(vals_all[:, np.concatenate([2 * pad_slots, 2 * pad_slots + 1])] == 0)
                  and np.all(nib[:, pad_slots] == 4))
    return vals, nibs, pad_ok


def wmeta_nibbles(wmeta: np.ndarray, nwin: int) -> np.ndarray:
    lo = wmeta & 0xF
    hi = wmeta >> 4
    out = np.stack([lo, hi], axis=2).reshape(wmeta.shape[0], -1)
    return out[:, :nwin]
