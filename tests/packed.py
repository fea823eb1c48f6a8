"""Independent numpy reader of packed pools (test helper).

Splits a pool's bytes into fp16 scales, integer codes and fp16 pivot / outlier values, so
parity tests can compare codes element by element. It follows the format as the header
include/sq.h states it and uses only numpy shifts and masks.
"""
from __future__ import annotations

from functools import lru_cache

import numpy as np


def _widths(unit: int, bits: np.ndarray, H: int, dk: int) -> np.ndarray:
    if unit == 0:
        return np.repeat(np.asarray(bits, np.int64)[:, None], dk, axis=1)
    return np.asarray(bits, np.int64).reshape(H, dk)


def _plan(unit: int, bits, H: int, dk: int, dv: int, n_outliers: int):
    return _plan_cached(unit, np.asarray(bits, np.uint8).tobytes(), H, dk, dv, n_outliers)


@lru_cache(maxsize=32)
def _plan_cached(unit: int, bits_bytes: bytes, H: int, dk: int, dv: int, n_outliers: int):
    """Byte offsets of every head block and row, as the format in include/sq.h lays them out."""
    W = _widths(unit, np.frombuffer(bits_bytes, np.uint8), H, dk)
    row_off = np.zeros((H, dk), np.int64)
    head_off = np.zeros(H, np.int64)
    out_off = np.zeros(H, np.int64)
    off = 0
    for h in range(H):
        head_off[h] = off
        if unit == 0 and W[h, 0] == 16:
            size = 2 * dk * dv
        else:
            p = off + 2 * (dk + dv)
            for i in range(dk):
                row_off[h, i] = p
                p += dv * int(W[h, i]) // 8
            out_off[h] = p
            size = p + 4 * n_outliers - off
        off += (size + 15) // 16 * 16
    return W, row_off, head_off, out_off


def _fields(raw: np.ndarray, b: int, dv: int) -> np.ndarray:
    """The dv b-bit fields of each row of raw [..., dv * b / 8] (uint8), LSB first: field j
    sits at bits [j b, (j + 1) b) of the row's little-endian bit stream."""
    x = raw.astype(np.int64)
    if b == 8:
        return x
    if b == 6:  # three bytes hold four fields
        g = x.reshape(*x.shape[:-1], dv // 4, 3)
        word = g[..., 0] | (g[..., 1] << 8) | (g[..., 2] << 16)
        return ((word[..., None] >> (6 * np.arange(4))) & 63).reshape(*x.shape[:-1], dv)
    per = 8 // b  # fields per byte
    return ((x[..., None] >> (b * np.arange(per))) & ((1 << b) - 1)).reshape(*x.shape[:-1], dv)


def decode(slots: np.ndarray, unit: int, bits, H: int, dk: int, dv: int, n_outliers: int = 0):
    """slots: uint8 [n, slot_bytes]. Returns dict of arrays over [n, H, ...]:
    codes int64 [n,H,dk,dv] (0 on fp16 rows), f16 float32 [n,H,dk,dv] (fp16 values on pivot
    rows / heads, outliers, else 0), r16/c16 float64, pivot bool [H,dk], out_idx/out_val."""
    n = slots.shape[0]
    W, row_off, head_off, out_off = _plan(unit, bits, H, dk, dv, n_outliers)
    codes = np.zeros((n, H, dk, dv), np.int64)
    f16 = np.zeros((n, H, dk, dv), np.float32)
    r16 = np.zeros((n, H, dk))
    c16 = np.ones((n, H, dv))
    outliers = np.zeros((n, H, n_outliers), np.int64)
    for h in range(H):
        off = head_off[h]
        if unit == 0 and W[h, 0] == 16:
            blk = slots[:, off:off + 2 * dk * dv]
            f16[:, h] = blk.copy().view(np.float16).reshape(n, dk, dv).astype(np.float32)
        else:
            r16[:, h] = slots[:, off:off + 2 * dk].copy().view(np.float16).astype(np.float64)
            c16[:, h] = slots[:, off + 2 * dk:off + 2 * (dk + dv)].copy().view(
                np.float16).astype(np.float64)
    quant_rows = ~((W == 16) & (np.asarray([unit == 0] * H)[:, None]))
    for b in (2, 4, 6, 8, 16):  # all rows of one width at once
        hs, rs = np.nonzero((W == b) & quant_rows)
        if hs.size == 0:
            continue
        nb = dv * b // 8
        raw = slots[:, row_off[hs, rs][:, None] + np.arange(nb)[None, :]]  # [n, rows, nb]
        if b == 16:
            f16[:, hs, rs] = raw.copy().view(np.float16).astype(np.float32)
        else:
            codes[:, hs, rs] = _fields(raw, b, dv) - (1 << (b - 1))
    for h in range(H):
        if unit == 0 and W[h, 0] == 16:
            continue
        p = out_off[h]
        for t in range(n_outliers):
            idx = slots[:, p + 4 * t:p + 4 * t + 2].copy().view(np.uint16)[:, 0].astype(np.int64)
            val = slots[:, p + 4 * t + 2:p + 4 * t + 4].copy().view(np.float16)[:, 0]
            outliers[:, h, t] = idx
            f16[np.arange(n), h, idx // dv, idx % dv] = val.astype(np.float32)
    pivot = W == 16
    return dict(codes=codes, f16=f16, r16=r16, c16=c16, pivot=pivot, outliers=outliers,
                widths=W)


def head_ranges(unit: int, bits, H: int, dk: int, dv: int, n_outliers: int = 0):
    """[(start, end)] byte range of each head block within a slot (end includes the padding)."""
    W, _, head_off, _ = _plan(unit, bits, H, dk, dv, n_outliers)
    ends = list(head_off[1:]) + [None]
    out = []
    for h in range(H):
        if ends[h] is None:
            if unit == 0 and W[h, 0] == 16:
                size = 2 * dk * dv
            else:
                size = 2 * (dk + dv) + sum(dv * int(b) // 8 for b in W[h]) + 4 * n_outliers
            ends[h] = head_off[h] + (size + 15) // 16 * 16
        out.append((int(head_off[h]), int(ends[h])))
    return out


def head_bits(unit: int, bits, h: int, dk: int) -> np.ndarray:
    """The bit map of head h alone (a one-head layout)."""
    b = np.asarray(bits, np.uint8)
    return b[h:h + 1] if unit == 0 else b[h * dk:(h + 1) * dk]


def dequant(d) -> np.ndarray:
    """fp32 state from a decoded pool: code * r16 * c16, fp16 values where stored."""
    D = (d["codes"] * d["r16"][..., None] * d["c16"][:, :, None, :]).astype(np.float32)
    piv = np.broadcast_to(d["pivot"][None, :, :, None], D.shape)
    D = np.where(piv, d["f16"], D)
    n, H, K = d["outliers"].shape
    if K:
        dv = D.shape[-1]
        for b in range(n):
            for h in range(H):
                idx = d["outliers"][b, h]
                D[b, h, idx // dv, idx % dv] = d["f16"][b, h, idx // dv, idx % dv]
    return D
