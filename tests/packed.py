"""Independent numpy reader of packed pools (test helper).

Splits a pool's bytes into fp16 scales, integer codes and fp16 pivot / outlier values, so
parity tests can compare codes element by element. It follows the format as the header
include/sq.h states it and uses only numpy bit unpacking.
"""
from __future__ import annotations

import numpy as np


def _widths(unit: int, bits: np.ndarray, H: int, dk: int) -> np.ndarray:
    if unit == 0:
        return np.repeat(np.asarray(bits, np.int64)[:, None], dk, axis=1)
    return np.asarray(bits, np.int64).reshape(H, dk)


def decode(slots: np.ndarray, unit: int, bits, H: int, dk: int, dv: int, n_outliers: int = 0):
    """slots: uint8 [n, slot_bytes]. Returns dict of arrays over [n, H, ...]:
    codes int64 [n,H,dk,dv] (0 on fp16 rows), f16 float32 [n,H,dk,dv] (fp16 values on pivot
    rows / heads, outliers, else 0), r16/c16 float64, pivot bool [H,dk], out_idx/out_val."""
    n = slots.shape[0]
    W = _widths(unit, bits, H, dk)
    codes = np.zeros((n, H, dk, dv), np.int64)
    f16 = np.zeros((n, H, dk, dv), np.float32)
    r16 = np.zeros((n, H, dk))
    c16 = np.ones((n, H, dv))
    outliers = np.zeros((n, H, n_outliers), np.int64)
    off = 0
    for h in range(H):
        pivot_head = unit == 0 and W[h, 0] == 16
        start = off
        if pivot_head:
            blk = slots[:, off:off + 2 * dk * dv]
            f16[:, h] = blk.copy().view(np.float16).reshape(n, dk, dv).astype(np.float32)
            size = 2 * dk * dv
        else:
            r16[:, h] = slots[:, off:off + 2 * dk].copy().view(np.float16).astype(np.float64)
            c16[:, h] = slots[:, off + 2 * dk:off + 2 * dk + 2 * dv].copy().view(
                np.float16).astype(np.float64)
            p = off + 2 * (dk + dv)
            for i in range(dk):
                b = int(W[h, i])
                nb = dv * b // 8
                raw = slots[:, p:p + nb]
                if b == 16:
                    f16[:, h, i] = raw.copy().view(np.float16).astype(np.float32)
                else:
                    bitsarr = np.unpackbits(raw, axis=1, bitorder="little")[:, :dv * b]
                    u = (bitsarr.reshape(n, dv, b).astype(np.int64) << np.arange(b)).sum(-1)
                    codes[:, h, i] = u - (1 << (b - 1))
                p += nb
            for t in range(n_outliers):
                idx = slots[:, p + 4 * t:p + 4 * t + 2].copy().view(np.uint16)[:, 0].astype(np.int64)
                val = slots[:, p + 4 * t + 2:p + 4 * t + 4].copy().view(np.float16)[:, 0]
                outliers[:, h, t] = idx
                f16[np.arange(n), h, idx // dv, idx % dv] = val.astype(np.float32)
            size = p + 4 * n_outliers - off
        off = start + (size + 15) // 16 * 16
    pivot = W == 16
    return dict(codes=codes, f16=f16, r16=r16, c16=c16, pivot=pivot, outliers=outliers,
                widths=W)


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
