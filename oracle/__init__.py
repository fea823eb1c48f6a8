"""Python access to the CPU oracle (test infrastructure only).

Only the tests, ``__graft_entry__.smoke()`` and the bench's CPU-baseline leg import this
package. It wraps ``liboracle.so`` (plain C, see ``sq_oracle.c``) with numpy arrays and holds
no arithmetic of its own beyond argument marshalling.
"""
from __future__ import annotations

import ctypes as C
import os
from dataclasses import dataclass, field

import numpy as np

from . import build as _build

ORC_OK, ORC_ERR_ARG, ORC_ERR_NONFINITE, ORC_ERR_RANGE = 0, 1, 2, 3
UNIT_HEAD, UNIT_ROW = 0, 1
GATE_SCALAR, GATE_DIAG = 0, 1


class OracleError(RuntimeError):
    pass


class _Layout(C.Structure):
    _fields_ = [(n, C.c_int32) for n in
                ("n_heads", "d_k", "d_v", "unit", "gate", "fit_iters", "window", "n_outliers")
                ] + [("omega", C.c_void_p)]


@dataclass(frozen=True)
class Layout:
    n_heads: int
    d_k: int
    d_v: int
    unit: int = UNIT_HEAD
    gate: int = GATE_SCALAR
    fit_iters: int = 2
    window: int = 1
    n_outliers: int = 0
    row_impact: object = field(default=None, compare=False, hash=False)  # [n_heads][d_k] > 0

    def omega(self):
        """Column-pass weights of the impact-weighted fit (orc_impact_weights), or None."""
        if self.row_impact is None:
            return None
        return impact_weights(self.row_impact, self.n_heads, self.d_k)

    def c(self) -> _Layout:
        lay = _Layout(self.n_heads, self.d_k, self.d_v, self.unit, self.gate, self.fit_iters,
                      self.window, self.n_outliers, None)
        om = self.omega()
        if om is not None:
            lay.omega = om.ctypes.data
            lay.keep = om  # the table lives as long as the structure
        return lay

    @property
    def alpha_width(self) -> int:
        return 1 if self.gate == GATE_SCALAR else self.d_k


_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = C.CDLL(path)
        P = C.c_void_p
        sig = {
            "orc_validate": [P, P],
            "orc_row_bytes": [C.c_int, C.c_int],
            "orc_head_bytes": [P, P, C.c_int],
            "orc_slot_layout": [P, P, P, P],
            "orc_pack_row": [C.c_int, C.c_int, P, P],
            "orc_unpack_row": [C.c_int, C.c_int, P, P],
            "orc_f32_to_f16_bits": [C.c_float],
            "orc_f16_bits_to_f32": [C.c_uint16],
            "orc_fit": [C.c_int, C.c_int, C.c_int, P, P, P, P, P, P],
            "orc_impact_weights": [C.c_int, C.c_int, P, P],
            "orc_select_outliers": [C.c_int, C.c_int, P, P, C.c_int, P],
            "orc_quantize_head": [P, P, C.c_int, P, P],
            "orc_dequantize_head": [P, P, C.c_int, P, P],
            "orc_delta_update": [C.c_int, C.c_int, C.c_int, P, P, P, P, P, C.c_double, P],
            "orc_quantize": [P, P, P, P, C.c_int, P, C.c_int],
            "orc_dequantize": [P, P, P, P, C.c_int, P, C.c_int],
            "orc_decode_step": [P, P, P, P, C.c_int, P, P, P, P, P, P, P, C.c_int],
            "orc_window_step": [P, P, P, P, C.c_int, P, P, P, P, P, P, P, P, C.c_int],
            "orc_window_flush": [P, P, P, P, C.c_int, P, P, C.c_int],
            "orc_allocate_bits": [C.c_int, P, P, C.c_double, C.c_int, P, P],
        }
        for name, args in sig.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = C.c_int
        L.orc_row_bytes.restype = C.c_size_t
        L.orc_head_bytes.restype = C.c_size_t
        L.orc_f32_to_f16_bits.restype = C.c_uint16
        L.orc_f16_bits_to_f32.restype = C.c_float
        L.orc_delta_update.restype = None
        L.orc_pack_row.restype = None
        L.orc_unpack_row.restype = None
        _lib = L
    return _lib


def _p(a: np.ndarray):
    return a.ctypes.data_as(C.c_void_p)


def _chk(st: int, what: str):
    if st != ORC_OK:
        raise OracleError(f"{what}: oracle status {st}")


def default_threads() -> int:
    return len(os.sched_getaffinity(0))


def _bits(bits) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(bits, dtype=np.uint8))


def validate(layout: Layout, bits) -> int:
    b = _bits(bits)
    lay = layout.c()
    return lib().orc_validate(C.byref(lay), _p(b))


def slot_layout(layout: Layout, bits):
    """(head offsets [H] int64, slot bytes)."""
    b = _bits(bits)
    lay = layout.c()
    off = np.zeros(layout.n_heads, dtype=np.uint64)
    sb = C.c_size_t(0)
    _chk(lib().orc_slot_layout(C.byref(lay), _p(b), _p(off), C.byref(sb)), "slot_layout")
    return off.astype(np.int64), int(sb.value)


def row_bytes(b: int, d_v: int) -> int:
    return int(lib().orc_row_bytes(b, d_v))


def pack_row(b: int, u) -> np.ndarray:
    u = np.ascontiguousarray(np.asarray(u, dtype=np.int32))
    out = np.zeros(row_bytes(b, u.size), dtype=np.uint8)
    lib().orc_pack_row(b, u.size, _p(u), _p(out))
    return out


def unpack_row(b: int, n: int, data) -> np.ndarray:
    d = np.ascontiguousarray(np.asarray(data, dtype=np.uint8))
    u = np.zeros(n, dtype=np.int32)
    lib().orc_unpack_row(b, n, _p(d), _p(u))
    return u


def f32_to_f16_bits(x: float) -> int:
    return int(lib().orc_f32_to_f16_bits(float(x)))


def fit(S: np.ndarray, qmax, fit_iters: int = 2, excluded=None, omega=None):
    """(r, c) of the dual-axis fit; omega: optional per-row column-pass weights in (0, 1]."""
    S = np.ascontiguousarray(S, dtype=np.float32)
    dk, dv = S.shape
    q = np.ascontiguousarray(np.asarray(qmax, dtype=np.int32))
    ex = None if excluded is None else np.ascontiguousarray(np.asarray(excluded, dtype=np.uint8))
    om = None if omega is None else np.ascontiguousarray(np.asarray(omega, dtype=np.float32))
    r = np.zeros(dk, dtype=np.float32)
    c = np.zeros(dv, dtype=np.float32)
    _chk(lib().orc_fit(dk, dv, fit_iters, _p(S), _p(q), None if ex is None else _p(ex),
                       None if om is None else _p(om), _p(r), _p(c)), "fit")
    return r, c


def impact_weights(impact, n_heads: int, d_k: int) -> np.ndarray:
    """Column-pass weights [n_heads][d_k] of the impact-weighted fit from row impact scores."""
    imp = np.ascontiguousarray(np.asarray(impact, dtype=np.float32).reshape(n_heads, d_k))
    om = np.zeros((n_heads, d_k), dtype=np.float32)
    _chk(lib().orc_impact_weights(n_heads, d_k, _p(imp), _p(om)), "impact_weights")
    return om


def select_outliers(S: np.ndarray, qmax, n: int) -> np.ndarray:
    S = np.ascontiguousarray(S, dtype=np.float32)
    dk, dv = S.shape
    q = np.ascontiguousarray(np.asarray(qmax, dtype=np.int32))
    idx = np.zeros(max(n, 1), dtype=np.int32)
    _chk(lib().orc_select_outliers(dk, dv, _p(S), _p(q), n, _p(idx)), "select_outliers")
    return idx[:n]


def quantize_head(layout: Layout, bits, h: int, S: np.ndarray) -> np.ndarray:
    b = _bits(bits)
    lay = layout.c()
    S = np.ascontiguousarray(S, dtype=np.float32)
    blk = np.zeros(int(lib().orc_head_bytes(C.byref(lay), _p(b), h)), dtype=np.uint8)
    _chk(lib().orc_quantize_head(C.byref(lay), _p(b), h, _p(S), _p(blk)), "quantize_head")
    return blk


def dequantize_head(layout: Layout, bits, h: int, block: np.ndarray) -> np.ndarray:
    b = _bits(bits)
    lay = layout.c()
    blk = np.ascontiguousarray(block, dtype=np.uint8)
    S = np.zeros((layout.d_k, layout.d_v), dtype=np.float32)
    _chk(lib().orc_dequantize_head(C.byref(lay), _p(b), h, _p(blk), _p(S)), "dequantize_head")
    return S


def delta_update(M: np.ndarray, q, k, v, alpha, beta: float, gate: int = GATE_SCALAR):
    """Exact (fp64) gated delta-rule update of M in place; returns o."""
    assert M.dtype == np.float64 and M.flags.c_contiguous
    dk, dv = M.shape
    q = np.ascontiguousarray(q, dtype=np.float64)
    k = np.ascontiguousarray(k, dtype=np.float64)
    v = np.ascontiguousarray(v, dtype=np.float64)
    a = np.ascontiguousarray(np.atleast_1d(alpha), dtype=np.float64)
    o = np.zeros(dv, dtype=np.float64)
    lib().orc_delta_update(dk, dv, gate, _p(M), _p(q), _p(k), _p(v), _p(a), float(beta), _p(o))
    return o


class Pool:
    """A host-side pool of packed slots, advanced by the oracle."""

    def __init__(self, layout: Layout, bits, n_slots: int):
        self.layout = layout
        self.bits = _bits(bits)
        self.head_off, self.slot_bytes = slot_layout(layout, self.bits)
        self.n_slots = n_slots
        self.data = np.zeros(n_slots * self.slot_bytes, dtype=np.uint8)
        self._lay = layout.c()
        self.wstate = None
        self.count = np.zeros(n_slots, dtype=np.int32)
        if layout.window > 1 or layout.n_outliers > 0:
            self.wstate = np.zeros((n_slots, layout.n_heads, layout.d_k, layout.d_v),
                                   dtype=np.float64)

    def slot(self, s: int) -> np.ndarray:
        return self.data[s * self.slot_bytes:(s + 1) * self.slot_bytes]

    def quantize(self, slot_idx, S: np.ndarray, threads: int | None = None):
        si = np.ascontiguousarray(np.asarray(slot_idx, dtype=np.int32))
        S = np.ascontiguousarray(S, dtype=np.float32)
        assert S.shape == (si.size, self.layout.n_heads, self.layout.d_k, self.layout.d_v)
        _chk(lib().orc_quantize(C.byref(self._lay), _p(self.bits), _p(self.data), _p(si),
                                si.size, _p(S), threads or default_threads()), "quantize")
        self.count[si] = 0

    def dequantize(self, slot_idx, threads: int | None = None) -> np.ndarray:
        si = np.ascontiguousarray(np.asarray(slot_idx, dtype=np.int32))
        S = np.zeros((si.size, self.layout.n_heads, self.layout.d_k, self.layout.d_v),
                     dtype=np.float32)
        _chk(lib().orc_dequantize(C.byref(self._lay), _p(self.bits), _p(self.data), _p(si),
                                  si.size, _p(S), threads or default_threads()), "dequantize")
        return S

    def _io(self, slot_idx, q, k, v, alpha, beta):
        si = np.ascontiguousarray(np.asarray(slot_idx, dtype=np.int32))
        B, H = si.size, self.layout.n_heads
        f = lambda a: np.ascontiguousarray(a, dtype=np.float32)
        q, k, v, alpha, beta = f(q), f(k), f(v), f(alpha), f(beta)
        assert q.shape == (B, H, self.layout.d_k) and k.shape == q.shape
        assert v.shape == (B, H, self.layout.d_v)
        assert alpha.size == B * H * self.layout.alpha_width and beta.size == B * H
        return si, q, k, v, alpha, beta

    def decode_step(self, slot_idx, q, k, v, alpha, beta, want_state: bool = False,
                    threads: int | None = None):
        """One per-step decode over the batch; returns o (fp64) and optionally S_new (fp32)."""
        si, q, k, v, alpha, beta = self._io(slot_idx, q, k, v, alpha, beta)
        B, H = si.size, self.layout.n_heads
        o = np.zeros((B, H, self.layout.d_v), dtype=np.float64)
        sn = (np.zeros((B, H, self.layout.d_k, self.layout.d_v), dtype=np.float32)
              if want_state else None)
        _chk(lib().orc_decode_step(C.byref(self._lay), _p(self.bits), _p(self.data), _p(si), B,
                                   _p(q), _p(k), _p(v), _p(alpha), _p(beta), _p(o),
                                   None if sn is None else _p(sn),
                                   threads or default_threads()), "decode_step")
        return (o, sn) if want_state else o

    def window_step(self, slot_idx, q, k, v, alpha, beta, threads: int | None = None):
        si, q, k, v, alpha, beta = self._io(slot_idx, q, k, v, alpha, beta)
        B, H = si.size, self.layout.n_heads
        o = np.zeros((B, H, self.layout.d_v), dtype=np.float64)
        _chk(lib().orc_window_step(C.byref(self._lay), _p(self.bits), _p(self.data), _p(si), B,
                                   _p(q), _p(k), _p(v), _p(alpha), _p(beta), _p(o),
                                   _p(self.wstate), _p(self.count),
                                   threads or default_threads()), "window_step")
        return o

    def window_flush(self, slot_idx, threads: int | None = None):
        si = np.ascontiguousarray(np.asarray(slot_idx, dtype=np.int32))
        _chk(lib().orc_window_flush(C.byref(self._lay), _p(self.bits), _p(self.data), _p(si),
                                    si.size, _p(self.wstate), _p(self.count),
                                    threads or default_threads()), "window_flush")


def allocate_bits(variance, lifetime, avg_bits: float, n_pivots: int = 0):
    """The optimal widths under the budget (exact dynamic program): (bits, objective)."""
    var = np.ascontiguousarray(np.asarray(variance, dtype=np.float64))
    life = np.ascontiguousarray(np.asarray(lifetime, dtype=np.float64))
    bits = np.zeros(var.size, dtype=np.uint8)
    obj = C.c_double(0.0)
    _chk(lib().orc_allocate_bits(var.size, _p(var), _p(life), float(avg_bits), int(n_pivots),
                                 _p(bits), C.byref(obj)), "allocate_bits")
    return bits, float(obj.value)
