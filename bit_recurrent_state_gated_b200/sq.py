"""ctypes binding of libsq (include/sq.h), argument marshalling only.

The functions carry the C names and take raw device addresses (ints) and a stream handle;
``StatePool`` wraps a pool whose device buffer is a torch uint8 tensor, passing tensors'
``data_ptr()`` and the current CUDA stream. Every step of the decode path runs in libsq's
kernels: if ``libsq.so`` is missing, loading it raises, and there is no other code path.
"""
from __future__ import annotations

import ctypes as C
import os
import re
from dataclasses import dataclass

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libsq.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "sq.h")

SQ_OK, SQ_ERR_INVALID_ARG, SQ_ERR_UNSUPPORTED, SQ_ERR_CUDA, SQ_ERR_OOM = 0, 1, 2, 3, 4
SQ_ERR_DEVICE_FLAG, SQ_ERR_TIMEOUT = 5, 6
SQ_GATE_SCALAR, SQ_GATE_DIAG = 0, 1
SQ_UNIT_HEAD, SQ_UNIT_KEY_ROW = 0, 1
SQ_IO_F32, SQ_IO_BF16 = 0, 1
SQ_FLAG_BAD_SLOT, SQ_FLAG_NONFINITE, SQ_FLAG_RANGE, SQ_FLAG_TIMEOUT = 1, 2, 4, 8


class SqError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {sq_status_string(status)} ({status})")
        self.status = status


class sq_layout(C.Structure):
    _fields_ = [(n, C.c_int32) for n in ("n_slots", "n_heads", "d_k", "d_v", "unit", "gate",
                                         "io_dtype", "fit_iters", "window", "n_outliers")]


@dataclass(frozen=True)
class Layout:
    n_slots: int
    n_heads: int
    d_k: int
    d_v: int
    unit: int = SQ_UNIT_HEAD
    gate: int = SQ_GATE_SCALAR
    io_dtype: int = SQ_IO_BF16
    fit_iters: int = 2
    window: int = 1
    n_outliers: int = 0

    def c(self) -> sq_layout:
        return sq_layout(self.n_slots, self.n_heads, self.d_k, self.d_v, self.unit, self.gate,
                         self.io_dtype, self.fit_iters, self.window, self.n_outliers)


_lib = None


def exported_names() -> list[str]:
    """Names of the functions include/sq.h declares."""
    with open(HEADER) as f:
        text = f.read()
    return re.findall(r"SQ_API\s+[\w\s\*]+?\b(sq_\w+)\s*\(", text)


def lib() -> C.CDLL:
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"libsq.so not built ({LIB_PATH}); run "
                           "`python -m bit_recurrent_state_gated_b200.build` first")
    L = C.CDLL(LIB_PATH)
    P, I32, SZ = C.c_void_p, C.c_int32, C.c_size_t
    sigs = {
        "sq_pool_required_bytes": [P, P, P, C.POINTER(SZ)],
        "sq_state_pool_create": [P, P, P, P, SZ, C.POINTER(P)],
        "sq_state_pool_destroy": [P],
        "sq_pool_info": [P, C.POINTER(SZ), P, C.POINTER(SZ)],
        "sq_quantize_fp32_state": [P, P, I32, P, P],
        "sq_dequantize_state": [P, P, I32, P, P],
        "sq_decode_step": [P, P, I32, P, P, P, P, P, P, P],
        "sq_window_flush": [P, P, I32, P],
        "sq_decode_chunk": [P, P, I32, I32, P, P, P, P, P, P, P],
        "sq_decode_step_split": [P, P, I32, P, P, P, P, P, P, P, P, P],
        "sq_decode_step_split_static": [P, P, I32, P, P, P, P, P, P, P],
        "sq_pool_set_row_impact": [P, P],
        "sq_pool_status": [P, C.POINTER(I32)],
        "sq_debug_decode_step_fp32": [P, P, I32, P, P, P, P, P, P, P, P],
        "sq_allocate_bits": [I32, P, P, C.c_float, I32, P, P],
        "sq_debug_set_wait": [P, C.c_uint64, C.c_uint32],
        "sq_debug_set_full_fit": [P, I32],
    }
    for name, args in sigs.items():
        fn = getattr(L, name)
        fn.argtypes = args
        fn.restype = C.c_int
    L.sq_status_string.argtypes = [C.c_int]
    L.sq_status_string.restype = C.c_char_p
    _lib = L
    return L


def _u8(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.uint8))


def _chk(st: int, what: str):
    if st != SQ_OK:
        raise SqError(st, what)


# ---- the C functions, one by one -----------------------------------------------------------

def sq_status_string(status: int) -> str:
    return lib().sq_status_string(int(status)).decode()


def sq_pool_required_bytes(layout: Layout, bits_map, pivot_mask=None) -> int:
    b = _u8(bits_map)
    pm = None if pivot_mask is None else _u8(pivot_mask)
    n = C.c_size_t(0)
    lay = layout.c()
    _chk(lib().sq_pool_required_bytes(C.byref(lay), b.ctypes.data,
                                      None if pm is None else pm.ctypes.data, C.byref(n)),
         "sq_pool_required_bytes")
    return int(n.value)


def sq_state_pool_create(layout: Layout, bits_map, pivot_mask, device_buf: int,
                         device_buf_bytes: int) -> int:
    b = _u8(bits_map)
    pm = None if pivot_mask is None else _u8(pivot_mask)
    h = C.c_void_p(0)
    lay = layout.c()
    _chk(lib().sq_state_pool_create(C.byref(lay), b.ctypes.data,
                                    None if pm is None else pm.ctypes.data, device_buf,
                                    device_buf_bytes, C.byref(h)), "sq_state_pool_create")
    return int(h.value)


def sq_state_pool_destroy(pool: int) -> None:
    _chk(lib().sq_state_pool_destroy(pool), "sq_state_pool_destroy")


def sq_pool_info(pool: int, n_heads: int):
    sb, side = C.c_size_t(0), C.c_size_t(0)
    off = np.zeros(n_heads, dtype=np.uint64)
    _chk(lib().sq_pool_info(pool, C.byref(sb), off.ctypes.data, C.byref(side)), "sq_pool_info")
    return int(sb.value), off.astype(np.int64), int(side.value)


def sq_quantize_fp32_state(pool: int, slot_idx: int, n: int, S: int, stream: int) -> None:
    _chk(lib().sq_quantize_fp32_state(pool, slot_idx, n, S, stream), "sq_quantize_fp32_state")


def sq_dequantize_state(pool: int, slot_idx: int, n: int, S_out: int, stream: int) -> None:
    _chk(lib().sq_dequantize_state(pool, slot_idx, n, S_out, stream), "sq_dequantize_state")


def sq_decode_step(pool: int, slot_idx: int, batch: int, q: int, k: int, v: int, alpha: int,
                   beta: int, out: int, stream: int) -> None:
    _chk(lib().sq_decode_step(pool, slot_idx, batch, q, k, v, alpha, beta, out, stream),
         "sq_decode_step")


def sq_decode_step_split(pool: int, slot_idx: int, batch: int, q: int, k: int, v: int,
                         alpha: int, beta: int, out: int, staging: int, stream: int,
                         side_stream: int) -> None:
    _chk(lib().sq_decode_step_split(pool, slot_idx, batch, q, k, v, alpha, beta, out, staging,
                                    stream, side_stream), "sq_decode_step_split")


def sq_decode_step_split_static(pool: int, slot_idx: int, batch: int, q: int, k: int, v: int,
                                alpha: int, beta: int, out: int, stream: int) -> None:
    """The split step with libsq's own 32 MiB staging array (for callers that cannot
    allocate device memory)."""
    _chk(lib().sq_decode_step_split_static(pool, slot_idx, batch, q, k, v, alpha, beta, out,
                                           stream), "sq_decode_step_split_static")


def sq_pool_set_row_impact(pool: int, impact) -> None:
    """impact: [n_heads][d_k] positive scores (host), or None to remove the weighting."""
    if impact is None:
        _chk(lib().sq_pool_set_row_impact(pool, None), "sq_pool_set_row_impact")
        return
    a = np.ascontiguousarray(np.asarray(impact, dtype=np.float32))
    _chk(lib().sq_pool_set_row_impact(pool, a.ctypes.data), "sq_pool_set_row_impact")


def sq_decode_chunk(pool: int, slot_idx: int, batch: int, n_tokens: int, q: int, k: int, v: int,
                    alpha: int, beta: int, out: int, stream: int) -> None:
    _chk(lib().sq_decode_chunk(pool, slot_idx, batch, n_tokens, q, k, v, alpha, beta, out,
                               stream), "sq_decode_chunk")


def sq_debug_decode_step_fp32(pool: int, slot_idx: int, batch: int, q: int, k: int, v: int,
                              alpha: int, beta: int, out: int, s_new: int, stream: int) -> None:
    _chk(lib().sq_debug_decode_step_fp32(pool, slot_idx, batch, q, k, v, alpha, beta, out,
                                         s_new, stream), "sq_debug_decode_step_fp32")


def sq_debug_set_wait(pool: int, wait_limit_ns: int, extra_expected_bytes: int) -> None:
    _chk(lib().sq_debug_set_wait(pool, int(wait_limit_ns), int(extra_expected_bytes)),
         "sq_debug_set_wait")


def sq_debug_set_full_fit(pool: int, full_fit: int) -> None:
    _chk(lib().sq_debug_set_full_fit(pool, int(full_fit)), "sq_debug_set_full_fit")


def sq_window_flush(pool: int, slot_idx: int, n: int, stream: int) -> None:
    _chk(lib().sq_window_flush(pool, slot_idx, n, stream), "sq_window_flush")


def sq_allocate_bits(variance, lifetime, avg_bits: float, n_pivots: int = 0):
    """Unit widths under an average budget (host): returns (bits_map, pivot_mask) uint8."""
    var = np.ascontiguousarray(np.asarray(variance, dtype=np.float32))
    life = np.ascontiguousarray(np.asarray(lifetime, dtype=np.float32))
    if var.shape != life.shape or var.ndim != 1:
        raise ValueError("variance and lifetime must be 1-D arrays of one length")
    bits = np.zeros(var.size, dtype=np.uint8)
    piv = np.zeros(var.size, dtype=np.uint8)
    _chk(lib().sq_allocate_bits(var.size, var.ctypes.data, life.ctypes.data, float(avg_bits),
                                int(n_pivots), bits.ctypes.data, piv.ctypes.data),
         "sq_allocate_bits")
    return bits, piv


def sq_pool_status(pool: int) -> tuple[int, int]:
    """(status, device flag word); the flag is cleared."""
    f = C.c_int32(0)
    st = lib().sq_pool_status(pool, C.byref(f))
    return int(st), int(f.value)


# ---- a pool over a torch buffer ------------------------------------------------------------

class StatePool:
    """A pool of packed states in a torch uint8 device buffer, driven through libsq."""

    def __init__(self, layout: Layout, bits_map, pivot_mask=None, device=None):
        import torch

        self.layout = layout
        self.bits = _u8(bits_map)
        self.nbytes = sq_pool_required_bytes(layout, self.bits, pivot_mask)
        self.buf = torch.zeros(self.nbytes, dtype=torch.uint8, device=device or "cuda")
        self.handle = sq_state_pool_create(layout, self.bits, pivot_mask, self.buf.data_ptr(),
                                           self.nbytes)
        self.slot_bytes, self.head_offsets, self.side_bytes = sq_pool_info(self.handle,
                                                                           layout.n_heads)

    @staticmethod
    def _stream() -> int:
        import torch
        return torch.cuda.current_stream().cuda_stream

    def close(self):
        if getattr(self, "handle", 0):
            sq_state_pool_destroy(self.handle)
            self.handle = 0

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def slots_view(self):
        """The slot region as a [n_slots, slot_bytes] uint8 tensor view."""
        n = self.layout.n_slots * self.slot_bytes
        return self.buf[:n].view(self.layout.n_slots, self.slot_bytes)

    def quantize(self, slot_idx, S):
        sq_quantize_fp32_state(self.handle, slot_idx.data_ptr(), slot_idx.numel(), S.data_ptr(),
                               self._stream())

    def dequantize(self, slot_idx, S_out):
        sq_dequantize_state(self.handle, slot_idx.data_ptr(), slot_idx.numel(),
                            S_out.data_ptr(), self._stream())

    def decode_step(self, slot_idx, q, k, v, alpha, beta, out, s_new=None):
        args = (self.handle, slot_idx.data_ptr(), slot_idx.numel(), q.data_ptr(), k.data_ptr(),
                v.data_ptr(), alpha.data_ptr(), beta.data_ptr(), out.data_ptr())
        if s_new is None:
            sq_decode_step(*args, self._stream())
        else:
            sq_debug_decode_step_fp32(*args, s_new.data_ptr(), self._stream())

    def decode_step_split(self, slot_idx, q, k, v, alpha, beta, out, staging, side_stream):
        """The step with the refit and requantization on `side_stream` (a torch stream)."""
        sq_decode_step_split(self.handle, slot_idx.data_ptr(), slot_idx.numel(), q.data_ptr(),
                             k.data_ptr(), v.data_ptr(), alpha.data_ptr(), beta.data_ptr(),
                             out.data_ptr(), staging.data_ptr(), self._stream(),
                             side_stream.cuda_stream)

    def decode_chunk(self, slot_idx, q, k, v, alpha, beta, out):
        """q, k [B][H][T][d_k], v [B][H][T][d_v], alpha [B][H][T](or [..][d_k]), beta
        [B][H][T], out [B][H][T][d_v]; T = q.shape[2]."""
        sq_decode_chunk(self.handle, slot_idx.data_ptr(), slot_idx.numel(), q.shape[2],
                        q.data_ptr(), k.data_ptr(), v.data_ptr(), alpha.data_ptr(),
                        beta.data_ptr(), out.data_ptr(), self._stream())

    def set_row_impact(self, impact):
        sq_pool_set_row_impact(self.handle, impact)

    def window_flush(self, slot_idx):
        sq_window_flush(self.handle, slot_idx.data_ptr(), slot_idx.numel(), self._stream())

    def status(self) -> tuple[int, int]:
        return sq_pool_status(self.handle)
