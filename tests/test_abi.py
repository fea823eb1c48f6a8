"""Host-side checks of the C ABI (no GPU): the library loads, exports what include/sq.h
declares, computes pool sizes that agree with the oracle's format, and rejects bad
arguments before touching CUDA."""
import numpy as np
import pytest

from bit_recurrent_state_gated_b200 import build as sqbuild
from bit_recurrent_state_gated_b200 import sq
from bit_recurrent_state_gated_b200 import workloads as W


@pytest.fixture(scope="module")
def lib():
    sqbuild.build()
    return sq.lib()


def test_exports_every_declared_symbol(lib):
    names = sq.exported_names()
    assert len(names) == 18, names  # the calls include/sq.h declares
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings(lib):
    for s in range(7):
        assert sq.sq_status_string(s) not in ("", "unknown status")
    assert sq.sq_status_string(99) == "unknown status"


@pytest.mark.parametrize("name", ["tiny", "gdn", "kda", "pool", "window"])
def test_pool_bytes_match_oracle_format(lib, oracle, name):
    wl = W.WORKLOADS[name]
    bits = wl.bits()
    lay = sq.Layout(1, wl.n_heads, wl.d_k, wl.d_v, wl.unit, wl.gate, wl.io_dtype, wl.fit_iters,
                    1, 0)
    n = sq.sq_pool_required_bytes(lay, bits, wl.pivot_mask())
    olay = oracle.Layout(wl.n_heads, wl.d_k, wl.d_v, wl.unit, wl.gate, wl.fit_iters)
    _, slot_bytes = oracle.slot_layout(olay, bits)
    assert n == slot_bytes
    lay5 = sq.Layout(3, wl.n_heads, wl.d_k, wl.d_v, wl.unit, wl.gate, wl.io_dtype, 2, 4, 8)
    olay5 = oracle.Layout(wl.n_heads, wl.d_k, wl.d_v, wl.unit, wl.gate, 2, 4, 8)
    _, sb5 = oracle.slot_layout(olay5, bits)
    assert sq.sq_pool_required_bytes(lay5, bits) >= 3 * sb5


@pytest.mark.parametrize("bad", [
    dict(d_k=8), dict(d_k=144), dict(d_v=24), dict(n_slots=0), dict(unit=2), dict(gate=5),
    dict(io_dtype=3), dict(fit_iters=0), dict(window=0), dict(window=1, n_outliers=4),
    dict(window=4, n_outliers=65)])
def test_invalid_layouts_rejected(lib, bad):
    base = dict(n_slots=2, n_heads=2, d_k=16, d_v=16, unit=0, gate=0, io_dtype=1, fit_iters=2,
                window=1, n_outliers=0)
    base.update(bad)
    with pytest.raises(sq.SqError) as e:
        sq.sq_pool_required_bytes(sq.Layout(**base), [4, 4])
    assert e.value.status == sq.SQ_ERR_INVALID_ARG


def test_invalid_bit_maps_rejected(lib):
    lay = sq.Layout(2, 2, 16, 16)
    for bits, pm in [([3, 4], None), ([4, 16], [0, 0]), ([4, 8], [1, 0]), ([0, 4], None)]:
        with pytest.raises(sq.SqError) as e:
            sq.sq_pool_required_bytes(lay, bits, pm)
        assert e.value.status == sq.SQ_ERR_INVALID_ARG
    assert sq.sq_pool_required_bytes(lay, [4, 16], [0, 1]) > 0


def test_create_rejects_bad_buffers_before_cuda(lib):
    lay = sq.Layout(2, 2, 16, 16)
    need = sq.sq_pool_required_bytes(lay, [4, 8])
    for ptr, n in [(0, need), (256 * 1024 + 16, need), (256 * 1024, need - 1)]:
        with pytest.raises(sq.SqError) as e:
            sq.sq_state_pool_create(lay, [4, 8], None, ptr, n)
        assert e.value.status == sq.SQ_ERR_INVALID_ARG


def test_calls_on_null_pool_rejected(lib):
    with pytest.raises(sq.SqError):
        sq.sq_decode_step(0, 16, 1, 16, 16, 16, 16, 16, 16, 0)
    with pytest.raises(sq.SqError):
        sq.sq_quantize_fp32_state(0, 16, 1, 16, 0)
    with pytest.raises(sq.SqError):
        sq.sq_pool_info(0, 1)
    with pytest.raises(sq.SqError):
        sq.sq_decode_chunk(0, 16, 1, 4, 16, 16, 16, 16, 16, 16, 0)
    with pytest.raises(sq.SqError):
        sq.sq_decode_step_split(0, 16, 1, 16, 16, 16, 16, 16, 16, 16, 0, 0)
    with pytest.raises(sq.SqError):
        sq.sq_decode_step_split_static(0, 16, 1, 16, 16, 16, 16, 16, 16, 0)
    sq.sq_state_pool_destroy(0)


def test_set_wait_rejects_a_null_pool(lib):
    assert lib.sq_debug_set_wait(None, 1000, 0) == sq.SQ_ERR_INVALID_ARG


def test_set_full_fit_rejects_a_null_pool(lib):
    assert lib.sq_debug_set_full_fit(None, 1) == sq.SQ_ERR_INVALID_ARG
