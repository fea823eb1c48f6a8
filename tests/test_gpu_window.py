"""GPU parity of the windowed variant (requantize every W tokens, fp16 compensation entries)
against the CPU oracle.

Lockstep per window: at each window start the oracle takes the GPU's packed block; both sides
then run W tokens on their own (the GPU holds the delta as low-rank factors, the oracle as an
exact dense state): o must agree at every token, and the requantized block after the W-th
token must agree code by code (>= 99.99 %, within 1 LSB; compensation entries within fp16
rounding of each other).
"""
import numpy as np
import pytest

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a GPU", allow_module_level=True)

from bit_recurrent_state_gated_b200 import build as sqbuild  # noqa: E402
from bit_recurrent_state_gated_b200 import sq  # noqa: E402
from bit_recurrent_state_gated_b200 import workloads as W  # noqa: E402

import gpu_util as G  # noqa: E402

sqbuild.build()

CASES = {
    "win-s": W.small("window", batch=3, n_heads=2, d=32).scaled(window=4),
    "win-d128": W.small("window", batch=2, n_heads=3, d=128).scaled(window=5),
    "win-mixed": W.small("gdn", batch=2, n_heads=4, d=64).scaled(window=3, n_outliers=4),
    "win-kda": W.small("kda", batch=2, n_heads=2, d=32).scaled(window=4, n_outliers=8),
    "win-f32io": W.small("window", batch=2, n_heads=2, d=64, io_dtype=W.IO_F32).scaled(window=4),
    "win-kda-pivots": W.small("kda", batch=2, n_heads=2, d=64, n_pivots=32).scaled(window=4,
                                                                                 n_outliers=8),
}


def _oracle_from_gpu(case):
    opool = G.oracle_pool_from(case.wl, case.bits, case.slots()[case.si_np])
    return opool


def _compare_blocks(case, opool, what):
    return G.compare_codes(case.wl, case.bits, case.slots()[case.si_np],
                           opool.data.reshape(case.wl.batch, -1), what)


@pytest.mark.parametrize("name", list(CASES))
def test_window_quantize_bit_exact(oracle, name):
    wl = CASES[name]
    case = G.GpuCase(wl)
    opool = oracle.Pool(G.orc_layout(wl), case.bits, wl.slots)
    opool.quantize(case.si_np, wl.initial_state(case.si_np))
    np.testing.assert_array_equal(case.slots()[case.si_np],
                                  opool.data.reshape(wl.slots, -1)[case.si_np])


@pytest.mark.parametrize("name", list(CASES))
def test_window_lockstep(name):
    wl = CASES[name]
    case = G.GpuCase(wl)
    n = np.arange(wl.batch)
    mis = tot = 0
    t = 0
    for window in range(3):
        opool = _oracle_from_gpu(case)
        frozen = case.slots().copy()
        for step in range(wl.window):
            x = wl.step_inputs(t)
            o_gpu, _ = case.step(x)
            o_ref = opool.window_step(n, x["q"], x["k"], x["v"], x["alpha"], x["beta"])
            G.close(o_gpu, o_ref, f"window {window} token {step} o")
            if step + 1 < wl.window:  # the packed block stays frozen inside the window
                np.testing.assert_array_equal(case.slots(), frozen)
            t += 1
        m, k = _compare_blocks(case, opool, f"window {window} end")
        mis, tot = mis + m, tot + k
    assert mis <= max(1, 1e-4 * tot), (mis, tot)
    assert case.pool.status() == (sq.SQ_OK, 0)


@pytest.mark.parametrize("name", ["win-s", "win-kda", "win-f32io"])
def test_window_flush_mid_window(name):
    wl = CASES[name]
    case = G.GpuCase(wl)
    n = np.arange(wl.batch)
    opool = _oracle_from_gpu(case)
    for t in range(wl.window - 2):
        x = wl.step_inputs(t)
        case.step(x)
        opool.window_step(n, x["q"], x["k"], x["v"], x["alpha"], x["beta"])
    case.pool.window_flush(case.si)
    opool.window_flush(n)
    _compare_blocks(case, opool, "flush")
    before = case.slots().copy()
    case.pool.window_flush(case.si)  # closed window: nothing to do
    np.testing.assert_array_equal(case.slots(), before)


def test_window_beta_zero_keeps_bytes():
    """P-3 through a whole window: alpha = 1, beta = 0 leaves every packed byte unchanged."""
    wl = CASES["win-s"]
    case = G.GpuCase(wl)
    before = case.slots()
    x = wl.step_inputs(0)
    x["alpha"] = np.ones_like(x["alpha"])
    x["beta"] = np.zeros_like(x["beta"])
    for _ in range(2 * wl.window):
        case.step(x)
    np.testing.assert_array_equal(case.slots(), before)


def test_window_full_size_sampled():
    """The windowed workload at full size (256 requests x 32 heads, W = 16): one window, a
    seeded sample of requests checked against the oracle."""
    wl = W.WORKLOADS["window"]
    case = G.GpuCase(wl)
    sample = np.sort(np.random.default_rng(5).choice(wl.batch, 4, replace=False))
    opool = G.oracle_pool_from(wl, case.bits, case.slots()[case.si_np[sample]])
    n = np.arange(sample.size)
    for t in range(wl.window):
        x = wl.step_inputs(t)
        o_gpu, _ = case.step(x)
        xs = G.sub_inputs(x, sample)
        o_ref = opool.window_step(n, xs["q"], xs["k"], xs["v"], xs["alpha"], xs["beta"])
        G.close(o_gpu[sample], o_ref, f"token {t} o")
    G.compare_codes(wl, case.bits, case.slots()[case.si_np[sample]],
                    opool.data.reshape(sample.size, -1), "window end")
