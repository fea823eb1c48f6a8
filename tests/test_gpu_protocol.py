"""Full-length runs of the serving-pool and windowed workloads at full size, checked the way
the parity protocol prescribes for large configurations: a seeded subset of 32 requests at
every step (every window for the windowed variant) and all requests at the first and the last.

Each check starts the oracle from the GPU's own packed bytes of the checked slots (gathered on
the device, so only those cross to the host): o within tolerance, requantized codes equal on
>= 99.99 % and within 1 LSB, counted over the whole run.
"""
import numpy as np
import pytest

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a GPU", allow_module_level=True)

from bit_recurrent_state_gated_b200 import build as sqbuild  # noqa: E402
from bit_recurrent_state_gated_b200 import workloads as W  # noqa: E402

import gpu_util as G  # noqa: E402

sqbuild.build()


def gather(case, slots):
    idx = torch.from_numpy(np.asarray(slots, dtype=np.int64)).cuda()
    torch.cuda.synchronize()
    return case.pool.slots_view().index_select(0, idx).cpu().numpy()


def test_pool_64_steps():
    """Serving pool: 1024 slots, 512 active by a seeded permutation, 64 steps."""
    wl = W.WORKLOADS["pool"]
    case = G.GpuCase(wl)
    sample = np.sort(np.random.default_rng(17).choice(wl.batch, 32, replace=False))
    idle = np.setdiff1d(np.arange(wl.slots), case.si_np)[:32]
    idle_before = gather(case, idle)
    mis = tot = 0
    for t in range(wl.steps):
        rows = np.arange(wl.batch) if t in (0, wl.steps - 1) else sample
        slots = case.si_np[rows]
        x = wl.step_inputs(t)
        pre = gather(case, slots)
        o_gpu, _ = case.step(x)
        post = gather(case, slots)
        opool = G.oracle_pool_from(wl, case.bits, pre)
        xs = G.sub_inputs(x, rows)
        o_ref = opool.decode_step(np.arange(rows.size), xs["q"], xs["k"], xs["v"], xs["alpha"],
                                  xs["beta"])
        G.close(o_gpu[rows], o_ref, f"step {t} o")
        m, n = G.compare_codes(wl, case.bits, post, opool.data.reshape(rows.size, -1),
                               f"step {t}")
        mis, tot = mis + m, tot + n
    assert mis <= 1e-4 * tot, f"{mis} of {tot} codes differ"
    np.testing.assert_array_equal(gather(case, idle), idle_before)
    assert case.pool.status() == (0, 0)


def test_window_512_steps():
    """Windowed variant: 256 requests, W = 16, 8 compensation entries per head, 512 tokens
    (32 windows); o checked at every token, the requantized blocks at every window end."""
    wl = W.WORKLOADS["window"]
    case = G.GpuCase(wl)
    sample = np.sort(np.random.default_rng(19).choice(wl.batch, 32, replace=False))
    n_win = wl.steps // wl.window
    mis = tot = 0
    for w in range(n_win):
        rows = np.arange(wl.batch) if w in (0, n_win - 1) else sample
        slots = case.si_np[rows]
        opool = G.oracle_pool_from(wl, case.bits, gather(case, slots))
        n = np.arange(rows.size)
        for s in range(wl.window):
            t = w * wl.window + s
            x = wl.step_inputs(t)
            o_gpu, _ = case.step(x)
            xs = G.sub_inputs(x, rows)
            o_ref = opool.window_step(n, xs["q"], xs["k"], xs["v"], xs["alpha"], xs["beta"])
            G.close(o_gpu[rows], o_ref, f"token {t} o")
        m, k = G.compare_codes(wl, case.bits, gather(case, slots),
                               opool.data.reshape(rows.size, -1), f"window {w} end")
        mis, tot = mis + m, tot + k
    assert mis <= 1e-4 * tot, f"{mis} of {tot} codes differ"
    assert case.pool.status() == (0, 0)
