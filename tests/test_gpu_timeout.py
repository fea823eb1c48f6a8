"""The bounded waits of the decode, window and chunk kernels, made to run out without faulting
anything.

sq_debug_set_wait shortens the wait limit to 2 ms and has every stage barrier expect 64 bytes
more than its bulk copies bring, so no wait can complete: each CTA must give up, flag
SQ_FLAG_TIMEOUT, let its own copies land, free its tensor memory and return. The host then reads
SQ_ERR_TIMEOUT from sq_pool_status, every slot keeps its bytes, and a normal step on the same
context (hook reset) passes lockstep against the oracle.
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


@pytest.mark.parametrize("name", ["gdn", "kda"])
def test_wait_runs_out_and_the_context_stays_usable(name):
    wl = W.small(name, batch=6, n_heads=4, d=128)
    case = G.GpuCase(wl)
    before = case.slots()
    sq.sq_debug_set_wait(case.pool.handle, 2_000_000, 64)
    out, _ = case.step(wl.step_inputs(0))
    st, flag = case.pool.status()
    assert st == sq.SQ_ERR_TIMEOUT and flag & sq.SQ_FLAG_TIMEOUT, (st, flag)
    np.testing.assert_array_equal(case.slots(), before)
    sq.sq_debug_set_wait(case.pool.handle, 0, 0)
    m, n = G.lockstep(case, 1)
    assert m <= max(1, 1e-4 * n)
    assert case.pool.status() == (sq.SQ_OK, 0)


def test_window_wait_runs_out_and_the_context_stays_usable():
    """The windowed kernel (one staging buffer, a separate term buffer): every CTA gives up at
    its first item, the packed blocks and the side state keep their bytes, and afterwards the
    window continues in lockstep with the oracle."""
    wl = W.small("window", batch=6, n_heads=4, d=128).scaled(window=4)
    case = G.GpuCase(wl)
    n = np.arange(wl.batch)
    case.step(wl.step_inputs(0))  # one token into the window: the side state holds a term
    torch.cuda.synchronize()
    before = case.pool.buf.cpu().numpy().copy()
    sq.sq_debug_set_wait(case.pool.handle, 2_000_000, 64)
    case.step(wl.step_inputs(1))
    st, flag = case.pool.status()
    assert st == sq.SQ_ERR_TIMEOUT and flag & sq.SQ_FLAG_TIMEOUT, (st, flag)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(case.pool.buf.cpu().numpy(), before)
    sq.sq_debug_set_wait(case.pool.handle, 0, 0)
    # the rest of the window from a fresh window start, against the oracle
    case.pool.window_flush(case.si)
    opool = G.oracle_pool_from(wl, case.bits, case.slots()[case.si_np])
    for t in range(2, 2 + wl.window):
        x = wl.step_inputs(t)
        o_gpu, _ = case.step(x)
        o_ref = opool.window_step(n, x["q"], x["k"], x["v"], x["alpha"], x["beta"])
        G.close(o_gpu, o_ref, f"token {t} o")
    assert case.pool.status() == (sq.SQ_OK, 0)


def test_chunk_wait_runs_out_and_the_context_stays_usable():
    wl = W.small("gdn", batch=6, n_heads=4, d=128)
    case = G.GpuCase(wl)
    before = case.slots()
    sq.sq_debug_set_wait(case.pool.handle, 2_000_000, 64)
    x = wl.chunk_inputs(0, 4)
    q, k, v, a, b = case.device_inputs(x)
    out = torch.empty((wl.batch, wl.n_heads, 4, wl.d_v), dtype=torch.float32, device="cuda")
    case.pool.decode_chunk(case.si, q, k, v, a, b, out)
    st, flag = case.pool.status()
    assert st == sq.SQ_ERR_TIMEOUT and flag & sq.SQ_FLAG_TIMEOUT, (st, flag)
    np.testing.assert_array_equal(case.slots(), before)
    sq.sq_debug_set_wait(case.pool.handle, 0, 0)
    m, n = G.lockstep(case, 1)
    assert m <= max(1, 1e-4 * n)
    assert case.pool.status() == (sq.SQ_OK, 0)


def test_set_wait_rejects_bad_arguments():
    wl = W.small("gdn", batch=2, n_heads=2, d=32)
    case = G.GpuCase(wl)
    with pytest.raises(sq.SqError):
        sq.sq_debug_set_wait(case.pool.handle, 1000, 4097)
    with pytest.raises(sq.SqError):
        sq.sq_debug_set_wait(0, 1000, 0)
