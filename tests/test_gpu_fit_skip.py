"""The scale fit skips its second alternation, or only its last column pass, when the rule's
rounding bounds prove that the skipped work cannot change any fp16 scale. The claim is
exactness: the stored bytes must be those of the full fit. Two pools start from the same packed
states and take the same steps, one with the skips allowed (the default) and one forced through
the full fit (sq_debug_set_full_fit); slots and outputs must stay bit-identical at every step,
at full head shape, for head units and key-row units, in the decode step and in the fold that
ends a window or a multi-token chunk."""
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


@pytest.mark.parametrize("name", ["gdn", "kda", "pool"])
def test_skipped_column_pass_gives_the_full_pass_bytes(name):
    wl = W.WORKLOADS[name].scaled(batch=32, n_slots=64 if W.WORKLOADS[name].n_slots else 0)
    fast, full = G.GpuCase(wl), G.GpuCase(wl)
    sq.sq_debug_set_full_fit(full.pool.handle, 1)
    np.testing.assert_array_equal(fast.slots(), full.slots())
    for t in range(8):
        x = wl.step_inputs(t)
        o_fast, _ = fast.step(x)
        o_full, _ = full.step(x)
        np.testing.assert_array_equal(o_fast, o_full)
        np.testing.assert_array_equal(fast.slots(), full.slots())
    assert fast.pool.status() == (sq.SQ_OK, 0)
    assert full.pool.status() == (sq.SQ_OK, 0)


@pytest.mark.parametrize("name", ["window", "window-kda"])
def test_skipped_fit_in_the_window_fold(name):
    wl = (W.WORKLOADS["window"].scaled(batch=16) if name == "window"
          else W.small("kda", batch=8, n_heads=4, d=128).scaled(window=4, n_outliers=8))
    fast, full = G.GpuCase(wl), G.GpuCase(wl)
    sq.sq_debug_set_full_fit(full.pool.handle, 1)
    for t in range(2 * wl.window):  # two folds
        x = wl.step_inputs(t)
        o_fast, _ = fast.step(x)
        o_full, _ = full.step(x)
        np.testing.assert_array_equal(o_fast, o_full)
        np.testing.assert_array_equal(fast.slots(), full.slots())
    assert fast.pool.status() == (sq.SQ_OK, 0)
    assert full.pool.status() == (sq.SQ_OK, 0)


@pytest.mark.parametrize("name", ["gdn", "kda"])
def test_skipped_fit_in_the_chunk_fold(name):
    wl = W.WORKLOADS[name].scaled(batch=16)
    fast, full = G.GpuCase(wl), G.GpuCase(wl)
    sq.sq_debug_set_full_fit(full.pool.handle, 1)
    for c in range(3):
        x = wl.chunk_inputs(8 * c, 8)
        outs = []
        for case in (fast, full):
            q, k, v, a, b = case.device_inputs(x)
            out = torch.empty((wl.batch, wl.n_heads, 8, wl.d_v), dtype=torch.float32, device="cuda")
            case.pool.decode_chunk(case.si, q, k, v, a, b, out)
            outs.append(out.cpu().numpy())
        np.testing.assert_array_equal(outs[0], outs[1])
        np.testing.assert_array_equal(fast.slots(), full.slots())
    assert fast.pool.status() == (sq.SQ_OK, 0)
    assert full.pool.status() == (sq.SQ_OK, 0)


def test_set_full_fit_rejects_bad_values():
    wl = W.small("gdn", batch=2, n_heads=2, d=32)
    case = G.GpuCase(wl)
    with pytest.raises(sq.SqError):
        sq.sq_debug_set_full_fit(case.pool.handle, 2)
