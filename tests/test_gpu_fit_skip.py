"""The decode step skips the last column pass of the scale fit when a bound proves that pass
cannot change any fp16 column scale. The claim is exactness: the stored bytes must be those of
the full pass. Two pools start from the same packed states and take the same steps, one with
the skip allowed (the default) and one forced through the full pass (sq_debug_set_full_fit);
slots and outputs must stay bit-identical at every step, at full head shape, for head units and
key-row units."""
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


def test_set_full_fit_rejects_bad_values():
    wl = W.small("gdn", batch=2, n_heads=2, d=32)
    case = G.GpuCase(wl)
    with pytest.raises(sq.SqError):
        sq.sq_debug_set_full_fit(case.pool.handle, 2)
