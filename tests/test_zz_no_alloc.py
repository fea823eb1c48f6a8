"""The allocation-free split step (sq_decode_step_split_static) against the split step with a
caller-allocated staging buffer (sq_decode_step_split).

sq_decode_step_split_static serves callers that cannot allocate device memory, such as a
serving engine whose allocator owns all device memory or a host with a fixed memory plan: its
staging state sits in a 32 MiB array inside libsq. Two pools start from the same states and take
the same two steps, one through each entry point (both through the C ABI, on one stream); the
outputs and the states must agree within the parity tolerance, and a batch too large for the
array must be refused. This file is collected last.
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


def _dequant(case):
    wl = case.wl
    S = torch.empty((wl.batch, wl.n_heads, wl.d_k, wl.d_v), dtype=torch.float32, device="cuda")
    case.pool.dequantize(case.si, S)
    torch.cuda.synchronize()
    return S.cpu().numpy()


@pytest.mark.parametrize("wl", [W.small("gdn", batch=3, n_heads=4, d=128),
                                W.small("kda", batch=2, n_heads=3, d=64)],
                         ids=["gdn-d128", "kda-d64"])
def test_static_staging_matches_caller_staging(wl):
    ref, new = G.GpuCase(wl), G.GpuCase(wl)
    stream = torch.cuda.current_stream().cuda_stream
    staging = torch.empty((wl.batch, wl.n_heads, wl.d_k, wl.d_v), dtype=torch.float32,
                          device="cuda")
    for t in range(2):  # two calls in a row
        x = wl.step_inputs(t)
        q, k, v, a, b = ref.device_inputs(x)
        o_ref = torch.empty((wl.batch, wl.n_heads, wl.d_v), dtype=torch.float32, device="cuda")
        o_new = torch.empty_like(o_ref)
        sq.sq_decode_step_split(ref.pool.handle, ref.si.data_ptr(), wl.batch, q.data_ptr(),
                                k.data_ptr(), v.data_ptr(), a.data_ptr(), b.data_ptr(),
                                o_ref.data_ptr(), staging.data_ptr(), stream, stream)
        sq.sq_decode_step_split_static(new.pool.handle, new.si.data_ptr(), wl.batch,
                                       q.data_ptr(), k.data_ptr(), v.data_ptr(), a.data_ptr(),
                                       b.data_ptr(), o_new.data_ptr(), stream)
        torch.cuda.synchronize()
        G.close(o_new.cpu().numpy(), o_ref.cpu().numpy(), f"call {t} o")
        G.close(_dequant(new), _dequant(ref), f"call {t} state")
    assert new.pool.status() == (sq.SQ_OK, 0)
    assert ref.pool.status() == (sq.SQ_OK, 0)


def test_static_staging_refuses_a_batch_beyond_the_array():
    wl = W.small("gdn", batch=17, n_heads=32, d=128)  # 17 x 32 x 64 KiB > 32 MiB
    case = G.GpuCase(wl)
    before = case.slots()
    q, k, v, a, b = case.device_inputs(wl.step_inputs(0))
    out = torch.empty((wl.batch, wl.n_heads, wl.d_v), dtype=torch.float32, device="cuda")
    with pytest.raises(sq.SqError) as e:
        sq.sq_decode_step_split_static(case.pool.handle, case.si.data_ptr(), wl.batch,
                                       q.data_ptr(), k.data_ptr(), v.data_ptr(), a.data_ptr(),
                                       b.data_ptr(), out.data_ptr(),
                                       torch.cuda.current_stream().cuda_stream)
    assert e.value.status == sq.SQ_ERR_INVALID_ARG
    np.testing.assert_array_equal(case.slots(), before)
