"""GPU parity: the CUDA path through the C ABI against the CPU oracle.

Bit-exact: quantize of identical fp32 states, dequantize, slot gather/scatter, and the two
invariants (beta = 0 keeps bytes; quantize after dequantize is the identity). Lockstep: every
decode step is checked against the oracle started from the GPU's own pre-step bytes: o and
the fp32 state within 2e-3 + 1e-3 |ref|, codes equal on >= 99.99 % and within 1 LSB.
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


def small_cases():
    return {
        "tiny": W.WORKLOADS["tiny"],
        "gdn-s": W.small("gdn", batch=3, n_heads=4, d=32),
        "gdn-d128": W.small("gdn", batch=2, n_heads=6, d=128),
        "gdn-d48": W.small("gdn", batch=3, n_heads=5, d=48),
        "kda-s": W.small("kda", batch=3, n_heads=2, d=32),
        "kda-d128": W.small("kda", batch=2, n_heads=3, d=128),
        "kda-d80": W.small("kda", batch=2, n_heads=2, d=80),
        "pool-s": W.small("pool", batch=3, n_heads=4, d=32),
        "gdn-fit1": W.small("gdn", batch=2, n_heads=4, d=64, fit_iters=1),
        "gdn-f32io": W.small("gdn", batch=2, n_heads=4, d=64, io_dtype=W.IO_F32),
        "kda-many": W.small("kda", batch=40, n_heads=16, d=32),  # > 2 items per CTA, ragged
        # a quarter of the key rows fp16: whole four-row chunks of fp16 rows (their own path)
        "kda-pivots": W.small("kda", batch=3, n_heads=2, d=64, n_pivots=32),
    }


CASES = small_cases()


@pytest.mark.parametrize("name", list(CASES))
def test_quantize_bit_exact(oracle, name):
    wl = CASES[name]
    case = G.GpuCase(wl)
    opool = oracle.Pool(G.orc_layout(wl), case.bits, wl.slots)
    opool.quantize(case.si_np, wl.initial_state(case.si_np))
    gpu = case.slots()
    ref = opool.data.reshape(wl.slots, -1)
    np.testing.assert_array_equal(gpu[case.si_np], ref[case.si_np])


@pytest.mark.parametrize("name", list(CASES))
def test_dequantize_bit_exact(oracle, name):
    wl = CASES[name]
    case = G.GpuCase(wl)
    out = torch.empty((wl.batch, wl.n_heads, wl.d_k, wl.d_v), dtype=torch.float32, device="cuda")
    case.pool.dequantize(case.si, out)
    opool = G.oracle_pool_from(wl, case.bits, case.slots())
    np.testing.assert_array_equal(out.cpu().numpy(), opool.dequantize(case.si_np))


@pytest.mark.parametrize("name", list(CASES))
def test_decode_lockstep(name):
    wl = CASES[name]
    case = G.GpuCase(wl)
    mis = tot = 0
    for t in range(8 if name != "kda-many" else 3):
        m, n = G.lockstep(case, t)
        mis, tot = mis + m, tot + n
    assert mis <= max(1, 1e-4 * tot), (mis, tot)


@pytest.mark.parametrize("name", ["gdn-s", "kda-s", "pool-s", "gdn-d128", "kda-d128", "tiny"])
def test_beta_zero_keeps_bytes_on_gpu(name):
    """P-3 on the GPU: alpha = 1, beta = 0 leaves every packed byte unchanged."""
    wl = CASES[name]
    case = G.GpuCase(wl)
    before = case.slots()
    x = wl.step_inputs(0)
    x["alpha"] = np.ones_like(x["alpha"])
    x["beta"] = np.zeros_like(x["beta"])
    for _ in range(3):
        case.step(x)
    np.testing.assert_array_equal(case.slots(), before)


@pytest.mark.parametrize("name", list(CASES))
def test_quantize_of_dequantize_is_identity_on_gpu(name):
    """P-4 on the GPU."""
    wl = CASES[name]
    case = G.GpuCase(wl)
    for t in range(2):
        case.step(wl.step_inputs(t))
    before = case.slots()
    D = torch.empty((wl.batch, wl.n_heads, wl.d_k, wl.d_v), dtype=torch.float32, device="cuda")
    case.pool.dequantize(case.si, D)
    case.pool.quantize(case.si, D)
    np.testing.assert_array_equal(case.slots(), before)


def test_rollout_256_steps_lockstep():
    """256 steps of a GDN-style workload, each step checked against the oracle started from
    the GPU's pre-step state."""
    wl = W.small("gdn", batch=2, n_heads=4, d=128)
    case = G.GpuCase(wl)
    mis = tot = 0
    for t in range(256):
        m, n = G.lockstep(case, t, want_state=False)
        mis, tot = mis + m, tot + n
    assert mis <= 1e-4 * tot, (mis, tot)


def test_bad_slot_is_flagged_and_skipped():
    wl = CASES["pool-s"]
    case = G.GpuCase(wl)
    st, _ = case.pool.status()
    assert st == sq.SQ_OK
    before = case.slots()
    bad = case.si.clone()
    bad[1] = wl.slots + 5
    x = wl.step_inputs(0)
    out, _ = case.step(x, slot_idx=bad)
    st, flag = case.pool.status()
    assert st == sq.SQ_ERR_DEVICE_FLAG and flag & sq.SQ_FLAG_BAD_SLOT
    assert np.isnan(out[1]).all() and np.isfinite(out[0]).all()
    after = case.slots()
    np.testing.assert_array_equal(after[np.setdiff1d(np.arange(wl.slots), case.si_np[[0, 2]])],
                                  before[np.setdiff1d(np.arange(wl.slots), case.si_np[[0, 2]])])
    assert case.pool.status() == (sq.SQ_OK, 0)


def test_nonfinite_input_is_flagged_and_skipped():
    wl = CASES["gdn-s"]
    case = G.GpuCase(wl)
    before = case.slots()
    x = wl.step_inputs(0)
    x["beta"] = x["beta"].copy()
    x["beta"][0, 2] = np.nan
    out, _ = case.step(x)
    st, flag = case.pool.status()
    assert st == sq.SQ_ERR_DEVICE_FLAG and flag & sq.SQ_FLAG_NONFINITE
    assert np.isnan(out[0, 2]).all()
    after = case.slots()
    # the skipped (request, head) keeps its bytes; the others moved on
    off = case.pool.head_offsets
    s0 = case.si_np[0]
    h2 = slice(off[2], off[3])
    np.testing.assert_array_equal(after[s0, h2], before[s0, h2])
    assert not np.array_equal(after[s0, off[0]:off[1]], before[s0, off[0]:off[1]])


def test_calls_reject_misaligned_pointers():
    wl = CASES["gdn-s"]
    case = G.GpuCase(wl)
    x = wl.step_inputs(0)
    q, k, v, a, b = case.device_inputs(x)
    out = torch.empty((wl.batch, wl.n_heads, wl.d_v), dtype=torch.float32, device="cuda")
    with pytest.raises(sq.SqError) as e:
        sq.sq_decode_step(case.pool.handle, case.si.data_ptr(), wl.batch, q.data_ptr() + 2,
                          k.data_ptr(), v.data_ptr(), a.data_ptr(), b.data_ptr(),
                          out.data_ptr(), 0)
    assert e.value.status == sq.SQ_ERR_INVALID_ARG


@pytest.mark.parametrize("name", ["gdn", "kda", "pool"])
def test_full_size_sampled(name):
    """Full-size workloads in the launch configuration the bench times: two steps, with a
    seeded sample of requests checked against the oracle (all heads of each)."""
    wl = W.WORKLOADS[name]
    case = G.GpuCase(wl)
    sample = np.sort(np.random.default_rng(7).choice(wl.batch, 6, replace=False))
    for t in range(2):
        G.lockstep(case, t, sample=sample, want_state=(t == 0))


@pytest.mark.parametrize("name", ["gdn-d128", "kda-d128", "gdn-s"])
@pytest.mark.parametrize("want_state", [False, True])
def test_extreme_gates(name, want_state):
    """A gate of 0 (the old state is erased: M_new = k b^T) and a gate of 1e-30 take the
    kernel's direct update form (the row factor A_i = alpha_i r16_i is outside [2^-60, 2^60]);
    the other requests keep the usual form. Lockstep against the oracle."""
    base = CASES[name]
    wl = base.scaled(batch=3)
    case = G.GpuCase(wl)
    mis = tot = 0
    for t in range(3):
        x = wl.step_inputs(t)
        x["alpha"] = x["alpha"].copy()
        x["alpha"][0] = 0.0
        x["alpha"][1] = 1e-30
        m, n = G.lockstep(case, t, want_state=want_state, x=x)
        mis, tot = mis + m, tot + n
    assert mis <= max(1, 1e-4 * tot), (mis, tot)
    assert case.pool.status() == (sq.SQ_OK, 0)


def test_empty_batches_are_no_ops():
    """batch = 0 (and n = 0) on every per-step call: SQ_OK, no launch, no byte changed."""
    wl = CASES["gdn-s"]
    case = G.GpuCase(wl)
    before = case.slots()
    q, k, v, a, b = case.device_inputs(wl.step_inputs(0))
    out = torch.empty((wl.batch, wl.n_heads, 4, wl.d_v), dtype=torch.float32, device="cuda")
    staging = torch.empty((wl.batch, wl.n_heads, wl.d_k, wl.d_v), device="cuda")
    h, si = case.pool.handle, case.si.data_ptr()
    ptrs = (q.data_ptr(), k.data_ptr(), v.data_ptr(), a.data_ptr(), b.data_ptr(), out.data_ptr())
    sq.sq_decode_step(h, si, 0, *ptrs, 0)
    sq.sq_decode_chunk(h, si, 0, 4, *ptrs, 0)
    sq.sq_decode_step_split(h, si, 0, *ptrs, staging.data_ptr(), 0, 0)
    sq.sq_decode_step_split_static(h, si, 0, *ptrs, 0)
    sq.sq_quantize_fp32_state(h, si, 0, staging.data_ptr(), 0)
    sq.sq_dequantize_state(h, si, 0, staging.data_ptr(), 0)
    torch.cuda.synchronize()
    assert case.pool.status() == (sq.SQ_OK, 0)
    np.testing.assert_array_equal(case.slots(), before)
