"""GPU parity of the side-stream split (sq_decode_step_split) against the CPU oracle.

The split runs the update on the caller's stream (fp32 state to a staging buffer) and the refit
and requantization on a second stream. Its result must follow the oracle's decode step like
the fused kernel's does (o within tolerance, codes >= 99.99 % equal and within 1 LSB), and the
stream ordering must make back-to-back calls, without host synchronization, give the same bytes
as calls separated by a device synchronization.
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
    "gdn-s": W.small("gdn", batch=3, n_heads=4, d=32),
    "gdn-d128": W.small("gdn", batch=2, n_heads=4, d=128),
    "kda-d128": W.small("kda", batch=2, n_heads=2, d=128),
    "pool-d64": W.small("pool", batch=3, n_heads=3, d=64),
}


class Split:
    def __init__(self, case):
        wl = case.wl
        self.case = case
        self.side = torch.cuda.Stream()
        self.staging = torch.empty((wl.batch, wl.n_heads, wl.d_k, wl.d_v), dtype=torch.float32,
                                   device="cuda")
        self.out = torch.empty((wl.batch, wl.n_heads, wl.d_v), dtype=torch.float32,
                               device="cuda")

    def step(self, x, sync=True):
        q, k, v, a, b = self.case.device_inputs(x)
        self.case.pool.decode_step_split(self.case.si, q, k, v, a, b, self.out, self.staging,
                                         self.side)
        if sync:
            torch.cuda.synchronize()
        return self.out.clone()


@pytest.mark.parametrize("name", list(CASES))
def test_split_lockstep(name):
    wl = CASES[name]
    case = G.GpuCase(wl)
    sp = Split(case)
    mis = tot = 0
    for t in range(4):
        x = wl.step_inputs(t)
        pre = case.slots()
        o = sp.step(x).cpu().numpy()
        post = case.slots()
        opool = G.oracle_pool_from(wl, case.bits, pre[case.si_np])
        o_ref = opool.decode_step(np.arange(wl.batch), x["q"], x["k"], x["v"], x["alpha"],
                                  x["beta"])
        G.close(o, o_ref, f"step {t} o")
        m, n = G.compare_codes(wl, case.bits, post[case.si_np],
                               opool.data.reshape(wl.batch, -1), f"step {t}")
        mis, tot = mis + m, tot + n
        untouched = np.setdiff1d(np.arange(wl.slots), case.si_np)
        if untouched.size:
            np.testing.assert_array_equal(post[untouched], pre[untouched])
    assert mis <= max(1, 1e-4 * tot), f"{mis} of {tot} codes differ"
    assert case.pool.status() == (sq.SQ_OK, 0)


@pytest.mark.parametrize("name", ["gdn-d128", "kda-d128"])
def test_split_stream_order(name):
    """Split steps back to back, mixed with fused steps and a read-back, with no host
    synchronization: the same bytes and outputs as the same calls with a device
    synchronization after each."""
    wl = CASES[name]
    runs = []
    for sync in (True, False):
        case = G.GpuCase(wl)
        sp = Split(case)
        outs = []
        for t in range(6):
            x = wl.step_inputs(t)
            if t == 3:  # a fused step on the caller's stream in between
                q, k, v, a, b = case.device_inputs(x)
                o = torch.empty_like(sp.out)
                case.pool.decode_step(case.si, q, k, v, a, b, o)
                outs.append(o)
            else:
                outs.append(sp.step(x, sync=sync))
            if sync:
                torch.cuda.synchronize()
        S = torch.empty((wl.batch, wl.n_heads, wl.d_k, wl.d_v), device="cuda")
        case.pool.dequantize(case.si, S)  # ordered after the last side-stream requantization
        torch.cuda.synchronize()
        runs.append(([o.cpu().numpy() for o in outs], S.cpu().numpy(), case.slots()))
    (o1, S1, b1), (o2, S2, b2) = runs
    for t in range(6):
        np.testing.assert_array_equal(o1[t], o2[t])
    np.testing.assert_array_equal(S1, S2)
    np.testing.assert_array_equal(b1, b2)


def test_split_nonfinite_input_keeps_bytes():
    wl = CASES["gdn-s"]
    case = G.GpuCase(wl)
    sp = Split(case)
    before = case.slots()
    x = wl.step_inputs(0)
    x["beta"] = x["beta"].copy()
    x["beta"][0, 2] = np.nan
    o = sp.step(x).cpu().numpy()
    st, flag = case.pool.status()
    assert st == sq.SQ_ERR_DEVICE_FLAG and flag == sq.SQ_FLAG_NONFINITE
    assert np.isnan(o[0, 2]).all() and not np.isnan(np.delete(o[0], 2, axis=0)).any()
    after = case.slots()
    off = case.pool.head_offsets
    s0 = case.si_np[0]
    np.testing.assert_array_equal(after[s0, off[2]:off[3]], before[s0, off[2]:off[3]])
    assert not np.array_equal(after[s0, off[0]:off[1]], before[s0, off[0]:off[1]])


def test_split_rejects_windowed_pools_and_bad_staging():
    wl = W.small("window", batch=2, n_heads=2, d=32).scaled(window=4)
    case = G.GpuCase(wl)
    with pytest.raises(sq.SqError):
        Split(case).step(wl.step_inputs(0))
    case = G.GpuCase(CASES["gdn-s"])
    sp = Split(case)
    sp.staging = torch.empty(sp.staging.numel() + 1, device="cuda")[1:]  # 4-byte aligned only
    with pytest.raises(sq.SqError):
        sp.step(case.wl.step_inputs(0))


def test_split_full_size_sampled():
    """The split workload at full size (64 requests x 32 heads, d = 128, the launch the bench
    times): two steps, a seeded sample of requests checked against the oracle each time."""
    wl = W.WORKLOADS["split"]
    case = G.GpuCase(wl)
    sp = Split(case)
    sample = np.sort(np.random.default_rng(9).choice(wl.batch, 4, replace=False))
    for t in range(2):
        x = wl.step_inputs(t)
        pre = case.slots()
        o = sp.step(x).cpu().numpy()
        post = case.slots()
        opool = G.oracle_pool_from(wl, case.bits, pre[case.si_np[sample]])
        xs = G.sub_inputs(x, sample)
        o_ref = opool.decode_step(np.arange(sample.size), xs["q"], xs["k"], xs["v"],
                                  xs["alpha"], xs["beta"])
        G.close(o[sample], o_ref, f"step {t} o")
        G.compare_codes(wl, case.bits, post[case.si_np[sample]],
                        opool.data.reshape(sample.size, -1), f"step {t}")
