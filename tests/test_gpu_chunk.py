"""GPU parity of the multi-token chunk step (sq_decode_chunk) against the CPU oracle.

A chunk of T tokens reads each state once and requantizes it once, after the T-th token; every
token's update and output are the decode step's. The oracle for it is the windowed oracle with
W = T and no compensation entries: it keeps the exact state through the window and
requantizes after the W-th token. Each check starts the oracle from the GPU's packed bytes:
o must agree at every token, and the requantized block code by code (>= 99.99 %, within 1 LSB).
"""
import numpy as np
import pytest

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a GPU", allow_module_level=True)

import oracle  # noqa: E402
from bit_recurrent_state_gated_b200 import build as sqbuild  # noqa: E402
from bit_recurrent_state_gated_b200 import sq  # noqa: E402
from bit_recurrent_state_gated_b200 import workloads as W  # noqa: E402

import gpu_util as G  # noqa: E402

sqbuild.build()

CASES = {
    "gdn-s": W.small("gdn", batch=3, n_heads=4, d=32),
    "gdn-d128": W.small("gdn", batch=2, n_heads=4, d=128),
    "kda-d64": W.small("kda", batch=2, n_heads=2, d=64),
    "kda-d128": W.small("kda", batch=2, n_heads=2, d=128),
    "pool-d96": W.small("pool", batch=3, n_heads=3, d=96),
    "kda-pivots": W.small("kda", batch=2, n_heads=2, d=64, n_pivots=32),
    "tiny": W.WORKLOADS["tiny"],
}


def device_chunk(case, x):
    wl = case.wl
    if wl.io_dtype == W.IO_BF16:
        q, k, v = (G.to_dev(x[n + "_bf16"], torch.bfloat16) for n in ("q", "k", "v"))
    else:
        q, k, v = (G.to_dev(x[n]) for n in ("q", "k", "v"))
    return q, k, v, G.to_dev(x["alpha"]), G.to_dev(x["beta"])


def run_chunk(case, x, slot_idx=None):
    wl = case.wl
    si = case.si if slot_idx is None else slot_idx
    T = x["q"].shape[2]
    q, k, v, a, b = device_chunk(case, x)
    out = torch.empty((si.numel(), wl.n_heads, T, wl.d_v), dtype=torch.float32, device="cuda")
    case.pool.decode_chunk(si, q, k, v, a, b, out)
    torch.cuda.synchronize()
    return out.cpu().numpy()


def oracle_chunk(wl, bits, pre_slots, x, rows):
    """The oracle's window of T tokens over the given packed slots: (o [n][H][T][d_v], bytes)."""
    T = x["q"].shape[2]
    lay = G.orc_layout(wl.scaled(window=T, n_outliers=0))
    opool = oracle.Pool(lay, bits, rows.size)
    assert opool.slot_bytes == pre_slots.shape[1]
    opool.data[:] = pre_slots.reshape(-1)
    n = np.arange(rows.size)
    o = np.zeros((rows.size, wl.n_heads, T, wl.d_v))
    for t in range(T):
        xs = {name: np.ascontiguousarray(a[rows][:, :, t]) for name, a in x.items()}
        o[:, :, t] = opool.window_step(n, xs["q"], xs["k"], xs["v"], xs["alpha"], xs["beta"])
    return o, opool.data.reshape(rows.size, -1)


def chunk_lockstep(case, x, rows=None, what="chunk"):
    wl = case.wl
    rows = np.arange(wl.batch) if rows is None else np.asarray(rows)
    pre = case.slots()
    o_gpu = run_chunk(case, x)
    post = case.slots()
    slots = case.si_np[rows]
    o_ref, ref_bytes = oracle_chunk(wl, case.bits, pre[slots], x, rows)
    G.close(o_gpu[rows], o_ref, what + " o")
    n_mis, n = G.compare_codes(wl, case.bits, post[slots], ref_bytes, what)
    untouched = np.setdiff1d(np.arange(wl.slots), case.si_np)
    if untouched.size:
        np.testing.assert_array_equal(post[untouched], pre[untouched])
    return n_mis, n


@pytest.mark.parametrize("T", [2, 5, 16])
@pytest.mark.parametrize("name", list(CASES))
def test_chunk_lockstep(name, T):
    case = G.GpuCase(CASES[name])
    mis = tot = 0
    for c in range(3):
        m, n = chunk_lockstep(case, case.wl.chunk_inputs(c * T, T), what=f"chunk {c} (T={T})")
        mis, tot = mis + m, tot + n
    assert mis <= max(1, 1e-4 * tot), f"{mis} of {tot} codes differ"


@pytest.mark.parametrize("name", ["gdn-s", "kda-d64"])
def test_chunk_rollout_256_tokens(name):
    """32 chunks of 8 tokens, each checked against the oracle from the GPU's own bytes."""
    case = G.GpuCase(CASES[name])
    mis = tot = 0
    for c in range(32):
        m, n = chunk_lockstep(case, case.wl.chunk_inputs(8 * c, 8), what=f"chunk {c}")
        mis, tot = mis + m, tot + n
    assert mis <= max(1, 1e-4 * tot), f"{mis} of {tot} codes differ"
    assert case.pool.status() == (sq.SQ_OK, 0)


def test_one_token_chunk_is_the_decode_step():
    wl = CASES["gdn-s"]
    a, b = G.GpuCase(wl), G.GpuCase(wl)
    for t in range(3):
        x = wl.chunk_inputs(t, 1)
        o_chunk = run_chunk(a, x)
        o_step, _ = b.step(wl.step_inputs(t))
        np.testing.assert_array_equal(o_chunk[:, :, 0], o_step)
    np.testing.assert_array_equal(a.slots(), b.slots())


@pytest.mark.parametrize("name", ["gdn-d128", "kda-d128", "gdn-s"])
@pytest.mark.parametrize("alpha", [0.0, 1e-12])
def test_chunk_gate_product_out_of_range(name, alpha):
    """A gate product below 1e-30 inside the chunk (alpha = 0 at one token, or 1e-12 for
    several) re-bases the on-chip state; the result still follows the oracle."""
    wl = CASES[name]
    case = G.GpuCase(wl)
    T = 7
    x = wl.chunk_inputs(0, T)
    if alpha == 0.0:
        x["alpha"][:, :, 3] = 0.0
    else:
        x["alpha"][:, :, 1:5] = alpha
    chunk_lockstep(case, x, what=f"alpha {alpha}")
    chunk_lockstep(case, wl.chunk_inputs(T, T), what="next chunk")


def test_chunk_beta_zero_keeps_bytes():
    """alpha = 1, beta = 0 through a chunk leaves every packed byte unchanged."""
    wl = CASES["gdn-d128"]
    case = G.GpuCase(wl)
    before = case.slots()
    x = wl.chunk_inputs(0, 9)
    x["alpha"] = np.ones_like(x["alpha"])
    x["beta"] = np.zeros_like(x["beta"])
    run_chunk(case, x)
    np.testing.assert_array_equal(case.slots(), before)


def test_chunk_nonfinite_token_skips_request_head():
    """A non-finite input at one token of one (request, head) skips that pair for the whole
    chunk (bytes kept, outputs NaN, flag raised); every other pair follows the oracle."""
    wl = CASES["gdn-s"]
    case = G.GpuCase(wl)
    pre = case.slots()
    T = 4
    x = wl.chunk_inputs(0, T)
    x["beta"][1, 2, 3] = np.nan
    o = run_chunk(case, x)
    st, flag = case.pool.status()
    assert st == sq.SQ_ERR_DEVICE_FLAG and flag == sq.SQ_FLAG_NONFINITE
    assert np.isnan(o[1, 2]).all()
    assert not np.isnan(np.delete(o[1], 2, axis=0)).any()
    after = case.slots()
    off = case.pool.head_offsets
    s1 = case.si_np[1]
    np.testing.assert_array_equal(after[s1, off[2]:off[3]], pre[s1, off[2]:off[3]])
    rows = np.array([0, 2])
    o_ref, ref_bytes = oracle_chunk(wl, case.bits, pre[case.si_np[rows]], x, rows)
    G.close(o[rows], o_ref, "other requests o")
    G.compare_codes(wl, case.bits, after[case.si_np[rows]], ref_bytes, "other requests")


def test_chunk_rejects_bad_arguments():
    wl = CASES["gdn-s"]
    case = G.GpuCase(wl)
    for T in (0, 17):
        x = wl.chunk_inputs(0, max(T, 1))
        q, k, v, a, b = device_chunk(case, x)
        out = torch.empty((wl.batch, wl.n_heads, max(T, 1), wl.d_v), device="cuda")
        with pytest.raises(sq.SqError):
            sq.sq_decode_chunk(case.pool.handle, case.si.data_ptr(), wl.batch, T, q.data_ptr(),
                               k.data_ptr(), v.data_ptr(), a.data_ptr(), b.data_ptr(),
                               out.data_ptr(), 0)
    wcase = G.GpuCase(W.small("window", batch=2, n_heads=2, d=32).scaled(window=4))
    x = wcase.wl.chunk_inputs(0, 3)
    with pytest.raises(sq.SqError):
        run_chunk(wcase, x)


def test_chunk_full_size_sampled():
    """The chunk workload at full size (64 requests x 32 heads, d = 128, 8 tokens per call, the
    launch the bench times): two chunks, a seeded sample of requests checked each time."""
    wl = W.WORKLOADS["chunk"]
    case = G.GpuCase(wl)
    sample = np.sort(np.random.default_rng(7).choice(wl.batch, 4, replace=False))
    for c in range(2):
        chunk_lockstep(case, wl.chunk_inputs(c * wl.tokens, wl.tokens), rows=sample,
                       what=f"chunk {c}")
