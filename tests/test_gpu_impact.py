"""GPU parity of the row-impact weighted fit (sq_pool_set_row_impact) against the CPU oracle.

The weighting changes the column passes of every refit (row i counts with the weight
min(1, sqrt(impact_i / mean impact)), and rows weighted below 1 are fit once more against the
final column scales); the cold-start quantization must stay bit-exact with the oracle's, and the
decode step, the chunk step and the window end must follow the oracle within the lockstep
bounds. Impacts are seeded log-uniform scores over two decades.
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
import test_gpu_chunk as CH  # noqa: E402

sqbuild.build()

CASES = {
    "gdn-s": W.small("gdn", batch=3, n_heads=4, d=32),
    "gdn-d128": W.small("gdn", batch=2, n_heads=4, d=128),
    "kda-d128": W.small("kda", batch=2, n_heads=2, d=128),
    "pool-d64": W.small("pool", batch=3, n_heads=3, d=64),
}


def impact_of(wl, seed=21):
    return np.exp(np.random.default_rng(seed).uniform(np.log(0.01), 0.0,
                                                      (wl.n_heads, wl.d_k))).astype(np.float32)


def orc_layout(wl, impact, **kw):
    wl = wl.scaled(**kw) if kw else wl
    return oracle.Layout(wl.n_heads, wl.d_k, wl.d_v, wl.unit, wl.gate, wl.fit_iters, wl.window,
                         wl.n_outliers, row_impact=impact)


def weighted_case(wl, impact):
    case = G.GpuCase(wl, init=False)
    case.pool.set_row_impact(impact)
    case.pool.quantize(case.si, G.to_dev(wl.initial_state(case.si_np)))
    torch.cuda.synchronize()
    return case


def oracle_pool(wl, impact, slot_bytes, **kw):
    p = oracle.Pool(orc_layout(wl, impact, **kw), wl.bits(), slot_bytes.shape[0])
    p.data[:] = slot_bytes.reshape(-1)
    return p


@pytest.mark.parametrize("name", list(CASES) + ["window"])
def test_weighted_quantize_bit_exact(name):
    wl = CASES[name] if name in CASES else W.small("window", batch=2, n_heads=3, d=32).scaled(
        window=4, n_outliers=4)
    imp = impact_of(wl)
    case = weighted_case(wl, imp)
    opool = oracle.Pool(orc_layout(wl, imp), case.bits, wl.slots)
    opool.quantize(case.si_np, wl.initial_state(case.si_np))
    np.testing.assert_array_equal(case.slots()[case.si_np],
                                  opool.data.reshape(wl.slots, -1)[case.si_np])
    plain = oracle.Pool(orc_layout(wl, None), case.bits, wl.slots)
    plain.quantize(case.si_np, wl.initial_state(case.si_np))
    assert not np.array_equal(plain.data, opool.data)  # the weighting did something


@pytest.mark.parametrize("name", list(CASES))
def test_weighted_decode_lockstep(name):
    wl = CASES[name]
    imp = impact_of(wl)
    case = weighted_case(wl, imp)
    mis = tot = 0
    for t in range(3):
        x = wl.step_inputs(t)
        pre = case.slots()
        o_gpu, s_gpu = case.step(x, want_state=True)
        post = case.slots()
        opool = oracle_pool(wl, imp, pre[case.si_np])
        o_ref, s_ref = opool.decode_step(np.arange(wl.batch), x["q"], x["k"], x["v"],
                                         x["alpha"], x["beta"], want_state=True)
        G.close(o_gpu, o_ref, f"step {t} o")
        G.close(s_gpu, s_ref, f"step {t} state")
        m, n = G.compare_codes(wl, case.bits, post[case.si_np],
                               opool.data.reshape(wl.batch, -1), f"step {t}")
        mis, tot = mis + m, tot + n
    assert mis <= max(1, 1e-4 * tot), f"{mis} of {tot} codes differ"


@pytest.mark.parametrize("name", ["gdn-d128", "kda-d128"])
def test_weighted_chunk_lockstep(name):
    wl = CASES[name]
    imp = impact_of(wl)
    case = weighted_case(wl, imp)
    T = 6
    x = wl.chunk_inputs(0, T)
    pre = case.slots()
    o_gpu = CH.run_chunk(case, x)
    post = case.slots()
    opool = oracle_pool(wl, imp, pre[case.si_np], window=T, n_outliers=0)
    n = np.arange(wl.batch)
    for t in range(T):
        xs = {k: np.ascontiguousarray(v[:, :, t]) for k, v in x.items()}
        o_ref = opool.window_step(n, xs["q"], xs["k"], xs["v"], xs["alpha"], xs["beta"])
        G.close(o_gpu[:, :, t], o_ref, f"token {t} o")
    G.compare_codes(wl, case.bits, post[case.si_np], opool.data.reshape(wl.batch, -1), "chunk")


def test_weighted_window_end():
    wl = W.small("gdn", batch=2, n_heads=4, d=64).scaled(window=3, n_outliers=4)
    imp = impact_of(wl)
    case = weighted_case(wl, imp)
    opool = oracle_pool(wl, imp, case.slots()[case.si_np])
    n = np.arange(wl.batch)
    for t in range(wl.window):
        x = wl.step_inputs(t)
        o_gpu, _ = case.step(x)
        o_ref = opool.window_step(n, x["q"], x["k"], x["v"], x["alpha"], x["beta"])
        G.close(o_gpu, o_ref, f"token {t} o")
    G.compare_codes(wl, case.bits, case.slots()[case.si_np], opool.data.reshape(wl.batch, -1),
                    "window end")


def test_removing_the_weighting_restores_the_plain_fit():
    wl = CASES["gdn-s"]
    plain = G.GpuCase(wl)
    case = weighted_case(wl, impact_of(wl))
    case.pool.set_row_impact(None)
    case.pool.quantize(case.si, G.to_dev(wl.initial_state(case.si_np)))
    np.testing.assert_array_equal(case.slots(), plain.slots())
    for t in range(2):
        plain.step(wl.step_inputs(t))
        case.step(wl.step_inputs(t))
    np.testing.assert_array_equal(case.slots(), plain.slots())


@pytest.mark.parametrize("bad", [0.0, -1.0, np.nan, np.inf])
def test_bad_impacts_rejected(bad):
    wl = CASES["gdn-s"]
    case = G.GpuCase(wl)
    imp = impact_of(wl)
    imp[1, 3] = bad
    with pytest.raises(sq.SqError):
        case.pool.set_row_impact(imp)


def test_weighted_full_size_sampled():
    """The GDN layer at full size (64 x 32 heads, d = 128) with a row-impact table: two steps,
    a seeded sample of requests checked against the oracle each time."""
    wl = W.WORKLOADS["gdn"]
    imp = impact_of(wl, seed=5)
    case = weighted_case(wl, imp)
    sample = np.sort(np.random.default_rng(13).choice(wl.batch, 4, replace=False))
    for t in range(2):
        x = wl.step_inputs(t)
        pre = case.slots()
        o_gpu, _ = case.step(x)
        post = case.slots()
        opool = oracle_pool(wl, imp, pre[case.si_np[sample]])
        xs = G.sub_inputs(x, sample)
        o_ref = opool.decode_step(np.arange(sample.size), xs["q"], xs["k"], xs["v"],
                                  xs["alpha"], xs["beta"])
        G.close(o_gpu[sample], o_ref, f"step {t} o")
        G.compare_codes(wl, case.bits, post[case.si_np[sample]],
                        opool.data.reshape(sample.size, -1), f"step {t}")
