"""The offline width allocator (sq_allocate_bits, host code in libsq) against the oracle's exact
optimum, and the oracle's optimum against brute force. CPU only.

Reading (the STEPQuant explainer's lifetime-aware allocation paragraph gives no formula): unit u
has risk R_u = lifetime_u * variance_u; at b bits its score is R_u 2^(-2b); the n_pivots largest
risks stay FP16; the other units get widths in {2, 4, 6, 8} with floor((avg - 2) n' / 2) steps
of 2 bits above 2, minimizing the total score.
"""
import itertools

import numpy as np
import pytest

from bit_recurrent_state_gated_b200 import sq


@pytest.fixture(scope="module")
def lib():
    from bit_recurrent_state_gated_b200 import build
    build.build()
    return sq.lib()


def objective(bits, variance, lifetime):
    R = np.asarray(variance, np.float64) * np.asarray(lifetime, np.float64)
    q = bits != 16
    return float(np.sum(R[q] * np.exp2(-2.0 * bits[q].astype(np.float64))))


def steps_of(avg, nq):
    return min(max(int(np.floor((avg - 2.0) * nq / 2.0 + 1e-9)), 0), 3 * nq)


def brute(variance, lifetime, avg, n_pivots):
    R = np.asarray(variance, np.float64) * np.asarray(lifetime, np.float64)
    order = sorted(range(R.size), key=lambda u: (-R[u], u))
    piv = set(order[:n_pivots])
    rest = [u for u in range(R.size) if u not in piv]
    K = steps_of(avg, len(rest))
    best = None
    for lv in itertools.product(range(4), repeat=len(rest)):
        if sum(lv) != K:
            continue
        val = sum(R[u] * 2.0 ** (-2 * (2 + 2 * l)) for u, l in zip(rest, lv))
        best = val if best is None or val < best else best
    return best, piv


def stats(rng, n):
    var = rng.lognormal(-4.0, 1.0, n).astype(np.float32)
    alpha = rng.uniform(0.5, 0.999, n)
    life = (1.0 / (1.0 - alpha)).astype(np.float32)
    return var, life


@pytest.mark.parametrize("n", [1, 2, 3, 5])
@pytest.mark.parametrize("avg", [2.0, 2.8, 4.0, 5.2, 8.0])
def test_oracle_dp_is_the_brute_force_optimum(oracle, n, avg):
    rng = np.random.default_rng(100 * n + int(avg * 10))
    var, life = stats(rng, n)
    for n_pivots in range(0, min(2, n - 1) + 1):
        bits, obj = oracle.allocate_bits(var.astype(np.float64), life.astype(np.float64), avg,
                                         n_pivots)
        ref, piv = brute(var.astype(np.float64), life.astype(np.float64), avg, n_pivots)
        assert obj == pytest.approx(ref, rel=1e-12)
        assert objective(bits, var, life) == pytest.approx(ref, rel=1e-12)
        assert set(np.flatnonzero(bits == 16)) == piv


@pytest.mark.parametrize("n", [7, 32, 200, 1000])
@pytest.mark.parametrize("avg", [2.5, 4.0, 6.0, 7.5])
def test_greedy_reaches_the_optimum(lib, oracle, n, avg):
    rng = np.random.default_rng(n + int(avg * 100))
    var, life = stats(rng, n)
    n_pivots = min(3, n // 10)
    bits, piv = sq.sq_allocate_bits(var, life, avg, n_pivots)
    ref_bits, ref_obj = oracle.allocate_bits(var.astype(np.float64), life.astype(np.float64),
                                             avg, n_pivots)
    assert objective(bits, var, life) == pytest.approx(ref_obj, rel=1e-9)
    np.testing.assert_array_equal(bits == 16, ref_bits == 16)
    np.testing.assert_array_equal(piv, (bits == 16).astype(np.uint8))
    q = bits != 16
    assert set(np.unique(bits[q])) <= {2, 4, 6, 8}
    assert int(np.sum(bits[q].astype(int) - 2)) == 2 * steps_of(avg, int(q.sum()))


def test_larger_risk_never_gets_fewer_bits(lib):
    rng = np.random.default_rng(5)
    var, life = stats(rng, 500)
    bits, _ = sq.sq_allocate_bits(var, life, 5.0, 0)
    R = var.astype(np.float64) * life
    o = np.argsort(-R, kind="stable")
    assert np.all(np.diff(bits[o].astype(int)) <= 0)


def test_special_cases(lib):
    n = 12
    one = np.ones(n, np.float32)
    for avg, want in ((2.0, 2), (8.0, 8)):
        bits, _ = sq.sq_allocate_bits(one, one, avg, 0)
        assert np.all(bits == want)
    bits, _ = sq.sq_allocate_bits(one, one, 5.0, 0)  # equal risks: balanced, lower index first
    assert np.all(bits == np.array([6] * 6 + [4] * 6))
    var = np.zeros(n, np.float32)
    var[3] = 1.0
    bits, piv = sq.sq_allocate_bits(var, one, 2.5, 1)  # the only risky unit becomes the pivot
    assert bits[3] == 16 and piv[3] == 1 and piv.sum() == 1


def test_bit_map_is_a_valid_layout(lib):
    rng = np.random.default_rng(9)
    var, life = stats(rng, 32)
    bits, piv = sq.sq_allocate_bits(var, life, 6.0, 2)
    lay = sq.Layout(4, 32, 128, 128)
    assert sq.sq_pool_required_bytes(lay, bits, piv) > 0


@pytest.mark.parametrize("bad", ["avg_low", "avg_high", "pivots", "neg", "nan"])
def test_rejects_bad_arguments(lib, bad):
    n = 8
    var, life = np.ones(n, np.float32), np.ones(n, np.float32)
    avg, n_pivots = 4.0, 1
    if bad == "avg_low":
        avg = 1.5
    elif bad == "avg_high":
        avg = 8.5
    elif bad == "pivots":
        n_pivots = n
    elif bad == "neg":
        var[2] = -1.0
    else:
        life[1] = np.nan
    with pytest.raises(sq.SqError) as e:
        sq.sq_allocate_bits(var, life, avg, n_pivots)
    assert e.value.status == sq.SQ_ERR_INVALID_ARG
