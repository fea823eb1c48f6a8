"""The rounding argument behind the decode kernels' exact fit shortcuts, checked on the CPU.

The dual-axis fit (STEPQuant explainer, Key-Row-Aware Dual-Axis Fitting paragraph; scales refit
on the updated state at every step, experimental-setup paragraph) alternates row and column
max-abs passes. In exact arithmetic the second alternation reproduces the first; in fp32 it moves
each scale by a few units of rounding. The kernels (csrc/sq_step.cuh, fit_scales) skip work that
provably cannot change an fp16 scale:

- the whole second alternation, when every row scale lies more than 16 fp32 ulps and every
  column scale more than 24 from an fp16 rounding boundary;
- only the rows near a boundary refit, when every column scale is settled;
- the last column pass, when the multipliers moved by less than every column scale's relative
  distance to a boundary (less 2^-21).

Their claim rests on three facts, restated here in numpy float32 (IEEE single, each operation
correctly rounded, no contraction), on the kernels' own chain of operations (the tile holds
T_ij with M_ij = t_i T_ij; row maximum fl(t_i max_j |T_ij|); w_i = fl(t_i fl(1/fl(r_i Q_i))),
correctly rounded reciprocals and m / Q):

1. fp16 rounding boundaries of values in the normal fp16 range are exactly the fp32 values whose
   low 13 bits are 0x1000;
2. the second row pass gives r'_i in r_i [1 - 12u, 1 + 10u] for rows above the 2^-14 floor,
   w'_i in w_i [1 - 16u, 1 + 18u], and the second column pass c'_j in c_j [1 - 18u, 1 + 20u],
   u = 2^-24;
3. hence each shortcut's fp16 scales equal the full fit's.

The inputs place half of the rows of every head, and some columns of half of the heads, within
a few ulps of an fp16 boundary, so the second alternation does move scales across one (the test asserts that it sees
such moves for rows and for columns), and a predicate that let one of them through would fail
here. Nothing here runs the kernels or the oracle: the GPU tests compare the kernels'
shortcut and full-fit bytes directly.
"""
import numpy as np
import pytest

f32 = np.float32
FLOOR = f32(2.0 ** -14)  # smallest normal fp16, the scale floor
U = 2.0 ** -24


def _rcp(x):
    return (f32(1) / x).astype(f32)


def _row_scale(t, m, Q, quantized):
    """Row scale and column multiplier of each row from its (unfactored) tile maximum m."""
    rq = ((t * m).astype(f32) / Q).astype(f32)
    r = np.minimum(np.maximum(rq, FLOOR), f32(65504))
    w = (t * _rcp((r * Q).astype(f32))).astype(f32)
    return np.where(quantized, r, f32(0)), np.where(quantized, w, f32(0)), rq


def _col_pass(A, w):
    return np.maximum((A * w[:, :, None]).astype(f32).max(axis=1), FLOOR)


def _two_alternations(T, t, Q, quantized):
    A = np.abs(T)
    r1, w1, rq1 = _row_scale(t, A.max(axis=2), Q, quantized)
    c1 = _col_pass(A, w1)
    m2 = (A * _rcp(c1)[:, None, :]).astype(f32).max(axis=2)
    r2, w2, _ = _row_scale(t, m2, Q, quantized)
    c2 = _col_pass(A, w2)
    return r1, w1, c1, r2, w2, c2, rq1


def _margin_ulps(x):
    """Distance of x's bit pattern from the nearest fp16 rounding boundary, in ulps of x."""
    return np.abs((x.view(np.uint32) & 0x1FFF).astype(np.int64) - 0x1000)


def _row_settled(r):
    return (r == 0) | ((r < 32768) & (_margin_ulps(r) > 16))


def _col_settled(c):
    return _margin_ulps(c) > 24


def _fp16_slack(c):
    """Relative distance from c to the nearest fp16 rounding boundary, rounded down."""
    h = c.astype(np.float16)
    hb = h.view(np.uint16)
    hf = h.astype(np.float64)
    up = (hb + 1).view(np.float16).astype(np.float64)
    dn = (hb - 1).view(np.float16).astype(np.float64)
    cd = c.astype(np.float64)
    dist = np.where(cd <= float(FLOOR), 0.5 * (hf + up) - cd,
                    np.minimum(0.5 * (hf + up) - cd, cd - 0.5 * (hf + dn)))
    return np.maximum(dist, 0) / cd * (1 - 2.0 ** -20)


def _heads(rng, kind, n, d):
    """n seeded heads: tile T, row factors t, per-row Q and quantized flags."""
    if kind == "key_rows":  # per-row widths, about 1 % fp16 rows
        b = rng.choice([2, 4, 6, 8, 16], p=[0.35, 0.39, 0.15, 0.10, 0.01], size=(n, d))
    else:
        b = np.broadcast_to(rng.choice([2, 4, 6, 8], size=(n, 1)), (n, d))
    quantized = b != 16
    Q = np.where(quantized, (1 << (np.minimum(b, 8) - 1)) - 1, 1).astype(f32)
    t = np.exp2(rng.uniform(-12, 3, size=(n, d))).astype(f32)
    spread = np.exp2(rng.uniform(-6, 4, size=(n, d, 1)))
    if kind == "laplace":
        T = rng.laplace(size=(n, d, d)) * spread
    elif kind == "spiky":  # a few large entries per row over a small background
        T = rng.standard_normal((n, d, d)) * 0.05
        idx = rng.integers(0, d, size=(n, d, 3))
        np.put_along_axis(T, idx, rng.standard_normal((n, d, 3)) * 4, axis=2)
        T = T * spread
    elif kind == "outlier_rows_cols":  # three rows and three columns scaled up 4x
        T = rng.standard_normal((n, d, d)) * spread
        T[:, :3, :] *= 4
        T[:, :, :3] *= 4
    elif kind == "ties":  # entries on a coarse grid: many equal magnitudes per row and column
        T = rng.integers(-3, 4, size=(n, d, d)) * np.exp2(np.round(np.log2(spread)))
    else:
        T = rng.standard_normal((n, d, d)) * spread
    return T.astype(f32), t, Q, quantized


def _near_boundary(rng, bits_above, k):
    """fp32 values whose low 13 bits are 0x1000 + k (k fp32 ulps from an fp16 rounding
    boundary), with the high bits of the given values."""
    return ((bits_above.view(np.uint32) & ~np.uint32(0x1FFF)) |
            (0x1000 + k).astype(np.uint32)).view(f32)


def _place_near_boundaries(rng, T, t, Q, qz):
    """Put scales where the second alternation can move them across an fp16 boundary: half of
    the rows get a row factor that puts their scale within 24 ulps of a boundary, and in half
    of the heads 16 columns are made to take their scale, within 8 ulps of a boundary, from one
    row that does not have its maximum in any of them (the column's other entries shrunk
    1000x). The other half keeps every column clear of the boundaries often enough that the
    skip of the last column pass applies."""
    n, d, _ = T.shape
    m = np.abs(T).max(axis=2).astype(np.float64)
    r_star = _near_boundary(rng, np.exp2(rng.uniform(-10, 4, size=(n, d))).astype(f32),
                            rng.integers(-24, 25, size=(n, d))).astype(np.float64)
    t_near = (r_star * Q / np.where(m > 0, m, 1)).astype(f32)
    pick = (rng.random((n, d)) < 0.5) & (m > 0) & np.isfinite(t_near) & (t_near > 0)
    t = np.where(pick, t_near, t)
    A = np.abs(T)
    _, w1, _ = _row_scale(t, A.max(axis=2), Q, qz)
    arg = A.argmax(axis=2)
    for h in np.nonzero(rng.random(n) < 0.5)[0]:
        cols = rng.choice(d, size=16, replace=False)
        rows = np.nonzero((w1[h] > 0) & ~np.isin(arg[h], cols))[0]
        if rows.size == 0:
            continue
        c_star = _near_boundary(rng, rng.uniform(0.25, 0.9, size=16).astype(f32),
                                rng.integers(-8, 9, size=16)).astype(np.float64)
        src = rng.choice(rows, size=16)
        T[h][:, cols] *= f32(1e-3)
        T[h, src, cols] = (c_star / w1[h, src]).astype(f32) * rng.choice([-1, 1], size=16)
    return T, t


def test_fp16_rounding_boundaries_are_low_bits_0x1000():
    # every fp16 interval of the scale range [2^-14, 2^16): one ulp below the fp32 midpoint
    # rounds down, one ulp above rounds up, and the midpoint is a tie (to even)
    e = np.arange(-14, 16)
    mant = np.arange(1024)
    lo = (np.exp2(e)[:, None] * (1 + mant[None, :] / 1024.0)).astype(f32).ravel()
    base = lo.view(np.uint32)
    below = (base | 0x0FFF).view(f32)
    mid = (base | 0x1000).view(f32)
    above = (base | 0x1001).view(f32)
    h_lo = lo.astype(np.float16)
    assert np.array_equal(lo, h_lo.astype(f32))  # lo is an fp16 value
    nxt = (h_lo.view(np.uint16) + 1).view(np.float16)  # fp16 infinity above 65504
    with np.errstate(over="ignore"):  # values above 65520 round to infinity, as they should
        h_below, h_mid, h_above = (x.astype(np.float16) for x in (below, mid, above))
    np.testing.assert_array_equal(h_below, h_lo)
    np.testing.assert_array_equal(h_above.view(np.uint16), nxt.view(np.uint16))
    even = np.where(h_lo.view(np.uint16) % 2 == 0, h_lo.view(np.uint16), nxt.view(np.uint16))
    np.testing.assert_array_equal(h_mid.view(np.uint16), even)
    assert np.all(_margin_ulps(mid) == 0) and np.all(_margin_ulps(lo) == 0x1000)


KINDS = ["gauss", "laplace", "spiky", "outlier_rows_cols", "ties", "key_rows"]


@pytest.mark.parametrize("kind", KINDS)
def test_second_alternation_bounds_and_shortcut_exactness(kind):
    rng = np.random.default_rng(20240 + KINDS.index(kind))
    n, d = 300, 128
    seen_row_moves = seen_col_moves = 0
    for _ in range(3):
        T, t, Q, qz = _heads(rng, kind, n, d)
        T, t = _place_near_boundaries(rng, T, t, Q, qz)
        r1, w1, c1, r2, w2, c2, rq1 = _two_alternations(T, t, Q, qz)

        # 2. ratio bounds (rows above the floor; fp16 rows carry no scale)
        live = qz & (rq1 > FLOOR)
        rr = r2[live].astype(np.float64) / r1[live] - 1
        ww = w2[live].astype(np.float64) / w1[live] - 1
        cc = c2.astype(np.float64) / c1 - 1
        assert rr.min() >= -12 * U and rr.max() <= 10 * U, (rr.min() / U, rr.max() / U)
        assert ww.min() >= -16 * U and ww.max() <= 18 * U, (ww.min() / U, ww.max() / U)
        assert cc.min() >= -18 * U and cc.max() <= 20 * U, (cc.min() / U, cc.max() / U)
        floored = qz & (rq1 <= FLOOR)
        assert np.all(r2[floored] >= FLOOR) and np.all(r2[floored] <= float(FLOOR) * (1 + 10 * U))

        # 3. the shortcuts' fp16 scales equal the full fit's
        h = lambda x: x.astype(np.float16).view(np.uint16)  # noqa: E731
        row_moves = h(r2) != h(r1)
        col_moves = h(c2) != h(c1)
        seen_row_moves += int(row_moves.sum())
        seen_col_moves += int(col_moves.sum())
        assert not np.any(row_moves & _row_settled(r1)), "a settled row scale changed"
        assert not np.any(col_moves & _col_settled(c1)), "a settled column scale changed"
        # whole alternation skipped: every row and column settled
        all_settled = _row_settled(r1).all(axis=1) & _col_settled(c1).all(axis=1)
        assert not np.any((row_moves.any(axis=1) | col_moves.any(axis=1)) & all_settled)
        # unsettled rows refit alone: columns settled, rows from the second pass where unsettled
        cols_ok = _col_settled(c1).all(axis=1)
        r_mix = np.where(_row_settled(r1), r1, r2)
        assert np.array_equal(h(r_mix)[cols_ok], h(r2)[cols_ok])
        assert np.array_equal(h(c1)[cols_ok], h(c2)[cols_ok])
        # last column pass skipped: largest multiplier change below the smallest slack
        dw = np.where(w1 > 0, np.abs(w2.astype(np.float64) - w1) / np.where(w1 > 0, w1, 1),
                      np.where(w2 != w1, np.inf, 0.0)) * (1 + 2.0 ** -20)
        skip = dw.max(axis=1) <= _fp16_slack(c1).min(axis=1) - 2.0 ** -21
        assert skip.any()
        assert np.array_equal(h(c1)[skip], h(c2)[skip])
    # the inputs do reach scales that the second alternation moves across a boundary
    assert seen_row_moves > 0 and seen_col_moves > 0, (seen_row_moves, seen_col_moves)
