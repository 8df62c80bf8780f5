"""Property pins of the oracle over generated inputs (hypothesis).

Each property follows from the definitions or from plain mathematics, not
from the oracle's own formulas: a code is the nearest of the grid's levels
(found by trying every level), the rounding error of an unclamped weight is
at most half a step, the activation mean equals the exact rational mean
(Python integers and fractions), negating or doubling the weights acts on
the results as the definitions say, and the searched error never exceeds
plain round-to-nearest.  The generators reach fp16 subnormals, zeros, exact
half-step ties and the largest fp16 magnitudes.  Runs are derandomised, so
every run checks the same examples.
"""
from fractions import Fraction

import numpy as np
import pytest
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st
from hypothesis.extra import numpy as hnp

import oracle

SETTINGS = settings(max_examples=80, deadline=None, derandomize=True,
                    suppress_health_check=[HealthCheck.too_slow])

f16 = st.floats(width=16, allow_nan=False, allow_infinity=False)
# finite fp16 weights of moderate size (so that w * s stays far from overflow)
f16_w = st.floats(min_value=-8.0, max_value=8.0, width=16, allow_nan=False)
scale = st.floats(min_value=2.0 ** -6, max_value=2.0 ** 6, width=32, allow_nan=False)


def _group(n):
    return hnp.arrays(np.float16, n, elements=f16_w)


def _scales(n):
    return hnp.arrays(np.float32, n, elements=scale)


def _nearest_level(v, qs, lo, hi, shift=0):
    """The level q in lo..hi nearest to v / qs by trying every one (ties: the
    even value of q - shift, as round-half-to-even of v / qs gives)."""
    best, best_d = None, None
    for q in range(lo, hi + 1):
        d = abs(Fraction(float(v)) - (q - shift) * Fraction(float(qs)))
        if best is None or d < best_d or (d == best_d and (q - shift) % 2 == 0):
            best, best_d = q, d
    return best


@SETTINGS
@given(st.sampled_from([8, 32, 128]).flatmap(lambda n: st.tuples(_group(n), _scales(n))),
       st.booleans())
def test_symmetric_codes_are_nearest_levels(ws_pair, fp32_scale):
    w, s = ws_pair
    flags = oracle.SCALE_FP32 if fp32_scale else 0
    q, qs, bad = oracle.fake_quant_group(w, s, flags)
    assert not bad
    assert np.all((q >= -7) & (q <= 7))
    prod = w.astype(np.float32) * s            # fp32 products (IEEE, one rounding)
    if qs == 0.0:
        assert np.all(q == 0) and np.all(prod == 0)
        return
    for v, c in zip(prod, q):
        assert c == _nearest_level(v, qs, -7, 7)
        if abs(Fraction(float(v))) <= Fraction(15, 2) * Fraction(qs):
            assert abs(Fraction(float(v)) - c * Fraction(qs)) <= Fraction(qs) / 2


@SETTINGS
@given(st.sampled_from([8, 32]).flatmap(lambda n: st.tuples(_group(n), _scales(n))))
def test_symmetric_sign_and_power_of_two_scaling(ws_pair):
    """Negating w negates every code (ties go to even either way); doubling
    w (exact in fp16 below 8 * 2) doubles the fp32 group scale exactly and
    keeps the codes."""
    w, s = ws_pair
    q, qs, _ = oracle.fake_quant_group(w, s, oracle.SCALE_FP32)
    qn, qsn, _ = oracle.fake_quant_group(-w, s, oracle.SCALE_FP32)
    assert qsn == qs and np.array_equal(qn, -q)
    q2, qs2, _ = oracle.fake_quant_group((w.astype(np.float32) * 2).astype(np.float16), s,
                                         oracle.SCALE_FP32)
    if qs > 2.0 ** -100:                     # far from the fp32 subnormal range
        assert qs2 == 2 * qs and np.array_equal(q2, q)


@SETTINGS
@given(st.sampled_from([8, 32, 128]).flatmap(lambda n: st.tuples(_group(n), _scales(n))))
def test_asymmetric_codes_are_nearest_shifted_levels(ws_pair):
    w, s = ws_pair
    q, qs, z = oracle.fake_quant_group_asym(w, s)
    assert 0 <= z <= 15 and np.all(q <= 15)
    prod = w.astype(np.float32) * s
    for v, c in zip(prod, q):
        assert c == _nearest_level(v, qs, 0, 15, shift=z)


@SETTINGS
@given(hnp.arrays(np.float16, st.tuples(st.integers(1, 40), st.sampled_from([8, 16])),
                  elements=f16))
def test_act_stats_is_the_exact_mean(X):
    """mean_t |X[t, j]| exactly (every |fp16| is an integer multiple of
    2^-24), rounded once to fp64 and then to fp32, for any token order."""
    x = oracle.act_stats(X)
    T = X.shape[0]
    for j in range(X.shape[1]):
        exact = sum(Fraction(abs(float(v))) for v in X[:, j]) / T
        assert x[j] == np.float32(float(exact))
    perm = np.random.default_rng(T).permutation(T)
    assert np.array_equal(oracle.act_stats(X[perm]), x)


@SETTINGS
@given(st.integers(1, 4).flatmap(lambda r: hnp.arrays(
           np.float16, (8 * r, 64), elements=f16_w)),
       hnp.arrays(np.float32, 64, elements=st.floats(min_value=0.0, max_value=100.0,
                                                      width=32)),
       st.sampled_from([1, 5, 20]))
def test_search_never_worse_than_round_to_nearest(W, x, n_grid):
    """Grid point 0 is s = 1 (plain round-to-nearest); the chosen error is
    the first minimum and never above it."""
    err, best, s = oracle.scale_search([W], x, 32, n_grid)
    assert np.all(np.isfinite(err))
    assert best == int(np.argmin(err)) and err[best] <= err[0]
    if n_grid == 1:
        assert best == 0 and np.all(s == 1.0)


@pytest.mark.parametrize("n", [1, 2, 3])
def test_geomean_of_equal_members_is_the_member(n):
    rng = np.random.default_rng(n)
    s = (rng.random(64) * 10 + 1e-3).astype(np.float32)
    assert np.array_equal(oracle.geomean_scales([s] * n), s)


@SETTINGS
@given(st.integers(1, 3).flatmap(
           lambda r: hnp.arrays(np.float16, (8 * r, 64), elements=f16_w)),
       hnp.arrays(np.float32, 64, elements=scale), st.sampled_from([7, 8]))
def test_pack_round_trip_and_dequant(W, s, zp):
    """Unpacked codes minus the zero point, times the stored fp16 scale, give
    exactly the group fake-quant's q * q_scale; qzeros holds the zero point
    in every nibble."""
    g = 32
    qw, sc, qz = oracle.quantize_pack(W, s, g, zp)
    u = oracle.unpack(qw, W.shape[0]).astype(np.int64)
    assert np.all(qz == np.int32(np.uint32(zp * 0x11111111).view(np.int32)))
    for r in range(W.shape[0]):
        for k in range(W.shape[1] // g):
            q, qs, _ = oracle.fake_quant_group(W[r, k * g:(k + 1) * g], s[k * g:(k + 1) * g])
            assert np.array_equal(u[r, k * g:(k + 1) * g] - zp, q)
            assert float(sc[k, r]) == qs


@SETTINGS
@given(st.sampled_from([8, 32]).flatmap(lambda n: st.tuples(_group(n), _scales(n))),
       st.integers(0, 19))
def test_clipped_codes_are_nearest_levels(ws_pair, i):
    """With the range shrunk to c_i * max|ws|, every code is still the nearest
    of the 15 levels of the clipped scale; ratio 0 is the plain quantiser."""
    w, s = ws_pair
    c = oracle.clip_ratio(i)
    q, qs = oracle.fake_quant_group_clip(w, s, c)
    prod = w.astype(np.float32) * s
    assert np.all((q >= -7) & (q <= 7))
    if qs > 0:
        for v, code in zip(prod, q):
            assert code == _nearest_level(v, qs, -7, 7)
    if i == 0:
        q0, qs0, _ = oracle.fake_quant_group(w, s)
        assert qs == qs0 and np.array_equal(q, q0)


@SETTINGS
@given(st.integers(1, 6).flatmap(lambda r: hnp.arrays(np.float16, (r, 16), elements=f16_w)))
def test_weight_mean_bounds(W):
    """|w| / max|w| of a row lies in [0, 1], so the mean does too; a channel
    holding every row's largest magnitude has mean exactly 1."""
    wm = oracle.weight_mean([W])
    assert np.all((wm >= 0) & (wm <= 1))
    W2 = W.copy()
    W2[:, 0] = np.float16(16.0)              # above every other |w| (all <= 8)
    assert oracle.weight_mean([W2])[0] == 1.0


pos_x = st.floats(min_value=0.0, max_value=1e4, width=32, allow_nan=False)


@SETTINGS
@given(hnp.arrays(np.float32, st.integers(2, 40), elements=pos_x), st.sampled_from([1, 7, 20]))
def test_scale_table_rows(x, n_grid):
    """Row 0 is exactly 1; every row is monotone in x (pow is, and one
    rounding keeps the order), which is what lets the GPU take the row's
    extremes from the extreme x; after the normalisation the row's largest
    times its smallest entry is 1 up to the two fp32 roundings."""
    S = oracle.scale_table(x, n_grid)
    assert np.all(S[0] == 1.0)
    order = np.argsort(x, kind="stable")
    for i in range(n_grid):
        row = S[i][order].astype(np.float64)
        assert np.all(np.diff(row) >= 0)
        assert abs(row.max() * row.min() - 1.0) <= 2.0 ** -22


@SETTINGS
@given(hnp.arrays(np.float32, 32, elements=pos_x),
       hnp.arrays(np.float64, 32, elements=st.floats(min_value=0.0, max_value=1.0)),
       st.sampled_from([1, 20]))
def test_duo_table_normalisation(x, wm, n_grid):
    """Every duo row is positive and normalised: largest times smallest entry
    is 1 up to the two fp32 roundings."""
    S = oracle.scale_table_duo(x, wm, n_grid).astype(np.float64)
    assert np.all(S > 0)
    for i in range(n_grid):
        assert abs(S[i].max() * S[i].min() - 1.0) <= 2.0 ** -22


@settings(max_examples=25, deadline=None, derandomize=True,
          suppress_health_check=[HealthCheck.too_slow])
@given(st.integers(1, 12).flatmap(lambda T: hnp.arrays(np.float16, (T, 64), elements=f16_w)),
       st.integers(1, 2).flatmap(lambda r: hnp.arrays(np.float16, (8 * r, 64), elements=f16_w)))
def test_output_error_nonnegative_and_quadratic_in_x(X, W):
    """||X (W - W_hat)^T||^2 is a sum of squares; with the same x (so the
    same scale table and W_hat), doubling X (exact in fp16 here) scales every
    product and partial sum by a power of two, so the error becomes exactly
    four times larger.  (Recomputing x from 2X would not do: the clamp at
    1e-4 and pow's rounding do not commute with the doubling.)"""
    x = oracle.act_stats(X)
    err = oracle.output_error(X, W, x, 32, 5)
    assert np.all(err >= 0)
    X2 = (X.astype(np.float32) * 2).astype(np.float16)
    err2 = oracle.output_error(X2, W, x, 32, 5)
    assert np.array_equal(err2, 4 * err)


def _f32_neighbours(r):
    r = np.float32(r)
    return np.nextafter(r, np.float32(-np.inf)), np.nextafter(r, np.float32(np.inf))


@SETTINGS
@given(hnp.arrays(np.float32, 2, elements=st.floats(min_value=2.0 ** -20, max_value=2.0 ** 20,
                                                     width=32)))
def test_geomean_of_two_is_the_rounded_square_root(ab):
    """For two members the shared scale is sqrt(a b) rounded once to fp32:
    r is the fp32 value whose neighbours' midpoints bracket sqrt(a b),
    decided exactly by comparing squares of rationals."""
    a, b = ab
    r = oracle.geomean_scales([np.array([a], np.float32), np.array([b], np.float32)])[0]
    P = Fraction(float(a)) * Fraction(float(b))
    lo, hi = _f32_neighbours(r)
    m_lo = (Fraction(float(lo)) + Fraction(float(r))) / 2
    m_hi = (Fraction(float(r)) + Fraction(float(hi))) / 2
    assert m_lo * m_lo <= P <= m_hi * m_hi


@SETTINGS
@given(st.sampled_from([8, 32]).flatmap(lambda n: st.tuples(_group(n), _scales(n),
                                                            st.integers(0, n - 1))),
       st.sampled_from([np.nan, np.inf, -np.inf]))
def test_nonfinite_weight_flags_the_group(wsk, bad_value):
    w, s, k = wsk
    w = w.copy()
    w[k] = bad_value
    assert oracle.fake_quant_group(w, s)[2]


@SETTINGS
@given(hnp.arrays(np.float16, st.tuples(st.integers(2, 30), st.just(8)), elements=f16_w),
       st.data())
def test_act_stats_nonfinite_columns(X, data):
    """A column holding an infinity has mean inf, one holding a NaN has mean
    NaN (NaN wins over inf), wherever they sit; other columns are unaffected."""
    X = X.copy()
    T = X.shape[0]
    ti = data.draw(st.integers(0, T - 1))
    tn = data.draw(st.integers(0, T - 1))
    ref = oracle.act_stats(X)
    X[ti, 2] = np.inf
    X[ti, 5] = -np.inf
    X[tn, 5] = np.nan if tn != ti else X[tn, 5]
    X[tn, 6] = np.nan
    x = oracle.act_stats(X)
    assert x[2] == np.inf and np.isnan(x[6])
    assert (np.isnan(x[5]) if tn != ti else x[5] == np.inf)
    keep = [0, 1, 3, 4, 7]
    assert np.array_equal(x[keep], ref[keep])
