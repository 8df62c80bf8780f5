"""Pins of the CPU oracle against what the pages and the mathematics fix.

Each test checks the oracle against something other than itself: a worked
example printed on a page, a closed form, a special case that reduces to a
textbook routine, an invariant, or brute force on tiny inputs.  No expected
value here comes from the CUDA path.
"""
import math

import numpy as np
import pytest

import oracle


def _floats(s):
    return [float(v) for v in s.split()]


def _nearest_level(v):
    """Nearest integer in [-7, 7] to the fp32 quotient v, ties to even --
    found by enumerating the 15 levels (not by calling a rounding routine)."""
    v = float(v)
    return min(range(-7, 8), key=lambda q: (abs(v - q), q % 2))


# ---------------------------------------------------------------- worked --
# "Weight-Only Quantization: GPTQ and AWQ", section 4 "Tiny example".

def test_worked_example_fp32_scale(golden):
    g = golden("worked_example.txt")
    w = np.array(_floats(g["w"]), np.float32)
    x = np.array(_floats(g["x"]), np.float64)
    sc = np.array(_floats(g["awq_scale"]), np.float32)
    wd = w.astype(np.float64)

    assert round(float(wd @ x), 3) == float(g["exact_dot"])

    qn, qs_n, bad = oracle.fake_quant_group(w, np.ones(4, np.float32), oracle.SCALE_FP32)
    assert not bad
    assert list(qn) == [4, -3, 7, 1]
    naive = qn.astype(np.float64) * qs_n
    assert np.allclose(np.round(naive, 3), _floats(g["naive_deq"]), atol=0)
    assert round(float(naive @ x), 3) == float(g["naive_dot"])

    qa, qs_a, bad = oracle.fake_quant_group(w, sc, oracle.SCALE_FP32)
    assert list(qa) == [7, -1, 3, 0]
    awq = qa.astype(np.float64) * qs_a / sc.astype(np.float64)
    assert np.allclose(np.round(awq, 3), _floats(g["awq_deq"]), atol=0)
    assert round(float(awq @ x), 3) == float(g["awq_dot"])

    exact = float(wd @ x)
    assert round(abs(exact - float(naive @ x)), 2) == float(g["naive_error"])
    assert round(abs(exact - float(awq @ x)), 3) == float(g["awq_error"])


def test_worked_example_codes_fp16_scale(golden):
    """The INT4 codes of the example do not depend on rounding q_scale to fp16."""
    g = golden("worked_example.txt")
    w = np.array(_floats(g["w"]), np.float32)
    sc = np.array(_floats(g["awq_scale"]), np.float32)
    qn, qs_n, _ = oracle.fake_quant_group(w, np.ones(4, np.float32), 0)
    qa, qs_a, _ = oracle.fake_quant_group(w, sc, 0)
    assert list(qn) == [4, -3, 7, 1] and list(qa) == [7, -1, 3, 0]
    # the fp16 group scale is the fp16 value nearest to max|ws| / 7
    assert qs_n == float(np.float16(np.float32(0.8) / np.float32(7)))
    assert qs_a == float(np.float16(np.float32(2.0) / np.float32(7)))


def test_weighted_error_of_worked_example():
    """Weight-space score of the example = sum ((w - w_hat) x)^2, by hand."""
    w = np.array([[0.5, -0.3, 0.8, 0.1]], np.float16)
    x = np.array([10, 0.1, 0.1, 0.1], np.float32)
    s = np.array([4, 1, 1, 1], np.float32)
    e = oracle.weighted_error(w, x, s, 4, oracle.SCALE_FP32)
    wf = w.astype(np.float32)[0]
    qs = float(np.float32(abs(wf[0] * 4)) / np.float32(7))
    codes = [7, -1, 3, 0]
    hand = sum(((float(wf[j]) - codes[j] * qs / float(s[j])) * float(x[j])) ** 2
               for j in range(4))
    assert e == pytest.approx(hand, rel=1e-12)


# ------------------------------------------------------------- rounding --

@pytest.mark.parametrize("w1,code", [(0.3125, 2), (0.4375, 4), (-0.3125, -2),
                                     (-0.4375, -4), (0.0625, 0), (0.1875, 2)])
def test_rint_ties_to_even(w1, code):
    """Exact half-way quotients round to the even level (round / rint)."""
    w = np.array([0.875, w1], np.float32)     # q_scale = 0.875 / 7 = 0.125 exactly
    q, qs, _ = oracle.fake_quant_group(w, np.ones(2, np.float32), 0)
    assert qs == 0.125
    assert q[1] == code


def test_codes_are_nearest_level_bruteforce():
    rng = np.random.default_rng(11)
    for trial in range(200):
        n = 32
        w = (rng.standard_normal(n) * 0.02).astype(np.float16).astype(np.float32)
        s = np.exp(rng.standard_normal(n)).astype(np.float32)
        q, qs, _ = oracle.fake_quant_group(w, s, 0)
        ws = (w * s).astype(np.float32)
        m = float(np.max(np.abs(ws)))
        assert qs == float(np.float16(np.float32(m) / np.float32(7)))
        for j in range(n):
            quot = np.float32(ws[j]) / np.float32(qs)
            assert q[j] == _nearest_level(quot)


def test_dequant_error_within_half_step():
    """|w s - q q_scale| <= q_scale / 2 for every weight that is not clamped
    ("up to s/2 per weight", section 2 of the GPTQ/AWQ tutorial page)."""
    rng = np.random.default_rng(12)
    for _ in range(100):
        w = (rng.standard_normal(128) * 0.02).astype(np.float16).astype(np.float32)
        s = np.exp(rng.standard_normal(128) * 2).astype(np.float32)
        q, qs, _ = oracle.fake_quant_group(w, s, 0)
        ws = (w * s).astype(np.float64)
        err = np.abs(ws - q.astype(np.float64) * qs)
        unclamped = np.abs(q) < 7
        assert np.all(err[unclamped] <= qs / 2 * (1 + 1e-6))
        # a clamped code only occurs at the group maximum
        assert np.all(np.abs(ws[~unclamped]) >= 6.5 * qs)


def test_zero_group_and_fp16_overflow():
    q, qs, bad = oracle.fake_quant_group(np.zeros(8, np.float32), np.ones(8, np.float32), 0)
    assert qs == 0.0 and not bad and not q.any()
    big = np.array([1e6, -3e5, 1.0, 0.0], np.float32)
    q, qs, _ = oracle.fake_quant_group(big, np.ones(4, np.float32), 0)
    assert qs == 65504.0              # held at the largest finite fp16
    assert q[0] == 7 and q[1] == -5   # 1e6/65504 = 15.3 -> clamped to 7
    q, qs, bad = oracle.fake_quant_group(np.array([1, np.nan], np.float32),
                                         np.ones(2, np.float32), 0)
    assert bad and math.isnan(qs)


# ---------------------------------------------------------- scale table --

def test_scale_table_closed_form_two_levels():
    """x taking two values a (first half) and b: s_i = (a/b)^(+-alpha/2)."""
    a, b = np.float32(7.5), np.float32(0.03)
    x = np.array([a] * 8 + [b] * 8, np.float32)
    S = oracle.scale_table(x, 20)
    for i in range(20):
        al = i / 20
        hi = (float(a) / float(b)) ** (al / 2)
        assert S[i, 0] == np.float32(hi)
        assert S[i, 15] == np.float32(1.0 / hi)


def test_scale_table_alpha0_is_one_and_normalised():
    rng = np.random.default_rng(3)
    x = np.exp(rng.standard_normal(512) * 2).astype(np.float32)
    x[5] = 0.0          # clamped to 1e-4 before the power
    x[6] = 1e-4
    S = oracle.scale_table(x, 20)
    assert np.all(S[0] == 1.0)
    assert np.all(S[:, 5] == S[:, 6])
    for i in range(20):
        assert float(S[i].max()) * float(S[i].min()) == pytest.approx(1.0, rel=1e-6)
        # s is monotone in x for alpha > 0
        if i:
            order = np.argsort(np.maximum(x, np.float32(1e-4)), kind="stable")
            assert np.all(np.diff(S[i][order]) >= 0)


# ----------------------------------------------------------------- stats --

def test_act_stats_closed_form():
    T, d = 3, 4
    X = np.array([[1, -2, 0.5, 0], [-1, 2, 0.25, 0], [1, -2, -0.25, 1]], np.float16)
    x = oracle.act_stats(X)
    assert list(x) == [1.0, 2.0, np.float32(1.0 / 3.0), np.float32(1.0 / 3.0)]
    # the mean is exact: independent of token order, bit for bit
    rng = np.random.default_rng(5)
    Y = (rng.standard_normal((257, 64)) * np.exp(rng.standard_normal(64) * 3)).astype(np.float16)
    ref = oracle.act_stats(Y)
    for _ in range(3):
        assert np.array_equal(oracle.act_stats(Y[rng.permutation(257)]), ref)
    exact = [float(np.float32(sum(abs(float(v)) for v in Y[:, j]) / 257)) for j in range(64)]
    # python sums in fp64 here; equal except where fp64 rounding of the sum matters
    assert np.allclose(ref, exact, rtol=1e-7, atol=0)


def test_act_stats_nonfinite():
    X = np.ones((4, 3), np.float16)
    X[1, 0] = np.inf
    X[2, 1] = np.nan
    x = oracle.act_stats(X)
    assert x[0] == np.inf and math.isnan(x[1]) and x[2] == 1.0


# ---------------------------------------------------------------- search --

def test_alpha0_error_is_rtn_bruteforce():
    """Grid index 0 gives s = 1, i.e. plain round-to-nearest; its error equals
    a brute-force nearest-level quantisation scored by sum ((w - w_hat) x)^2.
    The searched error is never above it ("AWQ scaling" section)."""
    rng = np.random.default_rng(21)
    d_out, d_in, g = 8, 64, 32
    W = (rng.standard_normal((d_out, d_in)) * 0.02).astype(np.float16)
    x = np.exp(rng.standard_normal(d_in)).astype(np.float32)
    err, best, s_best = oracle.scale_search([W], x, g, 20)
    Wf = W.astype(np.float32)
    total = 0.0
    for r in range(d_out):
        for k in range(d_in // g):
            grp = Wf[r, k * g:(k + 1) * g]
            qs = float(np.float16(np.float32(np.max(np.abs(grp))) / np.float32(7)))
            for j in range(g):
                q = _nearest_level(np.float32(grp[j]) / np.float32(qs))
                total += ((float(grp[j]) - q * qs) * float(x[k * g + j])) ** 2
    assert err[0] == pytest.approx(total, rel=1e-12)
    assert err[best] <= err[0]
    assert err[best] == err.min() and best == int(np.argmin(err))


def test_uniform_x_gives_ties_and_first_index():
    """x constant => every s_i = 1 => all errors tie => index 0 wins."""
    rng = np.random.default_rng(22)
    W = (rng.standard_normal((16, 128)) * 0.02).astype(np.float16)
    x = np.full(128, 3.0, np.float32)
    err, best, s_best = oracle.scale_search([W], x, 128, 20)
    assert np.all(err == err[0]) and best == 0 and np.all(s_best == 1.0)


def test_shared_input_segments_add():
    """A search over segments sharing x scores the sum of their errors
    (the grid search concatenates the linears of a group on dim 0)."""
    rng = np.random.default_rng(23)
    W1 = (rng.standard_normal((16, 64)) * 0.02).astype(np.float16)
    W2 = (rng.standard_normal((8, 64)) * 0.02).astype(np.float16)
    x = np.exp(rng.standard_normal(64) * 2).astype(np.float32)
    e12, b12, _ = oracle.scale_search([W1, W2], x, 32, 20)
    ecat, bcat, _ = oracle.scale_search([np.concatenate([W1, W2])], x, 32, 20)
    e1, _, _ = oracle.scale_search([W1], x, 32, 20)
    e2, _, _ = oracle.scale_search([W2], x, 32, 20)
    assert np.allclose(e12, e1 + e2, rtol=1e-12)
    assert np.allclose(e12, ecat, rtol=1e-12) and b12 == bcat


def test_salient_channel_search_beats_rtn():
    """With one loud input channel the search picks alpha > 0 and lowers the
    weighted error well below RTN (the effect the worked example shows)."""
    rng = np.random.default_rng(24)
    W = (rng.standard_normal((64, 128)) * 0.02).astype(np.float16)
    x = np.full(128, 0.1, np.float32)
    x[:2] = 10.0
    err, best, _ = oracle.scale_search([W], x, 128, 20)
    assert best > 0 and err[best] < 0.8 * err[0]


# ------------------------------------------------------------------ pack --

def _rows_with_codes(codes_per_row, width=32):
    """fp16 rows whose group max sets q_scale = 0.125 and whose column 1 holds
    the given signed code."""
    W = np.zeros((len(codes_per_row), width), np.float16)
    for r, q in enumerate(codes_per_row):
        W[r, :] = np.float16(q * 0.125)
        W[r, 0] = np.float16(-0.875)
    return W


def test_pack_order_golden(golden):
    g = golden("pack_order.txt")
    assert [int(v) for v in g["order"].split()] == [0, 2, 4, 6, 1, 3, 5, 7]
    W = _rows_with_codes([r - 7 for r in range(8)])
    qw, sc, qz = oracle.quantize_pack(W, None, 32, 8)
    assert qw.shape == (32, 1) and sc.shape == (1, 8) and qz.shape == (1, 1)
    assert np.uint32(qw[1, 0]) == int(g["word_rows_r_plus_1"], 16)
    assert np.uint32(qw[0, 0]) == int(g["word_all_minus7"], 16)
    assert np.uint32(qz[0, 0]) == int(g["qzeros_zp8"], 16)
    assert np.all(sc == np.float16(0.125))
    qw7, _, _ = oracle.quantize_pack(W, None, 32, 7)
    assert np.uint32(qw7[1, 0]) == int(g["word_rows_r_zp7"], 16)


@pytest.mark.parametrize("zp", [8, 7])
def test_pack_roundtrip_and_zero_requant_error(zp):
    """unpack(pack) returns the codes, and the runtime dequant (u - zero) * scale
    equals the signed group dequant q * q_scale exactly (exporter step 4)."""
    rng = np.random.default_rng(31)
    d_out, d_in, g = 48, 256, 64
    W = (rng.standard_normal((d_out, d_in)) * 0.02).astype(np.float16)
    s = np.exp(rng.standard_normal(d_in)).astype(np.float32)
    qw, sc, qz = oracle.quantize_pack(W, s, g, zp)
    u = oracle.unpack(qw, d_out)
    Wf = W.astype(np.float32)
    for r in range(d_out):
        for k in range(d_in // g):
            q, qs, _ = oracle.fake_quant_group(Wf[r, k * g:(k + 1) * g], s[k * g:(k + 1) * g], 0)
            assert np.array_equal(u[r, k * g:(k + 1) * g].astype(np.int32), q.astype(np.int32) + zp)
            assert sc[k, r] == np.float16(qs)
            deq_rt = (u[r, k * g:(k + 1) * g].astype(np.float64) - zp) * float(sc[k, r])
            assert np.array_equal(deq_rt, q.astype(np.float64) * qs)
    assert u.min() >= zp - 7 and u.max() <= zp + 7


def test_bits_per_weight_and_stack_size():
    """4 + 16/128 + 4/128 ~ 4.16 bits per weight at g128 (storage sections of
    the architecture and tutorial pages); the Qwen3-8B linear stack is
    13.9 GB in fp16 and its INT4 codes are 4.0x smaller (results section)."""
    d_out, d_in, g = 64, 256, 128
    W = np.zeros((d_out, d_in), np.float16)
    qw, sc, qz = oracle.quantize_pack(W, None, g, 8)
    bits = 8 * (qw.nbytes + sc.nbytes + qz.nbytes) / (d_out * d_in)
    assert bits == 4 + 16 / 128 + 4 / 128 and round(bits, 2) == 4.16
    from post_int4_weight_b200.workloads import WORKLOADS
    n = WORKLOADS["qwen3_8b_stack36"].params
    assert round(2 * n / 1e9, 1) == 13.9
    assert round(n / 2 / 1e9, 1) == 3.5 and (2 * n) / (n / 2) == 4.0


# ----------------------------------------------------------- output mode --

def test_output_mode_diagonal_x_equals_weight_space():
    """X = diag(c) => ||X dW^T||^2 = sum_{r,j} dW[r,j]^2 c_j^2, the weight-space
    score with x = c."""
    rng = np.random.default_rng(41)
    d_out, d_in, g = 16, 64, 32
    W = (rng.standard_normal((d_out, d_in)) * 0.02).astype(np.float16)
    c = np.exp(rng.standard_normal(d_in)).astype(np.float16)
    X = np.diag(c.astype(np.float32)).astype(np.float16)
    x = c.astype(np.float32)
    eo = oracle.output_error(X, W, x, g, 20)
    ew, _, _ = oracle.scale_search([W], x, g, 20)
    assert np.allclose(eo, ew, rtol=1e-12)


def test_output_mode_token_additivity_and_scaling():
    rng = np.random.default_rng(42)
    d_out, d_in, g, T = 8, 64, 32, 12
    W = (rng.standard_normal((d_out, d_in)) * 0.02).astype(np.float16)
    X = rng.standard_normal((T, d_in)).astype(np.float16)
    x = np.exp(rng.standard_normal(d_in)).astype(np.float32)
    e = oracle.output_error(X, W, x, g, 20)
    e1 = oracle.output_error(X[:5], W, x, g, 20)
    e2 = oracle.output_error(X[5:], W, x, g, 20)
    assert np.allclose(e, e1 + e2, rtol=1e-12)
    e4 = oracle.output_error((2 * X.astype(np.float32)).astype(np.float16), W, x, g, 20)
    assert np.allclose(e4, 4 * e, rtol=1e-12)


# ------------------------------------------------------------- clip search --
# The pages name the clip search (pipeline step 5 of the AWQ architecture
# page: shrink the quantisation range per output channel to cut rounding
# error on outliers) without a formula; the reading pinned here: ratios
# c_i = (20 - i) / 20, range c_i * max|w s|, codes saturating at +-7, the
# same activation-weighted error, first minimum per (row, group).

def test_clip_ratio_grid():
    assert oracle.clip_ratio(0) == 1.0
    assert oracle.clip_ratio(10) == 0.5          # exactly representable
    for i in range(20):
        assert oracle.clip_ratio(i) == float(np.float32((20 - i) / 20))


def test_clip_ratio_one_is_the_unclipped_quantiser():
    rng = np.random.default_rng(41)
    for _ in range(100):
        n = 128
        w = (rng.standard_normal(n) * 0.02).astype(np.float16).astype(np.float32)
        s = np.exp(rng.standard_normal(n)).astype(np.float32)
        q0, qs0, _ = oracle.fake_quant_group(w, s, 0)
        q1, qs1 = oracle.fake_quant_group_clip(w, s, 1.0, 0)
        assert np.array_equal(q0, q1) and qs0 == qs1


@pytest.mark.parametrize("i", [1, 3, 6, 9, 14])
def test_clipped_codes_are_nearest_of_15_levels(i):
    """With the range shrunk to c * max|ws|, every code is the nearest of the
    15 levels -7..7 to the IEEE quotient (saturating beyond the range), and
    the scale is fp16(fl32(fl32(c m) / 7))."""
    rng = np.random.default_rng(42 + i)
    c = np.float32(oracle.clip_ratio(i))
    for _ in range(50):
        n = 64
        w = (rng.standard_normal(n) * 0.02).astype(np.float16).astype(np.float32)
        s = np.exp(rng.standard_normal(n)).astype(np.float32)
        q, qs = oracle.fake_quant_group_clip(w, s, float(c), 0)
        ws = (w * s).astype(np.float32)
        m = np.float32(np.max(np.abs(ws)))
        assert qs == float(np.float16(np.float32(m * c) / np.float32(7)))
        for j in range(n):
            quot = np.float32(ws[j]) / np.float32(qs)
            assert q[j] == _nearest_level(quot)


def test_clip_search_never_worse_and_first_minimum():
    rng = np.random.default_rng(43)
    d_out, d_in, g, n_clip = 24, 256, 64, 10
    W = (rng.standard_normal((d_out, d_in)) * 0.02).astype(np.float16)
    W[3, 5] = np.float16(0.3)                     # a lone outlier in one group
    x = np.exp(rng.standard_normal(d_in)).astype(np.float32)
    s = np.exp(rng.standard_normal(d_in) * 0.5).astype(np.float32)
    idx, err = oracle.clip_search(W, x, s, g, n_clip)
    assert err[1] <= err[0]
    Wf = W.astype(np.float32)
    total0 = total1 = 0.0
    for r in range(d_out):
        for k in range(d_in // g):
            sl = slice(k * g, (k + 1) * g)
            e = [oracle.clip_group_error(Wf[r, sl], s[sl], x[sl], oracle.clip_ratio(i))
                 for i in range(n_clip)]
            b = int(np.argmin(e))                  # numpy argmin: first minimum
            assert idx[r, k] == b
            total0 += e[0]
            total1 += e[b]
    assert math.isclose(err[0], total0, rel_tol=1e-12)
    assert math.isclose(err[1], total1, rel_tol=1e-12)
    assert idx[3, 0] > 0                           # the outlier's group is clipped


def test_clip_search_one_ratio_is_the_weighted_error():
    rng = np.random.default_rng(44)
    W = (rng.standard_normal((16, 256)) * 0.02).astype(np.float16)
    x = np.exp(rng.standard_normal(256)).astype(np.float32)
    s = np.exp(rng.standard_normal(256) * 0.5).astype(np.float32)
    idx, err = oracle.clip_search(W, x, s, 128, 1)
    assert not idx.any()
    e = oracle.weighted_error(W, x, s, 128)
    assert err[0] == err[1]
    assert math.isclose(err[0], e, rel_tol=1e-12)


def test_clip_constant_magnitude_group_keeps_full_range():
    """|w s| equal across a group: the unclipped codes are all +-7 and any
    shrink saturates every weight below its value, so index 0 wins."""
    g = 32
    rng = np.random.default_rng(45)
    signs = np.where(rng.standard_normal((8, g)) > 0, 1.0, -1.0)
    W = (signs * 0.0123).astype(np.float16)
    x = np.ones(g, np.float32)
    idx, err = oracle.clip_search(W, x, None, g, 20)
    assert not idx.any()
    assert err[0] == err[1]


def test_clip_scaling_by_power_of_two():
    """Scaling W by 2 leaves every decision unchanged and multiplies the
    errors by 4 (every rounding step commutes with a power of two)."""
    rng = np.random.default_rng(46)
    W = (rng.standard_normal((16, 256)) * 0.02).astype(np.float16)
    x = np.exp(rng.standard_normal(256)).astype(np.float32)
    idx1, err1 = oracle.clip_search(W, x, None, 64, 10)
    idx2, err2 = oracle.clip_search((W.astype(np.float32) * 2).astype(np.float16), x, None, 64, 10)
    assert np.array_equal(idx1, idx2)
    assert np.allclose(err2, 4 * err1, rtol=1e-12)


def test_clip_pack_matches_clipped_groups():
    """The pack with clip indices stores the clipped group's codes and fp16
    scale; index 0 everywhere is the unclipped pack."""
    rng = np.random.default_rng(47)
    d_out, d_in, g = 16, 256, 64
    W = (rng.standard_normal((d_out, d_in)) * 0.02).astype(np.float16)
    s = np.exp(rng.standard_normal(d_in) * 0.5).astype(np.float32)
    idx = rng.integers(0, 10, size=(d_out, d_in // g)).astype(np.uint8)
    qw, sc, qz = oracle.quantize_pack(W, s, g, 8, idx)
    u = oracle.unpack(qw, d_out)
    Wf = W.astype(np.float32)
    for r in range(d_out):
        for k in range(d_in // g):
            sl = slice(k * g, (k + 1) * g)
            q, qs = oracle.fake_quant_group_clip(Wf[r, sl], s[sl], oracle.clip_ratio(idx[r, k]), 0)
            assert np.array_equal(u[r, sl].astype(np.int32), q.astype(np.int32) + 8)
            assert sc[k, r] == np.float16(qs)
    zero = np.zeros_like(idx)
    a = oracle.quantize_pack(W, s, g, 8, zero)
    b = oracle.quantize_pack(W, s, g, 8)
    for t1, t2 in zip(a, b):
        assert np.array_equal(t1.view(np.uint8), t2.view(np.uint8))


# ----------------------------------------------------- norm-group scales --
# "From-Scratch AWQ INT4 Quantization on Qwen3-8B", exporter steps 1-2: one
# shared scale per norm group, the geometric mean of the members' scales.

def test_geomean_closed_forms():
    rng = np.random.default_rng(51)
    a = np.exp(rng.standard_normal(1000)).astype(np.float32)
    b = np.exp(rng.standard_normal(1000)).astype(np.float32)
    assert np.array_equal(oracle.geomean_scales([a]), a)
    assert np.array_equal(oracle.geomean_scales([a, a]), a)          # sqrt(a^2) = a exactly
    # (a^3)^(1/3) is within ~1e-16 of the fp32 value a, far inside half an fp32 ulp
    assert np.array_equal(oracle.geomean_scales([a, a, a]), a)
    # two members: the correctly rounded sqrt of the exact product
    two = oracle.geomean_scales([a, b])
    exact = np.array([math.sqrt(float(x) * float(y)) for x, y in zip(a, b)])
    assert np.array_equal(two, exact.astype(np.float32))
    # powers of two pass through: 4 and 16 give 8; 2, 4, 8 give 4
    assert oracle.geomean_scales([np.float32([4.0]), np.float32([16.0])])[0] == 8.0
    assert oracle.geomean_scales([np.float32([2.0]), np.float32([4.0]),
                                  np.float32([8.0])])[0] == np.float32(4.0)


def test_geomean_bounds_and_homogeneity():
    rng = np.random.default_rng(52)
    ss = [np.exp(rng.standard_normal(500) * 2).astype(np.float32) for _ in range(3)]
    g = oracle.geomean_scales(ss).astype(np.float64)
    lo = np.minimum.reduce([x.astype(np.float64) for x in ss])
    hi = np.maximum.reduce([x.astype(np.float64) for x in ss])
    am = sum(x.astype(np.float64) for x in ss) / 3
    assert np.all(g >= lo * (1 - 1e-7)) and np.all(g <= hi * (1 + 1e-7))
    assert np.all(g <= am * (1 + 1e-7))                               # AM-GM
    g2 = oracle.geomean_scales([x * np.float32(8.0) for x in ss])     # scaling by 2^3
    assert np.array_equal(g2, (g * 8).astype(np.float32))


# ------------------------------------------------------------ duo scaling --
# "AWQ architecture, in depth", section "The scale search as code": with duo
# scaling the candidate is x^r / (w_mean^(1-r) + 1e-4), w_mean the mean over
# rows of |w| divided by its row's largest |w|; clamped at 1e-4, normalised.

def test_weight_mean_closed_forms():
    W = np.array([[1, 0.5, 0.25, 1], [2, 2, 1, 0.5]], np.float16)
    # rows divided by their maxima 1 and 2: [1, .5, .25, 1] and [1, 1, .5, .25]
    assert np.array_equal(oracle.weight_mean([W]), np.array([1, 0.75, 0.375, 0.625]))
    # split into two segments: the same rows, the same mean
    assert np.array_equal(oracle.weight_mean([W[:1], W[1:]]), np.array([1, 0.75, 0.375, 0.625]))
    # an all-zero row adds 0 to every channel and counts as a row
    Z = np.vstack([W, np.zeros((1, 4), np.float16)])
    assert np.array_equal(oracle.weight_mean([Z]), np.array([1, 0.75, 0.375, 0.625]) * 2 / 3)


def test_weight_mean_row_scaling_invariance():
    """Each row is divided by its own maximum, so scaling rows by powers of
    two leaves w_mean unchanged (and signs do not matter).  Scaling up only:
    that is exact in fp16 for every value, subnormals included."""
    rng = np.random.default_rng(71)
    W = (rng.standard_normal((32, 256)) * 0.02).astype(np.float16)
    f = (2.0 ** rng.integers(0, 4, size=(32, 1))) * np.where(rng.random((32, 1)) > 0.5, 1, -1)
    W2 = (W.astype(np.float32) * f).astype(np.float16)
    assert np.array_equal(oracle.weight_mean([W]), oracle.weight_mean([W2]))


def test_weight_mean_nonfinite_weights():
    """IEEE rules fix what a NaN or an infinity does: the row maximum skips a
    NaN (|w| >= 0, so it acts as a 0 there) and the NaN's own quotient is
    NaN; an infinite maximum makes every finite quotient of its row 0 and
    its own quotient inf / inf = NaN."""
    rng = np.random.default_rng(73)
    W = (rng.standard_normal((16, 64)) * 0.02).astype(np.float16)
    Wn = W.copy()
    Wn[3, 5] = np.nan
    Wz = W.copy()
    Wz[3, 5] = 0
    got, ref = oracle.weight_mean([Wn]), oracle.weight_mean([Wz])
    assert np.isnan(got[5]) and np.array_equal(np.delete(got, 5), np.delete(ref, 5))
    Wi = W.copy()
    Wi[7, 9] = np.inf
    Wr = np.delete(W, 7, axis=0)            # the inf row adds 0 to the finite channels
    got = oracle.weight_mean([Wi])
    ref = oracle.weight_mean([Wr]) * 15 / 16
    assert np.isnan(got[9])
    assert np.allclose(np.delete(got, 9), np.delete(ref, 9), rtol=1e-15, atol=0)


def test_duo_table_r0_closed_form_and_constant_weights():
    x = np.array([0.5, 2.0, 8.0, 1e-6], np.float32)
    wm = np.array([1, 0.75, 0.375, 0.625])
    S = oracle.scale_table_duo(x, wm, 20)
    s0 = [max(1.0 / (w + 1e-4), 1e-4) for w in wm]        # r = 0: x^0 = 1
    norm = math.sqrt(max(s0) * min(s0))
    assert np.array_equal(S[0], np.array([v / norm for v in s0]).astype(np.float32))
    # every |w| equal: w_mean = 1, the constant 1/(1 + 1e-4) cancels in the
    # normalisation, leaving the plain table (x well above the clamps)
    x2 = np.exp(np.random.default_rng(72).standard_normal(300)).astype(np.float32)
    Sd = oracle.scale_table_duo(x2, np.ones(300), 20)
    Sp = oracle.scale_table(x2, 20)
    ulp = np.abs(Sd.view(np.int32).astype(np.int64) - Sp.view(np.int32).astype(np.int64))
    assert ulp.max() <= 1


def test_duo_search_uses_duo_table():
    rng = np.random.default_rng(73)
    W = (rng.standard_normal((48, 256)) * 0.02).astype(np.float16)
    X = (rng.standard_normal((64, 256)) * np.exp(rng.standard_normal(256))).astype(np.float16)
    x = oracle.act_stats(X)
    err, best, s = oracle.scale_search([W], x, 128, 20, oracle.DUO)
    S = oracle.scale_table_duo(x, oracle.weight_mean([W]), 20)
    assert np.array_equal(s, S[best])
    for i in (0, best, 19):
        assert math.isclose(err[i], oracle.weighted_error(W, x, S[i], 128), rel_tol=1e-12)
    assert err[best] == err.min() and best == int(np.argmin(err))


# ------------------------------------------------------- asymmetric INT4 --
# "AWQ architecture, in depth": a 16-bit scale and a 4-bit zero point per
# group and output channel; the worked example in "The scale search as code"
# (values up to 0.5: step about 1/15 = 0.067, worst rounding error about
# 0.033).  Reading: min-max grid of 16 levels, zero = rint(-min / scale).

def _nearest_int_in(v, lo, hi):
    """Nearest integer in [lo, hi] to v, ties to even (by enumeration)."""
    v = float(v)
    return min(range(lo, hi + 1), key=lambda c: (abs(v - c), c % 2))


def test_asym_worked_example_step_and_error():
    w = np.linspace(-0.5, 0.5, 128).astype(np.float16).astype(np.float32)
    s = np.ones(128, np.float32)
    q, qs, z = oracle.fake_quant_group_asym(w, s)
    assert qs == float(np.float16(np.float32(1.0) / np.float32(15)))   # 0.06665...
    assert abs(qs - 1 / 15) < 1e-4
    err = np.abs(w.astype(np.float64) - (q.astype(np.float64) - z) * qs)
    inside = (q > 0) & (q < 15)
    assert np.all(err[inside] <= qs / 2 * (1 + 1e-6))
    # the page's "about 0.033": the fp16 step is a little under 1/15, so the
    # largest value lands just past the top level and clamps (0.0334)
    assert abs(err.max() - 1 / 30) < 1e-3


def test_asym_codes_zero_and_scale_bruteforce():
    rng = np.random.default_rng(81)
    for trial in range(200):
        n = 64
        w = (rng.standard_normal(n) * 0.02 + (0.01 if trial % 3 == 0 else 0.0)
             ).astype(np.float16).astype(np.float32)
        s = np.exp(rng.standard_normal(n)).astype(np.float32)
        q, qs, z = oracle.fake_quant_group_asym(w, s)
        ws = (w * s).astype(np.float32)
        rng_ = max(np.float32(ws.max() - ws.min()), np.float32(1e-5))
        assert qs == float(np.float16(np.float32(rng_) / np.float32(15)))
        assert z == _nearest_int_in(np.float32(-ws.min()) / np.float32(qs), 0, 15)
        for j in range(n):
            quot = np.float32(ws[j]) / np.float32(qs)
            assert q[j] == _nearest_int_in(float(quot) + z, 0, 15) or \
                abs(abs(float(quot) + z - q[j]) - 0.5) < 1e-6   # a tie in the shifted grid
            assert q[j] == min(15, max(0, int(np.rint(quot)) + z))


def test_asym_zero_group_and_nonfinite():
    q, qs, z = oracle.fake_quant_group_asym(np.zeros(32, np.float32), np.ones(32, np.float32))
    assert z == 0 and not q.any()
    assert qs == float(np.float16(np.float32(1e-5) / np.float32(15)))
    w = np.ones(32, np.float32)
    w[3] = np.inf
    q, qs, z = oracle.fake_quant_group_asym(w, np.ones(32, np.float32))
    assert np.isnan(qs) and z == 8 and (q == 8).all()


def test_asym_dequant_within_half_step():
    rng = np.random.default_rng(82)
    for _ in range(100):
        w = (rng.standard_normal(128) * 0.02).astype(np.float16).astype(np.float32)
        s = np.exp(rng.standard_normal(128)).astype(np.float32)
        q, qs, z = oracle.fake_quant_group_asym(w, s)
        ws = (w * s).astype(np.float64)
        err = np.abs(ws - (q.astype(np.float64) - z) * qs)
        inside = (q > 0) & (q < 15)
        assert np.all(err[inside] <= qs / 2 * (1 + 1e-6))


@pytest.mark.parametrize("g", [32, 128])
def test_asym_pack_roundtrip(g):
    """Codes and per-group zero points unpack exactly; the runtime dequant
    (u - zero) * scale equals the group dequant (q - zero) * q_scale."""
    rng = np.random.default_rng(83 + g)
    d_out, d_in = 24, 256
    W = (rng.standard_normal((d_out, d_in)) * 0.02).astype(np.float16)
    s = np.exp(rng.standard_normal(d_in) * 0.5).astype(np.float32)
    qw, sc, qz = oracle.quantize_pack(W, s, g, -1)
    u = oracle.unpack(qw, d_out)
    zz = oracle.unpack(qz, d_out)          # [d_out, G]: the zeros use the same packing
    Wf = W.astype(np.float32)
    for r in range(d_out):
        for k in range(d_in // g):
            sl = slice(k * g, (k + 1) * g)
            q, qs, z = oracle.fake_quant_group_asym(Wf[r, sl], s[sl])
            assert np.array_equal(u[r, sl], q) and zz[r, k] == z
            assert sc[k, r] == np.float16(qs)
            assert np.array_equal((u[r, sl].astype(np.float64) - zz[r, k]) * float(sc[k, r]),
                                  (q.astype(np.float64) - z) * qs)


def test_asym_search_alpha0_is_asym_rtn():
    rng = np.random.default_rng(84)
    W = (rng.standard_normal((32, 256)) * 0.02).astype(np.float16)
    X = (rng.standard_normal((64, 256)) * np.exp(rng.standard_normal(256))).astype(np.float16)
    x = oracle.act_stats(X)
    err, best, s = oracle.scale_search([W], x, 128, 20, oracle.ASYM)
    e0 = oracle.weighted_error(W, x, np.ones(256, np.float32), 128, oracle.ASYM)
    assert math.isclose(err[0], e0, rel_tol=1e-12)
    assert err[best] <= err[0]
    e_sym = oracle.weighted_error(W, x, np.ones(256, np.float32), 128)
    assert e0 != e_sym
