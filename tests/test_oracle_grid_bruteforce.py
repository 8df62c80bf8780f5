"""Brute-force pins of the oracle's whole alpha grid on tiny layers.

"From-Scratch AWQ INT4 Quantization on Qwen3-8B", section "AWQ scaling";
"AWQ architecture, in depth", section "The scale search as code";
"Weight-Only Quantization: GPTQ and AWQ", section 4 "Tiny example".

Every error of every grid point is recomputed here in plain numpy, with
none of the oracle's functions: the candidate scales from Python's fp64
``pow``, each group's scale from the fp32 maximum, every code as the nearest
of the allowed integer levels found by trying them all (ties to the even
level), and the activation-weighted squared error in fp64.  The layers have
several rows, several groups and several segments, and x varies per channel,
so a scale or an activation taken from the wrong channel, group or segment
changes the errors.  The grid search of the oracle (plain, asymmetric, duo,
fp32 scales) must reproduce every error within 1e-12 relative, its first
minimum and its scale vector bit for bit.
"""
import math

import numpy as np
import pytest

import oracle

F32 = np.float32


# --------------------------------------------------- independent restatement

def _alphas(n_grid):
    return [i / n_grid for i in range(n_grid)]


def _table_plain(x, n_grid):
    """s_i[j] = max(x_j, 1e-4)^alpha_i / sqrt(max_j * min_j), fp64 -> fp32."""
    xc = [float(max(F32(v), F32(1e-4))) for v in x]
    rows = []
    for a in _alphas(n_grid):
        sd = [math.pow(v, a) for v in xc]
        norm = math.sqrt(max(sd) * min(sd))
        rows.append([F32(v / norm) for v in sd])
    return np.array(rows, F32)


def _table_duo(x, Ws, n_grid):
    """Duo candidates: x^r / (w_mean^(1-r) + 1e-4), clamped below at 1e-4,
    normalised; w_mean = mean over all rows of |w| / (row's max |w|)."""
    d_in = len(x)
    acc = [0.0] * d_in
    rows = 0
    for W in Ws:
        for row in W.astype(np.float64):
            mx = max(abs(v) for v in row)
            for j in range(d_in):
                acc[j] += abs(row[j]) / mx if mx > 0 else 0.0
            rows += 1
    wm = [v / rows for v in acc]
    out = []
    for r in _alphas(n_grid):
        sd = [max(math.pow(float(x[j]), r) / (math.pow(wm[j], 1.0 - r) + 1e-4), 1e-4)
              for j in range(d_in)]
        norm = math.sqrt(max(sd) * min(sd))
        out.append([F32(v / norm) for v in sd])
    return np.array(out, F32)


def _nearest(v, levels):
    """Index into `levels` (ascending integers) of the level nearest to each
    fp32 value in v; a value halfway between two levels takes the even one."""
    v = np.asarray(v, np.float64)[..., None]
    lv = np.asarray(levels, np.float64)
    dist = np.abs(v - lv)                       # exact: fp32 minus a small integer
    best = dist.min(axis=-1, keepdims=True)
    cand = dist == best
    even = cand & (np.asarray(levels) % 2 == 0)
    pick = np.where(even.any(axis=-1, keepdims=True), even, cand)
    return pick.argmax(axis=-1)


def _fp16_scale(v, fp32_scale):
    v = F32(v)
    if fp32_scale:
        return v
    h = np.float16(v)
    return F32(65504.0) if np.isinf(h) else F32(h)


def _group_dequant(w, s, asym, fp32_scale):
    """w, s: fp32 [rows, g].  Returns the dequantised w_hat in fp64 (the
    level times the group scale over s, evaluated in fp64)."""
    ws = (w * s).astype(F32)                    # fp32 products
    rows, g = ws.shape
    what = np.zeros((rows, g), np.float64)
    for r in range(rows):
        if asym:
            mx, mn = ws[r].max(), ws[r].min()
            rng = max(F32(mx - mn), F32(1e-5))
            qs = _fp16_scale(F32(rng / F32(15.0)), fp32_scale)
            z = int(_nearest([F32(-mn / qs)], range(0, 16))[0])
            levels = list(range(-z, 16 - z))
            m = np.array(levels)[_nearest((ws[r] / qs).astype(F32), levels)]
        else:
            qs = _fp16_scale(F32(np.abs(ws[r]).max() / F32(7.0)), fp32_scale)
            if qs == 0:
                m = np.zeros(g)
            else:
                levels = list(range(-7, 8))
                m = np.array(levels)[_nearest((ws[r] / qs).astype(F32), levels)]
        what[r] = m.astype(np.float64) * np.float64(qs) / s[r].astype(np.float64)
    return what


def _grid_errors(Ws, x, S, g, asym=False, fp32_scale=False):
    x64 = np.asarray(x, np.float64)
    errs = []
    for s in S:
        e = 0.0
        for W in Ws:
            w = W.astype(F32)
            for k in range(W.shape[1] // g):
                cols = slice(k * g, (k + 1) * g)
                sk = np.broadcast_to(s[cols], (W.shape[0], g))
                what = _group_dequant(w[:, cols], sk, asym, fp32_scale)
                d = (w[:, cols].astype(np.float64) - what) * x64[cols]
                e += float((d * d).sum())
        errs.append(e)
    return np.array(errs)


def _first_min(errs):
    b = 0
    for i, e in enumerate(errs):
        if e < errs[b]:
            b = i
    return b


# ----------------------------------------------------------------- inputs --

def _layer(seed, rows, d_in, outlier=(5, 40.0)):
    rng = np.random.default_rng(seed)
    Ws = [(rng.standard_normal((r, d_in)) * 0.02).astype(np.float16) for r in rows]
    x = np.exp(rng.standard_normal(d_in)).astype(F32)
    x[outlier[0]] *= F32(outlier[1])
    x[d_in - 3] = F32(3e-5)                     # below the 1e-4 clamp
    return Ws, x


CASES = [
    # (seed, segment rows, d_in, group size, n_grid)
    (1, (16,), 96, 32, 20),
    (2, (16, 8), 96, 32, 20),
    (3, (8, 8, 24), 128, 64, 20),
    (4, (12,), 256, 128, 7),
]


@pytest.mark.parametrize("asym", [False, True], ids=["sym", "asym"])
@pytest.mark.parametrize("fp32_scale", [False, True], ids=["fp16scale", "fp32scale"])
@pytest.mark.parametrize("case", CASES, ids=lambda c: f"seed{c[0]}")
def test_plain_grid_bruteforce(case, asym, fp32_scale):
    seed, rows, d_in, g, n_grid = case
    Ws, x = _layer(seed, rows, d_in)
    S = _table_plain(x, n_grid)
    flags = (oracle.ASYM if asym else 0) | (oracle.SCALE_FP32 if fp32_scale else 0)
    err, best, s_best = oracle.scale_search(Ws, x, g, n_grid, flags)
    ref = _grid_errors(Ws, x, S, g, asym, fp32_scale)
    np.testing.assert_allclose(err, ref, rtol=1e-12, atol=0)
    assert best == _first_min(ref)
    assert np.array_equal(s_best.view(np.uint32), S[best].view(np.uint32))
    # the table itself, bit for bit
    assert np.array_equal(oracle.scale_table(x, n_grid).view(np.uint32), S.view(np.uint32))


@pytest.mark.parametrize("asym", [False, True], ids=["sym", "asym"])
@pytest.mark.parametrize("case", CASES[:3], ids=lambda c: f"seed{c[0]}")
def test_duo_grid_bruteforce(case, asym):
    seed, rows, d_in, g, n_grid = case
    Ws, x = _layer(seed + 10, rows, d_in)
    S = _table_duo(x, Ws, n_grid)
    flags = oracle.DUO | (oracle.ASYM if asym else 0)
    err, best, s_best = oracle.scale_search(Ws, x, g, n_grid, flags)
    ref = _grid_errors(Ws, x, S, g, asym)
    np.testing.assert_allclose(err, ref, rtol=1e-12, atol=0)
    assert best == _first_min(ref)
    assert np.array_equal(s_best.view(np.uint32), S[best].view(np.uint32))


def test_grid_errors_move_with_the_group_index():
    """The layers above distinguish groups: permuting the groups of W while
    keeping x and s in place changes the errors (so a scale or activation
    read from the wrong group would not go unnoticed)."""
    Ws, x = _layer(2, (16, 8), 96)
    S = _table_plain(x, 20)
    a = _grid_errors(Ws, x, S, 32)
    Wp = [np.concatenate([W[:, 32:64], W[:, :32], W[:, 64:]], axis=1) for W in Ws]
    b = _grid_errors(Wp, x, S, 32)
    assert np.max(np.abs(a - b) / a) > 1e-3


# ---------------------------------------------------------- worked example --
# "Weight-Only Quantization: GPTQ and AWQ", section 4: w = [0.5, -0.3, 0.8,
# 0.1], x = [10, 0.1, 0.1, 0.1], one group of four weights.

@pytest.mark.parametrize("fp32_scale", [False, True], ids=["fp16scale", "fp32scale"])
def test_worked_example_grid(fp32_scale):
    W = np.array([[0.5, -0.3, 0.8, 0.1]], np.float16)
    x = np.array([10, 0.1, 0.1, 0.1], F32)
    S = _table_plain(x, 20)
    ref = _grid_errors([W], x, S, 4, fp32_scale=fp32_scale)
    err, best, _ = oracle.scale_search([W], x, 4, 20, oracle.SCALE_FP32 if fp32_scale else 0)
    np.testing.assert_allclose(err, ref, rtol=1e-12, atol=0)
    # the first minimum is grid point 3 (alpha = 0.15) in both scale modes
    assert best == 3 == _first_min(ref)
    # from alpha = 0.7 on the salient channel's product dominates the group:
    # the other three codes are 0 and channel 0 is reproduced up to the
    # rounding of its scale, so the error is that of dropping channels 1..3
    dropped = sum((float(W[0, j]) * float(x[j])) ** 2 for j in (1, 2, 3))
    plateau = err[14:20]
    if fp32_scale:
        np.testing.assert_allclose(plateau, dropped, rtol=1e-6)
        assert np.ptp(plateau) <= 1e-9 * dropped
    else:
        np.testing.assert_allclose(plateau, dropped, rtol=1e-3)
    assert err[13] < dropped / 1.4            # alpha = 0.65 still keeps a code


# ------------------------------------------------------------ output space --
# "AWQ architecture, in depth", section "The scale search as code" (the
# group's output after fake quantisation against the full-precision output);
# "Weight-Only Quantization: GPTQ and AWQ", section 2 (the output error is
# X (W - W_hat)).  err[i] = ||X (W - W_hat_i)^T||_F^2, recomputed here as a
# plain fp64 matrix product from the brute-force W_hat_i above.

@pytest.mark.parametrize("asym", [False, True], ids=["sym", "asym"])
@pytest.mark.parametrize("fp32_scale", [False, True], ids=["fp16scale", "fp32scale"])
def test_output_error_grid_bruteforce(asym, fp32_scale):
    rng = np.random.default_rng(77)
    T, d_out, d_in, g, n_grid = 12, 8, 96, 32, 20
    W = (rng.standard_normal((d_out, d_in)) * 0.02).astype(np.float16)
    X = (rng.standard_normal((T, d_in)) * np.exp(rng.standard_normal(d_in))).astype(np.float16)
    x = np.abs(X.astype(np.float64)).mean(axis=0).astype(F32)
    S = _table_plain(x, n_grid)
    Xd = X.astype(np.float64)
    ref = []
    for s in S:
        w = W.astype(F32)
        what = np.concatenate(
            [_group_dequant(w[:, k * g:(k + 1) * g], np.broadcast_to(s[k * g:(k + 1) * g], (d_out, g)),
                            asym, fp32_scale) for k in range(d_in // g)], axis=1)
        y = Xd @ (W.astype(np.float64) - what).T
        ref.append(float((y * y).sum()))
    flags = (oracle.ASYM if asym else 0) | (oracle.SCALE_FP32 if fp32_scale else 0)
    err = oracle.output_error(X, W, x, g, n_grid, flags)
    np.testing.assert_allclose(err, ref, rtol=1e-12, atol=0)


def test_output_error_asym_diagonal_x_is_weight_space():
    """X = diag(c): the asymmetric output-space score equals the asymmetric
    weight-space score with x = c."""
    rng = np.random.default_rng(43)
    d_out, d_in, g = 16, 64, 32
    W = (rng.standard_normal((d_out, d_in)) * 0.02).astype(np.float16)
    c = np.exp(rng.standard_normal(d_in)).astype(np.float16)
    X = np.diag(c.astype(np.float32)).astype(np.float16)
    x = c.astype(F32)
    eo = oracle.output_error(X, W, x, g, 20, oracle.ASYM)
    ew, _, _ = oracle.scale_search([W], x, g, 20, oracle.ASYM)
    np.testing.assert_allclose(eo, ew, rtol=1e-12)
