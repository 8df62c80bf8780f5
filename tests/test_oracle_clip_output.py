"""Pins of the oracle's output-space clip search.

The pages name the clip search ("AWQ architecture, in depth", section "The
pipeline end to end", step 5) without a formula and score candidates on the
output ("The scale search as code").  The reading pinned here: ratios
c_i = RN((20 - i) / 20), the group's range c_i * max|w s| (fp32), q_scale =
fp16(range / 7), codes saturating at +-7, and each (row, group) scored by
sum_t (X[t, group] . (w - w_hat))^2 -- the group's share of the output
error -- first minimum per (row, group).

Expected values come from numpy brute force (every code the nearest allowed
level, found by trying them all) and from the special case X = diag(c),
where the score is the weight-space clip score with x = c.
"""
import numpy as np
import pytest

import oracle

F32 = np.float32


def _nearest_codes(v):
    """Nearest of -7..7 to each fp32 quotient, ties to the even level."""
    v = np.asarray(v, np.float64)[..., None]
    lv = np.arange(-7, 8, dtype=np.float64)
    dist = np.abs(v - lv)
    cand = dist == dist.min(axis=-1, keepdims=True)
    even = cand & (np.arange(-7, 8) % 2 == 0)
    pick = np.where(even.any(axis=-1, keepdims=True), even, cand)
    return lv[pick.argmax(axis=-1)]


def _clipped_dw(w, s, c):
    """w - w_hat (fp64) for one group at clip ratio c (fp32 arithmetic for
    the decisions, as the method states)."""
    ws = (w * s).astype(F32)
    m = F32(F32(np.abs(ws).max()) * F32(c))
    qs = F32(np.float16(F32(m / F32(7.0))))
    if np.isinf(qs):
        qs = F32(65504.0)
    q = np.zeros_like(ws, dtype=np.float64) if qs == 0 else _nearest_codes((ws / qs).astype(F32))
    return w.astype(np.float64) - q * np.float64(qs) / s.astype(np.float64)


def _bruteforce(X, W, s, g, n_clip):
    d_out, d_in = W.shape
    G = d_in // g
    Xd = X.astype(np.float64)
    ratios = [F32((20 - i) / 20) for i in range(n_clip)]
    idx = np.zeros((d_out, G), np.uint8)
    tot0 = tot1 = 0.0
    for r in range(d_out):
        for k in range(G):
            cols = slice(k * g, (k + 1) * g)
            w = W[r, cols].astype(F32)
            e = []
            for c in ratios:
                y = Xd[:, cols] @ _clipped_dw(w, s[cols], c)
                e.append(float(y @ y))
            b = 0
            for i, v in enumerate(e):
                if v < e[b]:
                    b = i
            idx[r, k] = b
            tot0 += e[0]
            tot1 += e[b]
    return idx, np.array([tot0, tot1])


@pytest.mark.parametrize("g,n_clip", [(32, 10), (64, 20), (128, 5)])
def test_clip_output_bruteforce(g, n_clip):
    rng = np.random.default_rng(g + n_clip)
    T, d_out, d_in = 24, 6, 256
    W = (rng.standard_normal((d_out, d_in)) * 0.02).astype(np.float16)
    W[2, 7] = np.float16(0.3)          # a lone outlier, whose group wants clipping
    X = (rng.standard_normal((T, d_in)) * np.exp(rng.standard_normal(d_in))).astype(np.float16)
    s = np.exp(rng.standard_normal(d_in) * 0.5).astype(F32)
    idx, err = oracle.clip_search_output(X, W, s, g, n_clip)
    ridx, rerr = _bruteforce(X, W, s, g, n_clip)
    assert np.array_equal(idx, ridx)
    np.testing.assert_allclose(err, rerr, rtol=1e-12, atol=0)
    assert err[1] <= err[0]
    assert idx.max() > 0                # some group does clip


def test_clip_output_diagonal_x_is_weight_space():
    """X = diag(c): each group's output-space score is the weight-space
    score with x = c, so indices and totals equal the weight-space search."""
    rng = np.random.default_rng(5)
    d_out, d_in, g = 8, 128, 32
    W = (rng.standard_normal((d_out, d_in)) * 0.02).astype(np.float16)
    W[1, 40] = np.float16(0.25)
    c = np.exp(rng.standard_normal(d_in)).astype(np.float16)
    X = np.diag(c.astype(np.float32)).astype(np.float16)
    s = np.exp(rng.standard_normal(d_in) * 0.3).astype(F32)
    io, eo = oracle.clip_search_output(X, W, s, g, 10)
    iw, ew = oracle.clip_search(W, c.astype(F32), s, g, 10)
    assert np.array_equal(io, iw)
    np.testing.assert_allclose(eo, ew, rtol=1e-12, atol=0)


def test_clip_output_scaling_and_ratio_one():
    rng = np.random.default_rng(9)
    T, d_out, d_in, g = 16, 4, 64, 32
    W = (rng.standard_normal((d_out, d_in)) * 0.02).astype(np.float16)
    X = rng.standard_normal((T, d_in)).astype(np.float16)
    i1, e1 = oracle.clip_search_output(X, W, None, g, 10)
    X2 = (2 * X.astype(np.float32)).astype(np.float16)
    i2, e2 = oracle.clip_search_output(X2, W, None, g, 10)
    assert np.array_equal(i1, i2)
    np.testing.assert_allclose(e2, 4 * e1, rtol=1e-12)
    # one ratio: nothing to choose, and the total is the unclipped score
    i3, e3 = oracle.clip_search_output(X, W, None, g, 1)
    assert not i3.any() and e3[0] == e3[1] == e1[0]
