"""Clip search (per row and group, at a fixed scale) and the clipped pack on
the GPU against the CPU oracle.

Bars: clip indices bit-exact except where the two ratios' exact errors tie
within 1e-6 relative (the kernel sums each group's error in fp32); totals
within 1e-5 relative; the clipped pack bit-exact (codes, words, scales,
zeros) for the same indices.
"""
import numpy as np
import pytest
import torch

import oracle
from post_int4_weight_b200 import awq
from post_int4_weight_b200 import workloads as wl

pytestmark = pytest.mark.gpu

ERR_RTOL = 1e-5
TIE_RTOL = 1e-6


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "the gpu tests need a CUDA device"


def _gpu_clip(W, x, s, g, n_clip, flags=0):
    idx, err = awq.clip_search(W.cuda(), torch.from_numpy(x).cuda(),
                               None if s is None else torch.from_numpy(s).cuda(),
                               g, n_clip, flags)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), err.cpu().numpy()


def _check_indices(idx_g, idx_o, W, x, s, g, flags=0):
    Wf = W.numpy().astype(np.float32)
    bad = np.argwhere(idx_g != idx_o)
    for r, k in bad:
        sl = slice(k * g, (k + 1) * g)
        sk = np.ones(g, np.float32) if s is None else s[sl]
        e_g = oracle.clip_group_error(Wf[r, sl], sk, x[sl], oracle.clip_ratio(idx_g[r, k]), flags)
        e_o = oracle.clip_group_error(Wf[r, sl], sk, x[sl], oracle.clip_ratio(idx_o[r, k]), flags)
        assert abs(e_g - e_o) <= TIE_RTOL * e_o, (r, k, idx_g[r, k], idx_o[r, k], e_g, e_o)
    return len(bad)


@pytest.mark.parametrize("d_out,d_in,g,n_clip,flags", [
    (64, 512, 128, 10, 0), (72, 256, 64, 20, 0), (40, 128, 32, 10, 0),
    (1, 128, 128, 10, 0), (200, 1024, 128, 1, 0), (48, 256, 64, 10, awq.SCALE_FP32)])
def test_clip_parity_small(d_out, d_in, g, n_clip, flags):
    seed = d_out * 3 + d_in + g + n_clip
    W = wl.weight(d_out, d_in, seed)
    X = wl.activations(64, d_in, seed + 1)
    x = oracle.act_stats(X.numpy())
    s = oracle.scale_table(x, 20)[9]                  # a mid-grid scale vector
    idx_g, err_g = _gpu_clip(W, x, s, g, n_clip, flags)
    idx_o, err_o = oracle.clip_search(W.numpy(), x, s, g, n_clip, flags)
    _check_indices(idx_g, idx_o, W, x, s, g, flags)
    np.testing.assert_allclose(err_g, err_o, rtol=ERR_RTOL, atol=0)
    assert err_g[1] <= err_g[0] * (1 + 1e-6)
    if n_clip == 1:
        assert not idx_g.any()


def test_clip_without_scale_is_rtn_clip():
    W = wl.weight(32, 256, 5)
    x = np.abs(np.random.default_rng(5).standard_normal(256)).astype(np.float32) + 0.1
    idx_g, err_g = _gpu_clip(W, x, None, 128, 10)
    idx_o, err_o = oracle.clip_search(W.numpy(), x, None, 128, 10)
    _check_indices(idx_g, idx_o, W, x, None, 128)
    np.testing.assert_allclose(err_g, err_o, rtol=ERR_RTOL, atol=0)


def test_clip_q_proj_full_and_clipped_pack():
    """The 4096 x 4096 q_proj layer at the oracle's chosen scale: clip
    indices and totals against the oracle, then the clipped pack of the GPU's
    indices bit-exact against the oracle's pack of the same indices."""
    work = wl.WORKLOADS["q_proj_4096x4096"]
    (grp, Ws, X), = wl.group_inputs(work)
    W = Ws[0]
    x = oracle.act_stats(X.numpy())
    _, best, s = oracle.scale_search([W.numpy()], x, 128, 20)
    idx_g, err_g = _gpu_clip(W, x, s, 128, 10)
    idx_o, err_o = oracle.clip_search(W.numpy(), x, s, 128, 10)
    n_ties = _check_indices(idx_g, idx_o, W, x, s, 128)
    assert n_ties <= idx_g.size // 1000
    np.testing.assert_allclose(err_g, err_o, rtol=ERR_RTOL, atol=0)
    assert err_o[1] < err_o[0]
    assert (idx_o > 0).any()
    Wd = W.cuda()
    qw, sc, qz = awq.quantize_pack(Wd, torch.from_numpy(s).cuda(), 128, 8,
                                   clip_idx=torch.from_numpy(idx_g).cuda())
    torch.cuda.synchronize()
    qw_o, sc_o, qz_o = oracle.quantize_pack(W.numpy(), s, 128, 8, idx_g)
    assert np.array_equal(qw.cpu().numpy(), qw_o)
    assert np.array_equal(sc.cpu().numpy().view(np.uint16), sc_o.view(np.uint16))
    assert np.array_equal(qz.cpu().numpy(), qz_o)


@pytest.mark.parametrize("g", [32, 64, 128])
def test_clipped_pack_every_index(g):
    """Every clip index 0..19 on ragged shapes, pack bit-exact vs oracle."""
    d_out, d_in = 72, 4 * 128
    W = wl.weight(d_out, d_in, 77 + g)
    rng = np.random.default_rng(g)
    s = np.exp(rng.standard_normal(d_in) * 0.5).astype(np.float32)
    idx = (np.arange(d_out * (d_in // g)) % 20).astype(np.uint8).reshape(d_out, d_in // g)
    rng.shuffle(idx.reshape(-1))
    qw, sc, qz = awq.quantize_pack(W.cuda(), torch.from_numpy(s).cuda(), g, 8,
                                   clip_idx=torch.from_numpy(idx).cuda())
    torch.cuda.synchronize()
    qw_o, sc_o, qz_o = oracle.quantize_pack(W.numpy(), s, g, 8, idx)
    assert np.array_equal(qw.cpu().numpy(), qw_o)
    assert np.array_equal(sc.cpu().numpy().view(np.uint16), sc_o.view(np.uint16))
    assert np.array_equal(qz.cpu().numpy(), qz_o)


def test_clip_nonfinite_zero_and_deterministic():
    W = wl.weight(64, 256, 91)
    W[3, 7] = float("nan")
    W[10, 128:] = 0.0                                  # row 10, group 1: all zero
    x = np.exp(np.random.default_rng(9).standard_normal(256)).astype(np.float32)
    idx_a, err_a = _gpu_clip(W, x, None, 128, 10)
    idx_b, err_b = _gpu_clip(W, x, None, 128, 10)
    assert np.array_equal(idx_a, idx_b)
    assert np.isnan(err_a).all() and np.isnan(err_b).all()
    assert idx_a[3, 0] == 0 and idx_a[10, 1] == 0
    W[3, 7] = 0.5
    idx_c, err_c = _gpu_clip(W, x, None, 128, 10)
    idx_d, err_d = _gpu_clip(W, x, None, 128, 10)
    assert np.array_equal(idx_c, idx_d) and np.array_equal(err_c, err_d)
    idx_o, err_o = oracle.clip_search(W.numpy(), x, None, 128, 10)
    _check_indices(idx_c, idx_o, W, x, None, 128)
    np.testing.assert_allclose(err_c, err_o, rtol=ERR_RTOL, atol=0)


# ------------------------------------------------------------ output space --
# awq_clip_search_output: each (row, group) and ratio scored by the group's
# share of the output error, against oracle.clip_search_output.  The GPU
# evaluates the scores as fp32 quadratic forms of fp64 Gram matrices, so an
# index may differ only where the oracle's two scores tie within 1e-5.

OUT_TIE_RTOL = 1e-5


def _out_score(X, w, s, g_cols, c):
    q, qs = oracle.fake_quant_group_clip(w[g_cols], s[g_cols], c)
    dw = w[g_cols].astype(np.float64) - q.astype(np.float64) * qs / s[g_cols].astype(np.float64)
    y = X[:, g_cols].astype(np.float64) @ dw
    return float(y @ y)


def _check_clip_output(X, W, s, g, n_clip, idx_g, err_g):
    idx_o, err_o = oracle.clip_search_output(X, W, s, g, n_clip)
    np.testing.assert_allclose(err_g, err_o, rtol=ERR_RTOL, atol=0)
    diff = np.argwhere(idx_g != idx_o)
    assert len(diff) <= max(2, idx_o.size // 1000)
    for r, k in diff:
        cols = slice(k * g, (k + 1) * g)
        w = W[r].astype(np.float32)
        sv = np.ones(W.shape[1], np.float32) if s is None else s
        a = _out_score(X, w, sv, cols, oracle.clip_ratio(int(idx_g[r, k])))
        b = _out_score(X, w, sv, cols, oracle.clip_ratio(int(idx_o[r, k])))
        assert abs(a - b) <= OUT_TIE_RTOL * b, (r, k, idx_g[r, k], idx_o[r, k], a, b)


@pytest.mark.parametrize("d_out,d_in,T,g,n_clip", [(64, 256, 64, 32, 10), (200, 512, 96, 64, 20),
                                                   (72, 384, 128, 128, 10), (8, 128, 1, 128, 3),
                                                   # Gram over 4 token slices, the last one
                                                   # ragged (232 and 124 tokens)
                                                   (96, 512, 1000, 64, 10),
                                                   (136, 256, 700, 128, 10)])
def test_clip_output_parity_small(d_out, d_in, T, g, n_clip):
    seed = d_out + d_in + T + g
    W = wl.weight(d_out, d_in, seed + 1)
    W[min(3, d_out - 1), 17] = 0.3           # an outlier whose group wants clipping
    X = wl.activations(T, d_in, seed)
    s = np.exp(np.random.default_rng(seed).standard_normal(d_in) * 0.5).astype(np.float32)
    idx, err = awq.clip_search_output(X.cuda(), W.cuda(), torch.from_numpy(s).cuda(), g, n_clip)
    torch.cuda.synchronize()
    _check_clip_output(X.numpy(), W.numpy(), s, g, n_clip, idx.cpu().numpy(), err.cpu().numpy())
    # without s: the scale is 1
    idx1, err1 = awq.clip_search_output(X.cuda(), W.cuda(), None, g, n_clip)
    torch.cuda.synchronize()
    _check_clip_output(X.numpy(), W.numpy(), None, g, n_clip, idx1.cpu().numpy(),
                       err1.cpu().numpy())


def test_clip_output_q_proj_rows_and_pack():
    """The full q_proj 4096 x 4096 layer with 4096 tokens at its searched
    scale: the first 64 rows' indices against the oracle on those rows
    (a row's indices depend only on its own weights and X), the slice's
    totals from a run on the slice, and the clipped pack of the full layer
    against the oracle's pack at the GPU's indices."""
    work = wl.WORKLOADS["q_proj_4096x4096"]
    (grp, Ws, X), = wl.group_inputs(work)
    W = Ws[0]
    dev = torch.device("cuda")
    Xd, Wd = X.to(dev), W.to(dev)
    x = awq.act_stats(Xd)
    _, best, s = awq.scale_search([Wd], x, 128, 20)
    idx, err = awq.clip_search_output(Xd, Wd, s, 128, 10)
    torch.cuda.synchronize()
    s_np = s.cpu().numpy()
    idx_np = idx.cpu().numpy()
    rows = 64
    idx_s, err_s = awq.clip_search_output(Xd, Wd[:rows].contiguous(), s, 128, 10)
    torch.cuda.synchronize()
    assert np.array_equal(idx_s.cpu().numpy(), idx_np[:rows])
    _check_clip_output(X.numpy(), W[:rows].numpy(), s_np, 128, 10, idx_np[:rows],
                       err_s.cpu().numpy())
    assert idx_np.max() > 0 and err.cpu().numpy()[1] <= err.cpu().numpy()[0]
    qw, sc, qz = awq.quantize_pack(Wd, s, 128, 8, clip_idx=idx)
    torch.cuda.synchronize()
    qw_o, sc_o, qz_o = oracle.quantize_pack(W.numpy(), s_np, 128, 8, idx_np)
    assert np.array_equal(qw.cpu().numpy(), qw_o)
    assert np.array_equal(sc.cpu().numpy().view(np.uint16), sc_o.view(np.uint16))


def test_clip_output_nonfinite_and_deterministic():
    W = wl.weight(64, 256, 91)
    X = wl.activations(32, 256, 92)
    a = awq.clip_search_output(X.cuda(), W.cuda(), None, 64, 10)
    b = awq.clip_search_output(X.cuda(), W.cuda(), None, 64, 10)
    torch.cuda.synchronize()
    assert np.array_equal(a[0].cpu().numpy(), b[0].cpu().numpy())
    assert np.array_equal(a[1].cpu().numpy(), b[1].cpu().numpy())
    W[5, 70] = float("nan")
    awq.last_device_flags(clear=True)
    idx, err = awq.clip_search_output(X.cuda(), W.cuda(), None, 64, 10)
    torch.cuda.synchronize()
    assert np.isnan(err.cpu().numpy()).all()
    assert int(idx.cpu().numpy()[5, 1]) == 0
    assert awq.last_device_flags() == (6, awq.FLAG_NONFINITE_SCORE)
