"""Duo scaling (AWQ_DUO_SCALING) on the GPU against the CPU oracle.

The weight mean is an fp64 sum whose order differs between the two sides
(rows in order on the CPU; row blocks, then the blocks' sums in a fixed
order on the GPU), so
an fp32 entry of the scale table may differ by one ulp when it lies within
~1e-16 of a rounding boundary; the chosen scale is compared bit for bit
except for such entries, and the pack is compared bit for bit at the GPU's
scale.  Bars otherwise as in the plain search: errors within 1e-5, index
exact or tied within 1e-6.
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


def _duo_case(Ws, X, g=128, n_grid=20):
    dev = torch.device("cuda")
    x_g = awq.act_stats(X.to(dev))
    err, best, s = awq.scale_search([W.to(dev) for W in Ws], x_g, g, n_grid, awq.DUO_SCALING)
    torch.cuda.synchronize()
    x = oracle.act_stats(X.numpy())
    assert np.array_equal(x_g.cpu().numpy(), x)
    err_o, best_o, s_o = oracle.scale_search([W.numpy() for W in Ws], x, g, n_grid, oracle.DUO)
    err, b, s = err.cpu().numpy(), int(best.cpu()[0]), s.cpu().numpy()
    np.testing.assert_allclose(err, err_o, rtol=ERR_RTOL, atol=0)
    if b != best_o:
        assert abs(err_o[b] - err_o[best_o]) <= TIE_RTOL * err_o[best_o]
        s_o = oracle.scale_table_duo(x, oracle.weight_mean([W.numpy() for W in Ws]), n_grid)[b]
    ulp = np.abs(s.view(np.int32).astype(np.int64) - s_o.view(np.int32).astype(np.int64))
    assert ulp.max() <= 1 and (ulp > 0).sum() <= max(1, s.size // 1000)
    return s


@pytest.mark.parametrize("shape", [((256,), 512, 64), ((200, 72, 8), 1024, 96),
                                   ((4096,), 4096, 256),
                                   # wider rows: 2, 3 and 4 chunks of 8 per thread of
                                   # the weight-mean pass; 600 rows give its CTAs
                                   # several batches, 40-64 rows leave most CTAs idle
                                   ((600,), 8192, 32), ((48, 16), 12288, 32),
                                   ((40,), 16384, 32)])
def test_duo_search_parity(shape):
    d_outs, d_in, T = shape
    seed = sum(d_outs) + d_in
    Ws = [wl.weight(d, d_in, seed + m + 1) for m, d in enumerate(d_outs)]
    X = wl.activations(T, d_in, seed)
    s = _duo_case(Ws, X)
    for W in Ws[:1]:
        qw, sc, qz = awq.quantize_pack(W.cuda(), torch.from_numpy(s).cuda(), 128, 8)
        torch.cuda.synchronize()
        qw_o, sc_o, qz_o = oracle.quantize_pack(W.numpy(), s, 128, 8)
        assert np.array_equal(qw.cpu().numpy(), qw_o)
        assert np.array_equal(sc.cpu().numpy().view(np.uint16), sc_o.view(np.uint16))


@pytest.mark.parametrize("n_grid", [1, 32])
def test_duo_grid_sizes(n_grid):
    """One grid point (r = 0: the candidate is 1 / (w_mean + 1e-4)) and the
    largest grid, whose alphas the candidates kernel's warps take in four
    rounds."""
    W = wl.weight(96, 512, 41 + n_grid)
    X = wl.activations(48, 512, 42 + n_grid)
    s = _duo_case([W], X, 128, n_grid)
    if n_grid == 1:
        assert np.all(np.isfinite(s)) and np.all(s > 0)


def test_duo_qwen3_gate_up_group():
    """The Qwen3-8B gate/up group (2 x 12288 rows x 4096) with duo scaling."""
    work = wl.WORKLOADS["qwen3_8b_stack36"]
    grp, Ws, X = wl.group_inputs(work, 0)[2]
    _duo_case(Ws, X)


def test_duo_zero_rows_and_columns():
    W = wl.weight(64, 256, 5)
    W[7] = 0.0                      # an all-zero row counts but adds nothing
    W[:, 130] = 0.0                 # an all-zero column: w_mean = 0
    X = wl.activations(32, 256, 6)
    X[:, 3] = 0.0                   # x = 0: x^r = 0 for r > 0, clamped at 1e-4
    _duo_case([W], X)


def test_duo_rejects_wide_inputs_and_small_workspace():
    W = torch.zeros(8, 32768, dtype=torch.float16, device="cuda")
    x = torch.ones(32768, dtype=torch.float32, device="cuda")
    ws = awq.workspace(awq.OP_SCALE_SEARCH, "cuda", 1, 8, 32768, 128, 20)
    with pytest.raises(awq.AwqError):
        awq.scale_search([W], x, 128, 20, awq.DUO_SCALING, ws=ws)
    W2 = torch.zeros(8, 1024, dtype=torch.float16, device="cuda")
    x2 = torch.ones(1024, dtype=torch.float32, device="cuda")
    small = awq.workspace(awq.OP_SCALE_SEARCH, "cuda", 1, 8, 1024, 128, 20)
    with pytest.raises(awq.AwqError):
        awq.scale_search([W2], x2, 128, 20, awq.DUO_SCALING, ws=small)


def test_duo_subnormal_rows():
    """Rows whose largest |w| is an fp16 subnormal, a row of subnormals and
    zeros, and a row mixing subnormal and normal magnitudes."""
    W = wl.weight(64, 256, 7)
    W[5] = W[5] * 1e-3              # largest |w| below 2^-14
    W[6] = W[6] * 1e-4              # deep subnormals, some rounded to 0
    W[9, ::3] = W[9, ::3] * 1e-3    # mixed within one row
    assert float(W[5].abs().max()) < 6.1035e-05
    X = wl.activations(32, 256, 8)
    _duo_case([W], X)


def test_duo_nonfinite_weight_reports_minus_one():
    """A NaN and an inf weight: the weighted errors are not finite on either
    side, so both report index -1 and the GPU a NaN scale vector."""
    W = wl.weight(64, 256, 9)
    W[3, 17] = float("nan")
    W[10, 40] = float("inf")
    X = wl.activations(16, 256, 10)
    x_g = awq.act_stats(X.cuda())
    err, best, s = awq.scale_search([W.cuda()], x_g, 128, 20, awq.DUO_SCALING)
    torch.cuda.synchronize()
    x = oracle.act_stats(X.numpy())
    err_o, best_o, _ = oracle.scale_search([W.numpy()], x, 128, 20, oracle.DUO)
    assert best_o == -1 and int(best.cpu()[0]) == -1
    assert np.all(np.isnan(s.cpu().numpy()))
    assert np.array_equal(np.isfinite(err.cpu().numpy()), np.isfinite(err_o))
