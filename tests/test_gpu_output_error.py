"""Output-space scoring (tcgen05 GEMM path) against the CPU oracle.

err[i] = ||X (W - W_hat_i)^T||^2.  The oracle evaluates it in fp64 from the
exact W - W_hat_i; the GPU splits the row-scaled W - W_hat_i into two fp16
parts and accumulates X dW^T in fp32 on the tensor cores, so the bar is the
error-sum tolerance, 1e-5 relative, and the chosen index must agree (or tie
within 1e-6).  The returned s_best is the scale-table row of the chosen
index, bit-exact.
"""
import numpy as np
import pytest
import torch

import oracle
from post_int4_weight_b200 import awq
from post_int4_weight_b200 import workloads as wl

pytestmark = pytest.mark.gpu

ERR_RTOL = 1e-5


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "the gpu tests need a CUDA device"


def _run(X, W, x_np, g, n_grid=20, flags=0):
    err, best, s_best = awq.output_error(X.cuda(), W.cuda(), torch.from_numpy(x_np).cuda(),
                                         g, n_grid, flags)
    torch.cuda.synchronize()
    b = int(best.cpu()[0])
    s_best = s_best.cpu().numpy()
    if b >= 0:
        S = oracle.scale_table(x_np, n_grid)
        np.testing.assert_array_equal(s_best.view(np.uint32), S[b].view(np.uint32))
    else:
        assert np.isnan(s_best).all()
    return err.cpu().numpy(), b


def _check(err_g, best_g, err_o):
    np.testing.assert_allclose(err_g, err_o, rtol=ERR_RTOL, atol=0)
    best_o = int(np.argmin(err_o))
    if best_g != best_o:
        assert abs(err_o[best_g] - err_o[best_o]) <= 1e-6 * err_o[best_o]


@pytest.mark.parametrize("T,d_out,d_in,g", [(64, 256, 512, 128), (100, 264, 640, 64),
                                            (256, 512, 1024, 32), (1, 8, 64, 32)])
def test_output_error_small_exact(T, d_out, d_in, g):
    seed = T + d_out + d_in + g
    W = wl.weight(d_out, d_in, seed + 1)
    X = wl.activations(T, d_in, seed)
    x = oracle.act_stats(X.numpy())
    err_g, best_g = _run(X, W, x, g)
    err_o = oracle.output_error(X.numpy(), W.numpy(), x, g, 20)
    _check(err_g, best_g, err_o)


def test_output_error_diagonal_x_full_down_proj():
    """X = diag(c) (T = d_in = 12288): the output error reduces to the
    weight-space score with x = c, which the oracle computes exactly, at the
    full down_proj shape 4096 x 12288."""
    d_out, d_in = 4096, 12288
    W = wl.weight(d_out, d_in, 901)
    c = wl.activations(1, d_in, 902)[0].abs() + 0.01
    c = c.to(torch.float16)
    X = torch.diag(c.float()).to(torch.float16)
    x = c.float().numpy()
    err_g, best_g = _run(X, W, x, 128)
    err_o, best_o, _ = oracle.scale_search([W.numpy()], x, 128, 20)
    _check(err_g, best_g, err_o)


def test_output_error_down_proj_config_sampled_and_additive():
    """The 4096 x 12288 down_proj with 8192 tokens: an 8-token sample is
    compared with the oracle, and the full run equals the sum of its two
    token halves (different M tilings) within 1e-6."""
    work = wl.WORKLOADS["down_proj_output_error"]
    (grp, Ws, X), = wl.group_inputs(work)
    W = Ws[0]
    x = oracle.act_stats(X.numpy())
    Xs = X[:8].contiguous()
    err_s, best_s = _run(Xs, W, x, 128)
    err_o = oracle.output_error(Xs.numpy(), W.numpy(), x, 128, 20)
    _check(err_s, best_s, err_o)
    err_full, _ = _run(X, W, x, 128)
    err_a, _ = _run(X[:4096].contiguous(), W, x, 128)
    err_b, _ = _run(X[4096:].contiguous(), W, x, 128)
    np.testing.assert_allclose(err_full, err_a + err_b, rtol=1e-6, atol=0)


def test_output_error_down_proj_row_slice_all_tokens():
    """Realistic dense X at the full config: 128 rows of the 4096 x 12288
    down_proj scored over all 8192 heavy-tailed tokens and all 12288
    channels, every grid point against the fp64 oracle on the same slice
    (x from the full X, as the method takes it)."""
    work = wl.WORKLOADS["down_proj_output_error"]
    (grp, Ws, X), = wl.group_inputs(work)
    W = Ws[0][:128].contiguous()
    x = oracle.act_stats(X.numpy())
    err_g, best_g = _run(X, W, x, 128)
    err_o = oracle.output_error(X.numpy(), W.numpy(), x, 128, 20)
    _check(err_g, best_g, err_o)


def test_output_error_fp32_scale_and_nonfinite():
    W = wl.weight(64, 256, 77)
    X = wl.activations(32, 256, 78)
    x = oracle.act_stats(X.numpy())
    err_g, best_g = _run(X, W, x, 128, 20, awq.SCALE_FP32)
    err_o = oracle.output_error(X.numpy(), W.numpy(), x, 128, 20, oracle.SCALE_FP32)
    _check(err_g, best_g, err_o)
    W[5, 9] = float("nan")
    err_g, best_g = _run(X, W, x, 128)
    assert best_g == -1 and np.isnan(err_g).all()


@pytest.mark.parametrize("T,d_out,d_in,g", [(64, 256, 512, 128), (100, 264, 640, 64),
                                            (256, 512, 1024, 32)])
def test_output_error_asym(T, d_out, d_in, g):
    """The asymmetric grid (AWQ_ASYMMETRIC) in output space against the fp64
    oracle; s_best is the plain scale-table row (the grid does not change the
    candidates)."""
    seed = 3 * T + d_out + d_in + g
    W = wl.weight(d_out, d_in, seed + 1)
    X = wl.activations(T, d_in, seed)
    x = oracle.act_stats(X.numpy())
    err_g, best_g = _run(X, W, x, g, 20, awq.ASYMMETRIC)
    err_o = oracle.output_error(X.numpy(), W.numpy(), x, g, 20, oracle.ASYM)
    _check(err_g, best_g, err_o)
    W[3, 17] = float("nan")
    err_g, best_g = _run(X, W, x, g, 20, awq.ASYMMETRIC)
    assert best_g == -1 and not np.isfinite(err_g).any()


@pytest.mark.parametrize("n_grid", [1, 32])
def test_output_error_grid_sizes(n_grid):
    W = wl.weight(64, 256, 31 + n_grid)
    X = wl.activations(48, 256, 32 + n_grid)
    x = oracle.act_stats(X.numpy())
    err_g, best_g = _run(X, W, x, 64, n_grid)
    err_o = oracle.output_error(X.numpy(), W.numpy(), x, 64, n_grid)
    _check(err_g, best_g, err_o)
    if n_grid == 1:
        assert best_g == 0
