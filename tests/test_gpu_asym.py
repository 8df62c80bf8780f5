"""Asymmetric INT4 (AWQ_ASYMMETRIC search, AWQ_ZERO_POINT_ASYM pack) on the
GPU against the CPU oracle: scale, zero points, codes, packed words and
qzeros bit-exact; searched errors within 1e-5; index exact or tied within
1e-6."""
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


def _pack_both(W, s, g):
    dev = torch.device("cuda")
    qw, sc, qz = awq.quantize_pack(W.to(dev), None if s is None else torch.from_numpy(s).to(dev),
                                   g, awq.ZERO_POINT_ASYM)
    torch.cuda.synchronize()
    qw_o, sc_o, qz_o = oracle.quantize_pack(W.numpy(), s, g, -1)
    assert np.array_equal(qw.cpu().numpy(), qw_o)
    assert np.array_equal(sc.cpu().numpy().view(np.uint16), sc_o.view(np.uint16))
    assert np.array_equal(qz.cpu().numpy(), qz_o)


@pytest.mark.parametrize("d_out,d_in,g", [(256, 512, 128), (72, 384, 64), (40, 256, 32),
                                          (8, 128, 128), (200, 1024, 128)])
def test_asym_pack_parity(d_out, d_in, g):
    W = wl.weight(d_out, d_in, d_out + d_in + g)
    rng = np.random.default_rng(g + d_out)
    s = np.exp(rng.standard_normal(d_in) * 0.7).astype(np.float32)
    _pack_both(W, s, g)
    _pack_both(W, None, g)


def test_asym_pack_edge_groups():
    g = 64
    W = wl.weight(16, 4 * g, 11)
    W[0, :g] = 0.0                              # zero group: range clamps to 1e-5
    W[1, :g] = 0.01                             # constant positive group: zero = 0
    W[2, :g] = -0.02                            # constant negative group: zero = 15
    W[3, g:2 * g] = torch.abs(W[3, g:2 * g])    # all non-negative: min > 0
    W[4, 5] = float("nan")                      # non-finite: scale NaN, codes 8
    W[5, g + 7] = float("inf")
    W[6, :g] = torch.linspace(-0.5, 0.5, g).half()   # the page's worked example range
    W[7, 2 * g:3 * g] = 60000.0                 # scale near the fp16 top
    W[7, 2 * g] = -60000.0
    _pack_both(W, None, g)
    s = np.full(4 * g, 3.0, np.float32)
    _pack_both(W, s, g)


def _search_both(Ws, X, g, flags):
    dev = torch.device("cuda")
    x_g = awq.act_stats(X.to(dev))
    err, best, s = awq.scale_search([W.to(dev) for W in Ws], x_g, g, 20, flags)
    torch.cuda.synchronize()
    x = oracle.act_stats(X.numpy())
    ofl = (oracle.ASYM if flags & awq.ASYMMETRIC else 0) | \
        (oracle.DUO if flags & awq.DUO_SCALING else 0) | (flags & 1)
    err_o, best_o, s_o = oracle.scale_search([W.numpy() for W in Ws], x, g, 20, ofl)
    err, b, s = err.cpu().numpy(), int(best.cpu()[0]), s.cpu().numpy()
    np.testing.assert_allclose(err, err_o, rtol=ERR_RTOL, atol=0)
    if b != best_o:
        assert abs(err_o[b] - err_o[best_o]) <= TIE_RTOL * err_o[best_o]
    elif not flags & awq.DUO_SCALING:
        assert np.array_equal(s, s_o)
    return s


@pytest.mark.parametrize("d_outs,d_in,T,g,flags", [
    ((256,), 512, 64, 128, awq.ASYMMETRIC),
    ((200, 72, 8), 1024, 96, 64, awq.ASYMMETRIC),
    ((64,), 256, 32, 32, awq.ASYMMETRIC | awq.SCALE_FP32),
    ((128,), 512, 64, 128, awq.ASYMMETRIC | awq.DUO_SCALING)])
def test_asym_search_parity(d_outs, d_in, T, g, flags):
    seed = sum(d_outs) + d_in + g + flags
    Ws = [wl.weight(d, d_in, seed + m + 1) for m, d in enumerate(d_outs)]
    X = wl.activations(T, d_in, seed)
    _search_both(Ws, X, g, flags)


def test_asym_q_proj_end_to_end():
    work = wl.WORKLOADS["q_proj_4096x4096"]
    (grp, Ws, X), = wl.group_inputs(work)
    s = _search_both(Ws, X, 128, awq.ASYMMETRIC)
    _pack_both(Ws[0], s, 128)


def test_asym_nonfinite_reports_minus_one():
    W = wl.weight(64, 256, 3)
    W[9, 100] = float("nan")
    X = wl.activations(32, 256, 4)
    x = awq.act_stats(X.cuda())
    err, best, s = awq.scale_search([W.cuda()], x, 128, 20, awq.ASYMMETRIC)
    torch.cuda.synchronize()
    assert int(best.cpu()[0]) == -1 and np.isnan(s.cpu().numpy()).all()


def test_asym_duo_stack_layer_gate_up():
    """The 36-layer stack's gate/up group (2 x 12288 rows, 2048 tokens) with
    the asymmetric grid and duo scaling together."""
    work = wl.WORKLOADS["qwen3_8b_stack36"]
    grp, Ws, X = wl.group_inputs(work, 17)[2]
    s = _search_both(Ws, X, 128, awq.ASYMMETRIC | awq.DUO_SCALING)
    _pack_both(Ws[1], s, 128)
