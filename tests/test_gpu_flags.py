"""Sticky device flags (awq_last_device_flags) on the GPU.

Non-finite data is made on the host (a NaN or an infinity written into an
input before it is copied to the device), never by a fault.  Each call that
meets it must raise its AWQ_FLAG_* bit besides what its outputs show; clean
inputs raise nothing; a clearing read zeroes the bits and a non-clearing
read keeps them.  The bounded-wait bit (AWQ_FLAG_WAIT_TIMEOUT) fires through
the search's test hook AWQ_TEST_STALL_WAIT: one weight load is armed for 16
bytes that never come, a phase that nothing completes (the copy itself
lands), so the waits run to their limits and give up; no fault, trap or
endless loop is involved.
"""
import time

import numpy as np
import pytest
import torch

import oracle
from post_int4_weight_b200 import awq
from post_int4_weight_b200 import workloads as wl

pytestmark = pytest.mark.gpu

OK, NONFINITE, TIMEOUT = 0, 6, 7


@pytest.fixture(autouse=True)
def _clean_flags():
    assert torch.cuda.is_available(), "the gpu tests need a CUDA device"
    awq.last_device_flags(clear=True)    # bits other tests may have left
    yield


def _clean_inputs(d_out=256, d_in=512, T=64, seed=7):
    W = wl.weight(d_out, d_in, seed + 1).cuda()
    X = wl.activations(T, d_in, seed).cuda()
    return W, X


def test_clean_path_raises_nothing():
    W, X = _clean_inputs()
    err, best, s, packed = awq.quantize_group([W], X, 128, 20, 8)
    st, bits = awq.last_device_flags()
    assert (st, bits) == (OK, 0)
    assert int(best.cpu()[0]) >= 0


def test_nonfinite_x_raises_x_and_clears():
    W, X = _clean_inputs()
    Xh = X.cpu()
    Xh[3, 17] = float("nan")
    Xh[5, 40] = float("inf")
    x = awq.act_stats(Xh.cuda())
    xs = x.cpu().numpy()
    assert np.isnan(xs[17]) and np.isinf(xs[40])
    st, bits = awq.last_device_flags(clear=False)
    assert st == NONFINITE and bits == awq.FLAG_NONFINITE_X
    st, bits = awq.last_device_flags(clear=True)     # still there, then cleared
    assert st == NONFINITE and bits == awq.FLAG_NONFINITE_X
    assert awq.last_device_flags() == (OK, 0)
    # the NaN mean makes the search's errors non-finite: a second bit
    err, best, s = awq.scale_search([W], x, 128, 20)
    assert int(best.cpu()[0]) == -1
    st, bits = awq.last_device_flags()
    assert st == NONFINITE and bits == awq.FLAG_NONFINITE_SCORE


def test_nonfinite_weight_raises_score_and_group():
    W, X = _clean_inputs()
    Wh = W.cpu()
    Wh[9, 130] = float("nan")
    Wn = Wh.cuda()
    x = awq.act_stats(X)
    err, best, s = awq.scale_search([Wn], x, 128, 20)
    assert int(best.cpu()[0]) == -1
    st, bits = awq.last_device_flags()
    assert st == NONFINITE and bits == awq.FLAG_NONFINITE_SCORE
    # the pack at a finite scale meets the NaN group
    s_ok = torch.ones(W.shape[1], dtype=torch.float32, device="cuda")
    qw, sc, qz = awq.quantize_pack(Wn, s_ok, 128, 8)
    assert torch.isnan(sc[1, 9].float()).item()
    st, bits = awq.last_device_flags()
    assert st == NONFINITE and bits == awq.FLAG_NONFINITE_GROUP
    # asymmetric pack as well
    awq.quantize_pack(Wn, s_ok, 128, awq.ZERO_POINT_ASYM)
    assert awq.last_device_flags() == (NONFINITE, awq.FLAG_NONFINITE_GROUP)
    # the clip search's totals
    idx, e2 = awq.clip_search(Wn, x, s_ok, 128, 10)
    assert not np.isfinite(e2.cpu().numpy()).all()
    assert awq.last_device_flags() == (NONFINITE, awq.FLAG_NONFINITE_SCORE)
    # and the output-space mode
    err, best, s = awq.output_error(X, Wn, x, 128, 20)
    assert int(best.cpu()[0]) == -1
    assert awq.last_device_flags() == (NONFINITE, awq.FLAG_NONFINITE_SCORE)


def test_nonfinite_member_scale_raises_scale():
    a = torch.full((256,), 2.0, dtype=torch.float32, device="cuda")
    b = a.clone()
    b[11] = float("inf")
    out = awq.norm_group_scale([a, b])
    assert torch.isinf(out[11]).item()
    assert awq.last_device_flags() == (NONFINITE, awq.FLAG_NONFINITE_SCALE)
    awq.norm_group_scale([a, a])
    assert awq.last_device_flags() == (OK, 0)


def test_bits_accumulate_until_read():
    W, X = _clean_inputs()
    Xh = X.cpu()
    Xh[0, 0] = float("nan")
    awq.act_stats(Xh.cuda())
    Wh = W.cpu()
    Wh[0, 0] = float("inf")
    s_ok = torch.ones(W.shape[1], dtype=torch.float32, device="cuda")
    awq.quantize_pack(Wh.cuda(), s_ok, 128, 8)
    st, bits = awq.last_device_flags()
    assert st == NONFINITE
    assert bits == awq.FLAG_NONFINITE_X | awq.FLAG_NONFINITE_GROUP


def test_stalled_wait_gives_up_and_the_next_call_runs():
    """The give-up path of the bounded waits, on the search kernel: with
    AWQ_TEST_STALL_WAIT, CTA 0's first weight load never completes its
    phase.  Its consumer warps give up after the 2 s limit, the CTA stops
    computing but takes every barrier, its drain gives up after 20 s (the
    copy has landed; only the phase is missing), and the call reports
    best_idx = -2, NaN s_best and AWQ_FLAG_WAIT_TIMEOUT.  The context stays
    usable: the same search without the hook then matches the oracle."""
    W, X = _clean_inputs(d_out=512, d_in=1024, T=128, seed=11)
    x = awq.act_stats(X)
    torch.cuda.synchronize()
    t0 = time.monotonic()
    err, best, s = awq.scale_search([W], x, 128, 20, awq.TEST_STALL_WAIT)
    b = int(best.cpu()[0])
    waited = time.monotonic() - t0
    assert b == -2
    assert np.isnan(s.cpu().numpy()).all()
    assert waited >= 2.0                     # the waits ran to their limit
    st, bits = awq.last_device_flags()
    assert st == TIMEOUT and (bits & awq.FLAG_WAIT_TIMEOUT)
    assert awq.last_device_flags() == (OK, 0)
    # the next call on the same context runs normally
    err2, best2, s2 = awq.scale_search([W], x, 128, 20)
    torch.cuda.synchronize()
    e_o, b_o, s_o = oracle.scale_search([W.cpu().numpy()], x.cpu().numpy(), 128, 20)
    np.testing.assert_allclose(err2.cpu().numpy(), e_o, rtol=1e-5, atol=0)
    b2 = int(best2.cpu()[0])
    if b2 != b_o:   # a tie within the method's 1e-6 (the first minimum may differ)
        assert abs(e_o[b2] - e_o[b_o]) <= 1e-6 * e_o[b_o]
    else:
        assert np.array_equal(s2.cpu().numpy(), s_o)
    assert awq.last_device_flags() == (OK, 0)
