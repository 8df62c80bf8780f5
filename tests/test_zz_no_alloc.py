"""awq_scale_search_noalloc: the scale search for callers that cannot
allocate device memory (their host framework owns all device memory, or a
cudaMalloc is not acceptable where they run), using the library's static
per-device scratch instead of a workspace.

Each call is compared with the workspace entry point (same bits expected:
the kernels are the same) and with the CPU oracle at the parity bars of the
other search tests (errors within 1e-5 relative, index exact or tied within
1e-6, the chosen scale bit for bit; duo scaling as in the duo tests, whose
fp64 weight mean may move an fp32 scale entry by one ulp).

Collected last (file name) so that a stop-at-first-failure run has already
run every other test; it must also pass alone in a fresh process.
"""
import numpy as np
import pytest
import torch

import oracle
from post_int4_weight_b200 import awq
from post_int4_weight_b200 import workloads as wl

pytestmark = pytest.mark.gpu

ERR_RTOL = 1e-5   # the tolerance the parity tests use for error sums
TIE_RTOL = 1e-6


def _inputs(d_outs, d_in, T, seed):
    Ws = [wl.weight(d, d_in, seed + k + 1) for k, d in enumerate(d_outs)]
    X = wl.activations(T, d_in, seed)
    return Ws, X


def _check_against_oracle(Ws, X, g, flags, err, best, s):
    x = oracle.act_stats(X.numpy())
    ofl = oracle.DUO if flags & awq.DUO_SCALING else 0
    err_o, best_o, s_o = oracle.scale_search([W.numpy() for W in Ws], x, g, 20, ofl)
    np.testing.assert_allclose(err, err_o, rtol=ERR_RTOL, atol=0)
    if best != best_o:
        assert abs(err_o[best] - err_o[best_o]) <= TIE_RTOL * err_o[best_o]
        if ofl:
            s_o = oracle.scale_table_duo(x, oracle.weight_mean([W.numpy() for W in Ws]), 20)[best]
        else:
            s_o = oracle.scale_table(x, 20)[best]
    if ofl:
        ulp = np.abs(s.view(np.int32).astype(np.int64) - s_o.view(np.int32).astype(np.int64))
        assert ulp.max() <= 1 and (ulp > 0).sum() <= max(1, s.size // 1000)
    else:
        assert np.array_equal(s.view(np.uint32), s_o.view(np.uint32))


def test_noalloc_matches_workspace_search_and_oracle_on_calls_in_a_row():
    assert torch.cuda.is_available(), "needs a CUDA device"
    calls = [([256, 64, 64], 512, 64, 128, 0, 101),
             ([200], 1024, 96, 64, 0, 202),
             ([96, 40], 1024, 80, 128, awq.DUO_SCALING, 303),   # duo tables in the array
             ([256, 64, 64], 512, 64, 128, 0, 101)]             # the first call again
    for d_outs, d_in, T, g, flags, seed in calls:
        Ws, X = _inputs(d_outs, d_in, T, seed)
        Wd = [W.cuda() for W in Ws]
        x = awq.act_stats(X.cuda())
        e_ref, b_ref, s_ref = awq.scale_search(Wd, x, g, 20, flags)
        e_na, b_na, s_na = awq.scale_search_noalloc(Wd, x, g, 20, flags)
        torch.cuda.synchronize()
        e_ref, e_na = e_ref.cpu().numpy(), e_na.cpu().numpy()
        b_na, s_na = int(b_na.cpu()[0]), s_na.cpu().numpy()
        np.testing.assert_allclose(e_na, e_ref, rtol=ERR_RTOL, atol=0)
        assert b_na == int(b_ref.cpu()[0])
        assert np.array_equal(s_na, s_ref.cpu().numpy())
        _check_against_oracle(Ws, X, g, flags, e_na, b_na, s_na)


def test_noalloc_rejects_sizes_beyond_its_scratch_and_bad_arguments():
    Ws, X = _inputs([64], 256, 16, 404)
    Wd = [W.cuda() for W in Ws]
    x = awq.act_stats(X.cuda())
    big = torch.zeros(1 << 17, dtype=torch.float32, device="cuda")
    Wbig = torch.zeros(8, 1 << 17, dtype=torch.float16, device="cuda")
    with pytest.raises(awq.AwqError) as ei:
        awq.scale_search_noalloc([Wbig], big, 128, 20)
    assert ei.value.status == 4   # AWQ_ERR_WORKSPACE
    # argument errors come back with the codes of the workspace entry point
    ws = awq.workspace(awq.OP_SCALE_SEARCH, x.device, 1, 8, x.shape[0], 128, 20)
    for call in (lambda: awq.scale_search(Wd, x, 96, 20, ws=ws),
                 lambda: awq.scale_search_noalloc(Wd, x, 96, 20)):
        with pytest.raises(awq.AwqError) as ei:
            call()                        # a group size the library does not support
        assert ei.value.status == 2       # AWQ_ERR_UNSUPPORTED
    # the entry point still works after rejected calls
    e, b, s = awq.scale_search_noalloc(Wd, x, 128, 20)
    torch.cuda.synchronize()
    _check_against_oracle(Ws, X, 128, 0, e.cpu().numpy(), int(b.cpu()[0]), s.cpu().numpy())
