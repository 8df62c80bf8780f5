"""awq_scale_search_noalloc: the scale search for callers that cannot
allocate device memory (their host framework owns all device memory, or a
cudaMalloc is not acceptable where they run), using the library's static
per-device scratch instead of a workspace.

Collected last (file name) so that a stop-at-first-failure run has already
run every other test; it must also pass alone in a fresh process.
"""
import numpy as np
import pytest
import torch

from post_int4_weight_b200 import awq
from post_int4_weight_b200 import workloads as wl

pytestmark = pytest.mark.gpu

ERR_RTOL = 1e-5   # the tolerance the parity tests use for error sums


def _inputs(d_outs, d_in, T, seed):
    Ws = [wl.weight(d, d_in, seed + k + 1).cuda() for k, d in enumerate(d_outs)]
    X = wl.activations(T, d_in, seed).cuda()
    return Ws, awq.act_stats(X)


def test_noalloc_matches_workspace_search_on_two_calls_in_a_row():
    assert torch.cuda.is_available(), "needs a CUDA device"
    calls = [([256, 64, 64], 512, 64, 128, 101),
             ([200], 1024, 96, 64, 202)]
    for d_outs, d_in, T, g, seed in calls:
        Ws, x = _inputs(d_outs, d_in, T, seed)
        e_ref, b_ref, s_ref = awq.scale_search(Ws, x, g, 20)
        e_na, b_na, s_na = awq.scale_search_noalloc(Ws, x, g, 20)
        torch.cuda.synchronize()
        e_ref, e_na = e_ref.cpu().numpy(), e_na.cpu().numpy()
        np.testing.assert_allclose(e_na, e_ref, rtol=ERR_RTOL, atol=0)
        assert int(b_na.cpu()[0]) == int(b_ref.cpu()[0])
        assert np.array_equal(s_na.cpu().numpy(), s_ref.cpu().numpy())


def test_noalloc_rejects_sizes_beyond_its_scratch():
    Ws, x = _inputs([64], 256, 16, 303)
    big = torch.zeros(1 << 17, dtype=torch.float32, device="cuda")
    Wbig = torch.zeros(8, 1 << 17, dtype=torch.float16, device="cuda")
    with pytest.raises(awq.AwqError) as ei:
        awq.scale_search_noalloc([Wbig], big, 128, 20)
    assert ei.value.status == 4   # AWQ_ERR_WORKSPACE
    # the entry point still works after a rejected call
    e, b, s = awq.scale_search_noalloc(Ws, x, 128, 20)
    torch.cuda.synchronize()
    assert np.isfinite(e.cpu().numpy()).all() and int(b.cpu()[0]) >= 0
