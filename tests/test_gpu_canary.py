"""Out-of-bounds writes and run-to-run determinism of every entry point.

No memory checker runs on this GPU pool, so every output and every
workspace here is carved out of a larger byte buffer whose margins (and the
slack up to the next 16 bytes) hold a pattern that no kernel may change.
The inputs are compared with copies taken before the calls.  The shapes are
ragged: rows not a multiple of the 128-row tiles, d_in not a multiple of
the 128-column tiles, several segments.  Each call runs twice; its outputs
must be the same bits both times.
"""
import numpy as np
import pytest
import torch

from post_int4_weight_b200 import awq
from post_int4_weight_b200 import workloads as wl

pytestmark = pytest.mark.gpu

PAD = 4096          # canary bytes on each side; keeps every carve 16-byte aligned
CANARY = 0xA5


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "the gpu tests need a CUDA device"


class Arena:
    """Tensors carved out of byte buffers with canary margins."""

    def __init__(self):
        self.bufs = []

    def take(self, shape, dtype):
        n = int(np.prod(shape)) * torch.tensor([], dtype=dtype).element_size()
        n16 = (max(n, 1) + 15) // 16 * 16
        buf = torch.full((PAD + n16 + PAD,), CANARY, dtype=torch.uint8, device="cuda")
        self.bufs.append((buf, n))
        return buf[PAD:PAD + n].view(dtype).view(shape)

    def workspace(self, op, T, d_out_total, d_in, g, n_grid):
        n = awq.workspace_size(op, T, d_out_total, d_in, g, n_grid)
        return self.take((max(n, 1),), torch.uint8)

    def check(self):
        torch.cuda.synchronize()
        for buf, n in self.bufs:
            b = buf.cpu().numpy()
            assert np.all(b[:PAD] == CANARY), "write before the start of a buffer"
            assert np.all(b[PAD + n:] == CANARY), "write past the end of a buffer"


def _bits(ts):
    torch.cuda.synchronize()
    return [t.detach().cpu().contiguous().view(torch.uint8).numpy().copy() for t in ts]


def _twice(call, inputs):
    """Runs call() twice: same output bits, inputs untouched."""
    before = _bits(inputs)
    first = _bits(call())
    second = _bits(call())
    for a, b in zip(first, second):
        assert np.array_equal(a, b), "two runs gave different bits"
    for a, b in zip(before, _bits(inputs)):
        assert np.array_equal(a, b), "an input was modified"
    return first


def test_act_stats_canary():
    X = wl.activations(513, 136, 201).cuda()
    ar = Arena()
    x = ar.take((136,), torch.float32)
    ws = ar.workspace(awq.OP_ACT_STATS, 513, 8, 136, 128, 20)
    _twice(lambda: [awq.act_stats(X, out=x, ws=ws)], [X])
    ar.check()


SEARCH_FLAGS = [awq.SCALE_FP16, awq.SCALE_FP32, awq.ASYMMETRIC, awq.DUO_SCALING,
                awq.ASYMMETRIC | awq.DUO_SCALING]


@pytest.mark.parametrize("flags", SEARCH_FLAGS)
@pytest.mark.parametrize("g", [128, 32])
def test_scale_search_canary(flags, g):
    d_in = 384
    Ws = [wl.weight(d, d_in, 210 + d).cuda() for d in (200, 72, 8)]
    x = awq.act_stats(wl.activations(64, d_in, 211).cuda())
    ar = Arena()
    out = (ar.take((20,), torch.float64), ar.take((1,), torch.int32),
           ar.take((d_in,), torch.float32))
    op = awq.OP_SCALE_SEARCH_DUO if flags & awq.DUO_SCALING else awq.OP_SCALE_SEARCH
    ws = ar.workspace(op, 1, 280, d_in, g, 20)
    res = _twice(lambda: awq.scale_search(Ws, x, g, 20, flags, out=out, ws=ws), Ws + [x])
    ar.check()
    assert 0 <= int(res[1].view(np.int32)[0]) < 20


@pytest.mark.parametrize("zp,with_clip", [(8, False), (7, False), (awq.ZERO_POINT_ASYM, False),
                                          (8, True)])
def test_quantize_pack_canary(zp, with_clip):
    d_out, d_in, g = 200, 384, 128
    W = wl.weight(d_out, d_in, 220).cuda()
    x = awq.act_stats(wl.activations(64, d_in, 221).cuda())
    flags = awq.ASYMMETRIC if zp == awq.ZERO_POINT_ASYM else awq.SCALE_FP16
    _, _, s = awq.scale_search([W], x, g, 20, flags)
    clip = awq.clip_search(W, x, s, g, 10)[0] if with_clip else None
    ar = Arena()
    out = (ar.take((d_in, d_out // 8), torch.int32),
           ar.take((d_in // g, d_out), torch.float16),
           ar.take((d_in // g, d_out // 8), torch.int32))
    inputs = [W, s] + ([clip] if with_clip else [])
    _twice(lambda: awq.quantize_pack(W, s, g, zp, out=out, clip_idx=clip), inputs)
    ar.check()


@pytest.mark.parametrize("g", [128, 64])
def test_clip_search_canary(g):
    d_out, d_in = 200, 384
    W = wl.weight(d_out, d_in, 230).cuda()
    x = awq.act_stats(wl.activations(64, d_in, 231).cuda())
    _, _, s = awq.scale_search([W], x, g, 20)
    ar = Arena()
    out = (ar.take((d_out, d_in // g), torch.uint8), ar.take((2,), torch.float64))
    ws = ar.workspace(awq.OP_CLIP_SEARCH, 1, d_out, d_in, g, 1)
    _twice(lambda: awq.clip_search(W, x, s, g, 10, out=out, ws=ws), [W, x, s])
    ar.check()


def test_norm_group_scale_canary():
    ss = [awq.act_stats(wl.activations(16, 392, 240 + k).cuda()) for k in range(3)]
    ar = Arena()
    out = ar.take((392,), torch.float32)
    _twice(lambda: [awq.norm_group_scale(ss, out=out)], ss)
    ar.check()


def test_output_error_canary():
    T, d_out, d_in, g = 100, 264, 640, 64
    W = wl.weight(d_out, d_in, 250).cuda()
    X = wl.activations(T, d_in, 251).cuda()
    x = awq.act_stats(X)
    ar = Arena()
    out = (ar.take((20,), torch.float64), ar.take((1,), torch.int32),
           ar.take((d_in,), torch.float32))
    ws = ar.workspace(awq.OP_OUTPUT_ERROR, T, d_out, d_in, g, 20)
    res = _twice(lambda: awq.output_error(X, W, x, g, 20, out=out, ws=ws), [X, W, x])
    ar.check()
    assert 0 <= int(res[1].view(np.int32)[0]) < 20


@pytest.mark.parametrize("g", [128, 32])
def test_clip_search_output_canary(g):
    T, d_out, d_in = 72, 200, 384
    W = wl.weight(d_out, d_in, 260).cuda()
    X = wl.activations(T, d_in, 261).cuda()
    x = awq.act_stats(X)
    _, _, s = awq.scale_search([W], x, g, 20)
    ar = Arena()
    out = (ar.take((d_out, d_in // g), torch.uint8), ar.take((2,), torch.float64))
    ws = ar.workspace(awq.OP_CLIP_SEARCH_OUTPUT, T, d_out, d_in, g, 1)
    _twice(lambda: awq.clip_search_output(X, W, s, g, 10, out=out, ws=ws), [X, W, s])
    ar.check()
