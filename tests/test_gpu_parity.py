"""CUDA path vs the CPU oracle, element by element, through the C ABI.

Bars (the method's contract): bit-exact activation means, scale vectors,
INT4 codes, packed words, fp16 group scales and the chosen grid index (a
different index is accepted only when the two errors tie within 1e-6
relative); error sums within 1e-5 relative.

Inputs come from the seeded generator in post_int4_weight_b200.workloads;
the oracle never receives a value computed by the CUDA path.
"""
import zlib

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
    torch.cuda.init()


def _np(t):
    return t.detach().cpu().numpy()


def _search_both(Ws, X, g=128, n_grid=20, flags=0):
    """GPU: stats + search on device; oracle: the same from the same inputs."""
    dev = torch.device("cuda")
    Xd = X.to(dev)
    Wd = [W.to(dev) for W in Ws]
    x_g = awq.act_stats(Xd)
    err_g, best_g, s_g = awq.scale_search(Wd, x_g, g, n_grid, flags)
    torch.cuda.synchronize()
    x_o = oracle.act_stats(X.numpy())
    err_o, best_o, s_o = oracle.scale_search([W.numpy() for W in Ws], x_o, g, n_grid, flags)
    return (dict(x=_np(x_g), err=_np(err_g), best=int(_np(best_g)[0]), s=_np(s_g),
                 Wd=Wd, x_dev=x_g, s_dev=s_g),
            dict(x=x_o, err=err_o, best=best_o, s=s_o))


def _assert_search_parity(gpu, orc):
    assert np.array_equal(gpu["x"], orc["x"], equal_nan=True)
    np.testing.assert_allclose(gpu["err"], orc["err"], rtol=ERR_RTOL, atol=0)
    if gpu["best"] != orc["best"]:
        e = orc["err"]
        assert abs(e[gpu["best"]] - e[orc["best"]]) <= TIE_RTOL * e[orc["best"]], (
            gpu["best"], orc["best"], e)
    else:
        assert np.array_equal(gpu["s"], orc["s"])


def _assert_pack_parity(W, s_np, s_dev, g, zp):
    qw, sc, qz = awq.quantize_pack(W, s_dev, g, zp)
    torch.cuda.synchronize()
    qw_o, sc_o, qz_o = oracle.quantize_pack(_np(W), s_np, g, zp)
    assert np.array_equal(_np(qw), qw_o)
    assert np.array_equal(_np(sc).view(np.uint16), sc_o.view(np.uint16))
    assert np.array_equal(_np(qz), qz_o)


# --------------------------------------------------------------- stats --

@pytest.mark.parametrize("T,d_in", [(64, 512), (1, 8), (37, 136), (513, 1024),
                                    (4096, 4096), (3, 12288)])
def test_act_stats_bit_exact(T, d_in):
    X = wl.activations(T, d_in, seed=T * 7 + d_in)
    x = awq.act_stats(X.cuda())
    torch.cuda.synchronize()
    assert np.array_equal(_np(x), oracle.act_stats(X.numpy()))


def test_act_stats_long_token_slices():
    """More than 4096 rows per thread (32 row lanes x 8 CTAs of a cluster:
    T > 8 * 32 * 4096): the exact fp64 partial sums are moved into the
    integer accumulators mid-way, and a column of 65504 drives a thread's
    count to the largest value the conversion allows (4096 x 65504 x 2^24)."""
    X = wl.activations(1_310_731, 16, seed=77)
    X[:, 3] = 65504.0                      # the largest sums the format allows
    x = awq.act_stats(X.cuda())
    torch.cuda.synchronize()
    assert np.array_equal(_np(x), oracle.act_stats(X.numpy()))


def test_act_stats_nonfinite_and_extremes():
    X = wl.activations(40, 64, seed=5)
    X[3, 1] = float("inf")
    X[7, 2] = float("nan")
    X[9, 3] = -float("inf")
    X[:, 4] = 65504.0            # largest fp16
    X[:, 5] = 5.96e-08           # smallest subnormal fp16
    X[:, 6] = 0.0
    x = _np(awq.act_stats(X.cuda()))
    torch.cuda.synchronize()
    xo = oracle.act_stats(X.numpy())
    assert np.array_equal(x, xo, equal_nan=True)
    assert x[1] == np.inf and np.isnan(x[2]) and x[3] == np.inf and x[4] == 65504.0


# -------------------------------------------------------------- search --

SEARCH_CASES = [
    # (name, [d_out per segment], d_in, T, g, n_grid, flags)
    ("single_linear_256x512_g128", [256], 512, 64, 128, 20, 0),
    ("g64", [256], 512, 64, 64, 20, 0),
    ("g32", [128], 256, 48, 32, 20, 0),
    ("ragged_rows_200", [200], 384, 32, 128, 20, 0),
    ("ragged_rows_72_g32", [72], 96, 16, 32, 20, 0),
    ("three_segments", [96, 24, 40], 256, 40, 64, 20, 0),
    ("eight_segments", [8, 16, 24, 8, 64, 8, 32, 72], 128, 24, 128, 20, 0),
    ("n_grid_1", [64], 256, 16, 128, 1, 0),
    ("n_grid_7", [64], 256, 16, 128, 7, 0),
    ("n_grid_32", [64], 256, 16, 128, 32, 0),
    ("fp32_scale", [128], 256, 32, 128, 20, 1),
    ("single_row", [1], 128, 8, 128, 20, 0),
]


@pytest.mark.parametrize("case", SEARCH_CASES, ids=[c[0] for c in SEARCH_CASES])
def test_search_parity(case):
    name, d_outs, d_in, T, g, n_grid, flags = case
    seed = zlib.crc32(name.encode()) % 10000
    Ws = [wl.weight(d, d_in, seed + k + 1) for k, d in enumerate(d_outs)]
    X = wl.activations(T, d_in, seed)
    gpu, orc = _search_both(Ws, X, g, n_grid, flags)
    _assert_search_parity(gpu, orc)


def test_search_is_deterministic():
    Ws = [wl.weight(512, 1024, 3)]
    X = wl.activations(256, 1024, 4)
    x = awq.act_stats(X.cuda())
    W = Ws[0].cuda()
    outs = [awq.scale_search([W], x, 128, 20) for _ in range(3)]
    torch.cuda.synchronize()
    for e, b, s in outs[1:]:
        assert np.array_equal(_np(e), _np(outs[0][0]))
        assert np.array_equal(_np(s), _np(outs[0][2]))


def test_search_zero_weights():
    W = torch.zeros(64, 256, dtype=torch.float16)
    X = wl.activations(16, 256, 9)
    gpu, orc = _search_both([W], X)
    assert np.all(gpu["err"] == 0) and gpu["best"] == 0
    _assert_search_parity(gpu, orc)


def test_search_tiny_and_huge_groups():
    """fp16-subnormal group scales (codes can clamp) and saturated ones."""
    W = wl.weight(64, 256, 10)
    W[:16] = (W[:16].float() * 1e-3).half()      # subnormal-range groups
    W[16:24, :128] = 65504.0 / 4                 # large groups
    W[24, 5] = 60000.0
    X = wl.activations(32, 256, 11)
    gpu, orc = _search_both([W], X)
    _assert_search_parity(gpu, orc)


def test_search_zero_activation_channels():
    W = wl.weight(64, 256, 12)
    X = wl.activations(16, 256, 13)
    X[:, :7] = 0.0                               # x = 0 -> clamped to 1e-4
    gpu, orc = _search_both([W], X)
    _assert_search_parity(gpu, orc)


def test_search_nonfinite_weight_reports_minus_one():
    W = wl.weight(64, 256, 14)
    W[3, 17] = float("nan")
    X = wl.activations(16, 256, 15)
    gpu, orc = _search_both([W], X)
    assert orc["best"] == -1 and gpu["best"] == -1
    assert np.all(np.isnan(gpu["s"]))


# ---------------------------------------------------------------- pack --

PACK_CASES = [
    # (d_out, d_in, g, zp, with_s)
    (256, 512, 128, 8, True),
    (256, 512, 128, 8, False),
    (256, 512, 128, 7, True),
    (512, 256, 64, 8, True),
    (256, 128, 32, 8, True),
    (200, 384, 128, 8, True),     # C = 25 words: scalar stores, ragged rows
    (264, 96, 32, 7, True),       # d_in not a multiple of the 128-column tile
    (8, 192, 64, 8, True),        # a single word row
    (120, 256, 64, 7, True),      # a 64-row tile, then one with 56 rows (a partial warp)
    (328, 640, 128, 8, True),     # five whole 64-row tiles and an 8-row one
]


@pytest.mark.parametrize("d_out,d_in,g,zp,with_s", PACK_CASES)
def test_pack_parity(d_out, d_in, g, zp, with_s):
    seed = d_out * 31 + d_in + g + zp
    W = wl.weight(d_out, d_in, seed)
    s_np = None
    s_dev = None
    if with_s:
        gen = torch.Generator().manual_seed(seed)
        s = torch.exp(torch.randn(d_in, generator=gen) * 1.5).float()
        s_np, s_dev = s.numpy(), s.cuda()
    _assert_pack_parity(W.cuda(), s_np, s_dev, g, zp)


def test_pack_edge_groups():
    W = wl.weight(64, 256, 21)
    W[0:8] = 0.0                                  # zero groups: scale 0
    W[8:16] = (W[8:16].float() * 1e-3).half()     # subnormal scales
    W[16:24, :128] = 65504.0                      # fp16 overflow -> 65504, clamp
    W[24, 3] = float("nan")                       # non-finite group
    W[25, 200] = float("inf")
    # exact half-way quotients: q_scale = 0.125, w = k * 0.0625
    W[32:40, 128:256] = 0.0
    W[32:40, 128] = -0.875
    for i in range(1, 15):
        W[32:40, 128 + i] = i * 0.0625 - 0.5
    _assert_pack_parity(W.cuda(), None, None, 128, 8)
    gen = torch.Generator().manual_seed(22)
    s = torch.exp(torch.randn(256, generator=gen)).float()
    _assert_pack_parity(W.cuda(), s.numpy(), s.cuda(), 128, 8)


def test_pack_every_fp16_quotient_below_many_maxima():
    """Row k's group holds its maximum m_k at column 0 and then every fp16
    value in [-m_k, m_k] in turn (s = 1, so ws = w exactly and q_scale =
    fp16(m_k / 7)): every rounding decision of those scales, ties included,
    is compared bit for bit."""
    rng = np.random.default_rng(5)
    all_pos = np.arange(1, 0x7C00, dtype=np.uint16).view(np.float16).astype(np.float32)
    maxima = np.concatenate([
        np.array([65504.0, 1.0, 0.875, 7 * 2.0 ** -14, 7 * 2.0 ** -14 * 0.999, 3e-7, 1e-3],
                 np.float32),
        np.float16(np.exp(rng.uniform(np.log(1e-6), np.log(6e4), 41))).astype(np.float32)])
    rows = []
    for m in np.float16(maxima).astype(np.float32):
        vals = all_pos[all_pos <= m]
        vals = np.concatenate([vals, -vals])
        for k in range(0, len(vals), 127):
            chunk = vals[k:k + 127]
            row = np.zeros(128, np.float32)
            row[0] = m
            row[1:1 + len(chunk)] = chunk
            rows.append(row)
    pad = (-len(rows)) % 8
    rows += [np.zeros(128, np.float32)] * pad
    W = torch.from_numpy(np.stack(rows).astype(np.float16))
    _assert_pack_parity(W.cuda(), None, None, 128, 8)


# ------------------------------------------------------- end to end --

def _end_to_end(workload, g, check_pack_rows=None):
    for grp, Ws, X in wl.group_inputs(workload):
        gpu, orc = _search_both(Ws, X, g, workload.n_grid)
        _assert_search_parity(gpu, orc)
        s_np = orc["s"] if gpu["best"] == orc["best"] else oracle.scale_table(
            orc["x"], workload.n_grid)[gpu["best"]]
        for W, Wd in zip(Ws, gpu["Wd"]):
            _assert_pack_parity(Wd, s_np, gpu["s_dev"], g, 8)
        del gpu
        torch.cuda.empty_cache()


def test_end_to_end_single_linear_config():
    _end_to_end(wl.WORKLOADS["single_linear_256x512"], 128)


def test_end_to_end_q_proj_4096():
    _end_to_end(wl.WORKLOADS["q_proj_4096x4096"], 128)


@pytest.mark.parametrize("g", [128, 64])
def test_end_to_end_qwen3_block(g):
    _end_to_end(wl.WORKLOADS["qwen3_8b_block"], g)
