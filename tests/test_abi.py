"""The C-ABI library loads on a host without a GPU, exports every symbol that
include/awq.h declares, and rejects bad arguments on the host before any
CUDA call (no compute call is made here)."""
import ctypes
import os
import re

import pytest

from post_int4_weight_b200 import awq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "awq.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(awq_[a-z_]+)\s*\(", text)))


def test_header_declares_the_four_calls():
    names = declared_functions()
    for n in ("awq_act_stats", "awq_scale_search", "awq_quantize_pack",
              "awq_output_error", "awq_workspace_size", "awq_status_string"):
        assert n in names


def test_library_exports_every_declared_symbol():
    lib = awq.lib()
    for name in declared_functions():
        assert hasattr(lib, name), name
        assert ctypes.cast(getattr(lib, name), ctypes.c_void_p).value


def test_status_strings_and_version():
    assert awq.string(0) == "AWQ_OK"
    for s in range(1, 8):
        assert awq.string(s).startswith("AWQ_ERR_")
    assert awq.string(6).startswith("AWQ_ERR_NONFINITE")
    assert awq.string(7).startswith("AWQ_ERR_DEVICE_TIMEOUT")
    assert awq.lib().awq_abi_version() == 101


def test_device_flag_bits_in_header_and_binding():
    """The AWQ_FLAG_* bits of the header are distinct powers of two and the
    binding carries the same values; a NULL output is an argument error,
    answered on the host."""
    text = open(HEADER).read()
    bits = {m.group(1): int(m.group(2), 16)
            for m in re.finditer(r"#define\s+(AWQ_FLAG_\w+)\s+0x([0-9a-fA-F]+)u", text)}
    assert set(bits) == {"AWQ_FLAG_NONFINITE_X", "AWQ_FLAG_NONFINITE_SCORE",
                         "AWQ_FLAG_NONFINITE_GROUP", "AWQ_FLAG_NONFINITE_SCALE",
                         "AWQ_FLAG_WAIT_TIMEOUT"}
    vals = sorted(bits.values())
    assert len(set(vals)) == len(vals) and all(v & (v - 1) == 0 for v in vals)
    for name, v in bits.items():
        assert getattr(awq, name[4:]) == v
    assert awq.lib().awq_last_device_flags(None, 0) == 1   # AWQ_ERR_INVALID_ARG


def test_workspace_sizes():
    n_stats = awq.workspace_size(awq.OP_ACT_STATS, 4096, 8, 4096, 128, 20)
    assert n_stats == 0
    n_search = awq.workspace_size(awq.OP_SCALE_SEARCH, 1, 8, 4096, 128, 20)
    assert n_search >= 2 * 20 * 4096 * 4
    with pytest.raises(awq.AwqError):
        awq.workspace_size(7, 1, 8, 4096, 128, 20)
    with pytest.raises(awq.AwqError):
        awq.workspace_size(awq.OP_SCALE_SEARCH, 1, 8, 4096, 96, 20)
    with pytest.raises(awq.AwqError):
        awq.workspace_size(awq.OP_SCALE_SEARCH, 1, 8, 4096, 128, 33)


def _vp(v):
    return ctypes.c_void_p(v)


def test_host_validation_without_a_gpu():
    L = awq.lib()
    fake = 0x10000           # 16-byte aligned, never dereferenced on the host
    odd = 0x10004
    # act_stats
    assert L.awq_act_stats(None, 4, 8, 8, fake, fake, 1 << 20, None) == 1
    assert L.awq_act_stats(fake, 0, 8, 8, fake, fake, 1 << 20, None) == 1
    assert L.awq_act_stats(fake, 4, 12, 12, fake, fake, 1 << 20, None) == 3
    assert L.awq_act_stats(odd, 4, 8, 8, fake, fake, 1 << 20, None) == 3
    assert L.awq_act_stats(fake, 1 << 24, 8, 8, fake, None, 0, None) == 1
    assert L.awq_act_stats(fake, 4, 8, 8, fake, odd, 0, None) == 3
    # scale_search
    W = (ctypes.c_void_p * 1)(fake)
    d = (ctypes.c_int64 * 1)(64)
    args = dict(n=1, W=W, d=d, d_in=256, x=fake, g=128, n_grid=20, flags=0)

    def search(**kw):
        a = dict(args, **kw)
        return L.awq_scale_search(a["n"], a["W"], a["d"], a["d_in"], a["x"], a["g"],
                                  a["n_grid"], a["flags"], fake, fake, fake, fake,
                                  1 << 24, None)
    assert search(n=0) == 1
    assert search(n=9) == 1
    assert search(g=96) == 2
    assert search(n_grid=0) == 1 and search(n_grid=33) == 1
    assert search(flags=8) == 1                      # an unknown flag bit
    assert search(flags=2, d_in=32768) == 2           # duo scaling: d_in <= 16384
    assert search(d_in=200) == 1
    assert search(W=(ctypes.c_void_p * 1)(odd)) == 3
    assert search(d=(ctypes.c_int64 * 1)(0)) == 1
    assert L.awq_scale_search(1, W, d, 256, fake, 128, 20, 0, fake, fake, fake, fake,
                              16, None) == 4
    plain = awq.workspace_size(awq.OP_SCALE_SEARCH, 1, 64, 256, 128, 20)
    duo = awq.workspace_size(awq.OP_SCALE_SEARCH_DUO, 1, 64, 256, 128, 20)
    assert duo > plain
    assert L.awq_scale_search(1, W, d, 256, fake, 128, 20, 2, fake, fake, fake, fake,
                              plain, None) == 4
    # quantize_pack
    assert L.awq_quantize_pack(fake, 12, 256, None, None, 128, 8, fake, fake, fake, None) == 1
    assert L.awq_quantize_pack(fake, 64, 256, None, None, 128, 9, fake, fake, fake, None) == 1
    assert L.awq_quantize_pack(fake, 64, 256, None, None, 48, 8, fake, fake, fake, None) == 2
    assert L.awq_quantize_pack(fake, 64, 256, odd, None, 128, 8, fake, fake, fake, None) == 3
    assert L.awq_quantize_pack(fake, 64, 256, None, None, 128, -2, fake, fake, fake, None) == 1
    assert L.awq_quantize_pack(fake, 64, 256, None, fake, 128, -1, fake, fake, fake,
                               None) == 2              # no clipping on the asymmetric grid
    # norm_group_scale
    ptrs1 = (ctypes.c_void_p * 1)(fake)
    ptrs_odd = (ctypes.c_void_p * 2)(fake, odd)
    assert L.awq_norm_group_scale(0, ptrs1, 256, fake, None) == 1
    assert L.awq_norm_group_scale(9, ptrs1, 256, fake, None) == 1
    assert L.awq_norm_group_scale(2, ptrs_odd, 256, fake, None) == 3
    assert L.awq_norm_group_scale(1, ptrs1, 256, odd, None) == 3
    # clip_search
    assert L.awq_clip_search(fake, 64, 256, fake, None, 128, 0, 0, fake, fake, fake,
                             1 << 20, None) == 1
    assert L.awq_clip_search(fake, 64, 256, fake, None, 128, 21, 0, fake, fake, fake,
                             1 << 20, None) == 1
    assert L.awq_clip_search(fake, 64, 256, fake, None, 48, 10, 0, fake, fake, fake,
                             1 << 20, None) == 2
    assert L.awq_clip_search(fake, 64, 200, fake, None, 128, 10, 0, fake, fake, fake,
                             1 << 20, None) == 1
    assert L.awq_clip_search(fake, 64, 256, fake, odd, 128, 10, 0, fake, fake, fake,
                             1 << 20, None) == 3
    assert L.awq_clip_search(fake, 64, 256, fake, None, 128, 10, 0, fake, fake, fake,
                             64, None) == 4
    # output_error
    assert L.awq_output_error(fake, 0, fake, 64, 256, fake, 128, 20, 0, fake, fake,
                              None, fake, 1 << 30, None) == 1
    assert L.awq_output_error(fake, 16, fake, 64, 256, fake, 128, 20, 0, fake, fake,
                              None, fake, 16, None) == 4
    assert L.awq_output_error(fake, 16, fake, 64, 256, fake, 128, 20, 0, fake, fake,
                              odd, fake, 1 << 30, None) == 3


def test_pipeline_workspace_sizes_from_host_query():
    """GroupJob sizes its workspaces through awq_workspace_size (a host-only
    call): the weight-space and output-space searches of the same group."""
    import torch
    from post_int4_weight_b200 import pipeline
    Ws = [torch.zeros(256, 512, dtype=torch.float16), torch.zeros(128, 512, dtype=torch.float16)]
    X = torch.zeros(64, 512, dtype=torch.float16)
    j = pipeline.GroupJob(Ws, X, 128, 20)
    st, se, cl = j.workspace_bytes()
    assert st >= 0 and se > 0 and cl == 0
    jo = pipeline.GroupJob(Ws[:1], X, 128, 20, output_mode=True)
    st_o, se_o, _ = jo.workspace_bytes()
    assert se_o >= 2 * 256 * 512 * 2            # the hi/lo dW buffer at least
    jc = pipeline.GroupJob(Ws, X, 128, 20, n_clip=10)
    assert jc.workspace_bytes()[2] > 0
    # stats 1; search 2 (table, search); output mode 1 + 2 * 20 + 1; clip 2 per
    # member ((x / s)^2, search), 3 in output space (Gram slices, their sum,
    # scoring); pack 1 per member
    assert j.launches == 1 + 2 + 2 and jo.launches == 1 + 42 + 1
    assert jc.launches == 1 + 2 + 2 * 2 + 2
    jco = pipeline.GroupJob(Ws, X, 128, 20, n_clip=10, clip_space="output")
    assert jco.launches == 1 + 2 + 2 * 3 + 2
    ws = pipeline.Workspaces([j, jo, jc], "cpu")
    assert ws.search.numel() == max(se, se_o)


def test_duo_workspace_growth_and_noalloc_limit():
    """The duo workspace adds, to the plain search's, one fp64 column-sum row
    per weight-mean CTA, the fp64 candidates of every grid point and their
    per-block extremes; it grows with d_in and n_grid.  The no-alloc entry's
    4 MiB scratch holds the duo search up to d_in 2048 at 20 grid points
    (the limit include/awq.h states) and not at 4096."""
    def duo(d_in, n_grid):
        return awq.workspace_size(awq.OP_SCALE_SEARCH_DUO, 1, 8, d_in, 128, n_grid)

    def plain(d_in, n_grid):
        return awq.workspace_size(awq.OP_SCALE_SEARCH, 1, 8, d_in, 128, n_grid)

    for d_in in (512, 2048, 4096, 16384):
        extra = duo(d_in, 20) - plain(d_in, 20)
        assert extra >= 148 * d_in * 8 + 20 * d_in * 8
        assert duo(d_in, 32) > duo(d_in, 20)
    assert duo(2048, 20) <= 4 << 20 < duo(4096, 20)
    with pytest.raises(awq.AwqError):
        duo(16384 + 128, 20)                    # beyond the weight-mean pass's 16384
