"""CPU oracle for the AWQ INT4 hot path -- TEST INFRASTRUCTURE ONLY.

Plain numpy wrappers around ``awq_oracle.c`` (built on first use into
``oracle/liborc.so``).  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  The CUDA library in ``post_int4_weight_b200`` neither imports nor
links it, and this package imports nothing from there.

Every array argument is a numpy array; fp16 tensors are passed as
``np.float16`` (their bit patterns go to C as ``uint16``).
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

SCALE_FP32 = 1  # keep the group scale unrounded (fp32) instead of fp16
DUO = 2         # duo scaling candidates in the scale search
ASYM = 4        # asymmetric INT4 (16 levels, per-group zero point)

_lib = None


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        i64, i32, f64 = ctypes.c_int64, ctypes.c_int, ctypes.c_double
        p = ctypes.c_void_p
        lib.orc_act_stats.argtypes = [p, i64, i64, i64, p]
        lib.orc_scale_table.argtypes = [p, i64, i32, p]
        lib.orc_fake_quant_group.argtypes = [p, p, i64, i32, p, p]
        lib.orc_fake_quant_group.restype = i32
        lib.orc_weighted_error.argtypes = [p, i64, i64, p, p, i64, i32]
        lib.orc_weighted_error.restype = f64
        lib.orc_scale_search.argtypes = [i32, p, p, i64, p, i64, i32, i32, p, p, p]
        lib.orc_quantize_pack.argtypes = [p, i64, i64, p, p, i64, i32, p, p, p]
        lib.orc_geomean_scales.argtypes = [i32, p, i64, p]
        lib.orc_fake_quant_group_asym.argtypes = [p, p, i64, i32, p, p, p]
        lib.orc_fake_quant_group_asym.restype = i32
        lib.orc_weight_mean.argtypes = [i32, p, p, i64, p]
        lib.orc_scale_table_duo.argtypes = [p, p, i64, i32, p]
        lib.orc_clip_ratio.argtypes = [i32]
        lib.orc_clip_ratio.restype = ctypes.c_float
        lib.orc_fake_quant_group_clip.argtypes = [p, p, i64, i32, ctypes.c_float, p, p]
        lib.orc_fake_quant_group_clip.restype = i32
        lib.orc_clip_group_error.argtypes = [p, p, p, i64, i32, ctypes.c_float]
        lib.orc_clip_group_error.restype = f64
        lib.orc_clip_search.argtypes = [p, i64, i64, p, p, i64, i32, i32, p, p]
        lib.orc_clip_search_output.argtypes = [p, i64, p, i64, i64, p, i64, i32, i32, p, p]
        lib.orc_unpack.argtypes = [p, i64, i64, p]
        lib.orc_output_error.argtypes = [p, i64, p, i64, i64, p, i64, i32, i32, p]
        _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _f16(a) -> np.ndarray:
    a = np.ascontiguousarray(a, dtype=np.float16)
    return a


def _f32(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float32)


def act_stats(X) -> np.ndarray:
    """x[j] = mean_t |X[t, j]| (exact, rounded once to fp32)."""
    X = _f16(X)
    T, d_in = X.shape
    x = np.empty(d_in, np.float32)
    _load().orc_act_stats(_ptr(X), T, d_in, d_in, _ptr(x))
    return x


def scale_table(x, n_grid: int = 20) -> np.ndarray:
    """S[i, j] = max(x_j,1e-4)^(i/n_grid) / sqrt(max_j * min_j), fp32."""
    x = _f32(x)
    S = np.empty((n_grid, x.shape[0]), np.float32)
    _load().orc_scale_table(_ptr(x), x.shape[0], n_grid, _ptr(S))
    return S


def fake_quant_group(w, s, flags: int = 0):
    """Codes and group scale of one group: returns (q int8[n], q_scale float)."""
    w, s = _f32(w), _f32(s)
    q = np.empty(w.shape[0], np.int8)
    qs = np.empty(1, np.float32)
    bad = _load().orc_fake_quant_group(_ptr(w), _ptr(s), w.shape[0], flags,
                                       _ptr(q), _ptr(qs))
    return q, float(qs[0]), bool(bad)


def weighted_error(W, x, s, group_size: int, flags: int = 0) -> float:
    W = _f16(W)
    x, s = _f32(x), _f32(s)
    d_out, d_in = W.shape
    return _load().orc_weighted_error(_ptr(W), d_out, d_in, _ptr(x), _ptr(s),
                                      group_size, flags)


def scale_search(Ws, x, group_size: int = 128, n_grid: int = 20, flags: int = 0):
    """Grid search over alpha for weight segments sharing the input x.

    Returns (err float64[n_grid], best_idx int, s_best float32[d_in]).
    """
    Ws = [_f16(W) for W in Ws]
    x = _f32(x)
    d_in = x.shape[0]
    n_seg = len(Ws)
    ptrs = (ctypes.c_void_p * n_seg)(*[W.ctypes.data for W in Ws])
    d_out = (ctypes.c_int64 * n_seg)(*[W.shape[0] for W in Ws])
    err = np.empty(n_grid, np.float64)
    best = np.empty(1, np.int32)
    s_best = np.empty(d_in, np.float32)
    _load().orc_scale_search(n_seg, ptrs, d_out, d_in, _ptr(x), group_size,
                             n_grid, flags, _ptr(err), _ptr(best), _ptr(s_best))
    return err, int(best[0]), s_best


def quantize_pack(W, s=None, group_size: int = 128, zero_point: int = 8, clip_idx=None):
    """AutoAWQ GEMM layout: (qweight int32[d_in, d_out/8],
    scales fp16[d_in/g, d_out], qzeros int32[d_in/g, d_out/8]).
    clip_idx: optional uint8 [d_out, d_in/g] clip ratio indices."""
    W = _f16(W)
    d_out, d_in = W.shape
    G = d_in // group_size
    qweight = np.empty((d_in, d_out // 8), np.int32)
    scales = np.empty((G, d_out), np.float16)
    qzeros = np.empty((G, d_out // 8), np.int32)
    s_arr = None if s is None else _f32(s)
    c_arr = None if clip_idx is None else np.ascontiguousarray(clip_idx, dtype=np.uint8)
    if c_arr is not None and c_arr.shape != (d_out, G):
        raise ValueError("clip_idx must be [d_out, d_in / group_size]")
    _load().orc_quantize_pack(_ptr(W), d_out, d_in,
                              None if s_arr is None else _ptr(s_arr),
                              None if c_arr is None else _ptr(c_arr),
                              group_size, zero_point, _ptr(qweight),
                              _ptr(scales), _ptr(qzeros))
    return qweight, scales, qzeros


def fake_quant_group_asym(w, s, flags: int = 0):
    """Asymmetric INT4 of one group: (codes uint8 0..15, q_scale, zero point)."""
    w, s = _f32(w), _f32(s)
    q = np.empty(w.shape[0], np.uint8)
    qs = np.empty(1, np.float32)
    z = np.empty(1, np.int32)
    _load().orc_fake_quant_group_asym(_ptr(w), _ptr(s), w.shape[0], flags, _ptr(q), _ptr(qs),
                                      _ptr(z))
    return q, float(qs[0]), int(z[0])


def weight_mean(Ws) -> np.ndarray:
    """Duo scaling's per-channel mean of |w| / (row max |w|), fp64 [d_in]."""
    Ws = [_f16(W) for W in Ws]
    d_in = Ws[0].shape[1]
    ptrs = (ctypes.c_void_p * len(Ws))(*[W.ctypes.data for W in Ws])
    d_out = (ctypes.c_int64 * len(Ws))(*[W.shape[0] for W in Ws])
    out = np.empty(d_in, np.float64)
    _load().orc_weight_mean(len(Ws), ptrs, d_out, d_in, _ptr(out))
    return out


def scale_table_duo(x, w_mean, n_grid: int = 20) -> np.ndarray:
    """Duo scale table S[i, j] (fp32) from x and the fp64 weight mean."""
    x = _f32(x)
    w_mean = np.ascontiguousarray(w_mean, dtype=np.float64)
    S = np.empty((n_grid, x.shape[0]), np.float32)
    _load().orc_scale_table_duo(_ptr(x), _ptr(w_mean), x.shape[0], n_grid, _ptr(S))
    return S


def geomean_scales(ss) -> np.ndarray:
    """Per-channel geometric mean of the member linears' scales (fp32)."""
    ss = [_f32(x) for x in ss]
    d_in = ss[0].shape[0]
    ptrs = (ctypes.c_void_p * len(ss))(*[x.ctypes.data for x in ss])
    out = np.empty(d_in, np.float32)
    _load().orc_geomean_scales(len(ss), ptrs, d_in, _ptr(out))
    return out


def clip_ratio(i: int) -> float:
    """Clip ratio of grid index i: (20 - i) / 20 rounded to fp32."""
    return float(_load().orc_clip_ratio(int(i)))


def fake_quant_group_clip(w, s, c: float, flags: int = 0):
    """Codes and group scale of one group with the range shrunk to c*max|ws|."""
    w, s = _f32(w), _f32(s)
    q = np.empty(w.shape[0], np.int8)
    qs = np.empty(1, np.float32)
    _load().orc_fake_quant_group_clip(_ptr(w), _ptr(s), w.shape[0], flags,
                                      ctypes.c_float(c), _ptr(q), _ptr(qs))
    return q, float(qs[0])


def clip_group_error(w, s, x, c: float, flags: int = 0) -> float:
    """Weighted error of one group at clip ratio c (fp64)."""
    w, s, x = _f32(w), _f32(s), _f32(x)
    return float(_load().orc_clip_group_error(_ptr(w), _ptr(s), _ptr(x), w.shape[0],
                                              flags, ctypes.c_float(c)))


def clip_search(W, x, s=None, group_size: int = 128, n_clip: int = 10, flags: int = 0):
    """Per (row, group) clip ratio index (uint8 [d_out, d_in/g]) and the
    totals (error without clipping, error with the chosen ratios)."""
    W = _f16(W)
    x = _f32(x)
    d_out, d_in = W.shape
    G = d_in // group_size
    idx = np.empty((d_out, G), np.uint8)
    err = np.empty(2, np.float64)
    s_arr = None if s is None else _f32(s)
    _load().orc_clip_search(_ptr(W), d_out, d_in, _ptr(x),
                            None if s_arr is None else _ptr(s_arr), group_size, n_clip,
                            flags, _ptr(idx), _ptr(err))
    return idx, err


def clip_search_output(X, W, s=None, group_size: int = 128, n_clip: int = 10,
                       flags: int = 0):
    """Output-space clip search: per (row, group) the ratio index minimising
    sum_t (X[t, group] . (w - w_hat_clip))^2 (uint8 [d_out, d_in/g]) and the
    totals (no clipping, chosen ratios) of those per-group errors."""
    X, W = _f16(X), _f16(W)
    T, d_in = X.shape
    d_out = W.shape[0]
    G = d_in // group_size
    idx = np.empty((d_out, G), np.uint8)
    err = np.empty(2, np.float64)
    s_arr = None if s is None else _f32(s)
    _load().orc_clip_search_output(_ptr(X), T, _ptr(W), d_out, d_in,
                                   None if s_arr is None else _ptr(s_arr), group_size,
                                   n_clip, flags, _ptr(idx), _ptr(err))
    return idx, err


def unpack(qweight, d_out: int) -> np.ndarray:
    """Unsigned codes u[d_out, d_in] from the packed words."""
    qweight = np.ascontiguousarray(qweight, dtype=np.int32)
    d_in = qweight.shape[0]
    u = np.empty((d_out, d_in), np.uint8)
    _load().orc_unpack(_ptr(qweight), d_out, d_in, _ptr(u))
    return u


def output_error(X, W, x, group_size: int = 128, n_grid: int = 20,
                 flags: int = 0) -> np.ndarray:
    """err[i] = ||X (W - W_hat_i)^T||_F^2 in fp64 (small shapes only)."""
    X, W = _f16(X), _f16(W)
    x = _f32(x)
    T, d_in = X.shape
    d_out = W.shape[0]
    err = np.empty(n_grid, np.float64)
    _load().orc_output_error(_ptr(X), T, _ptr(W), d_out, d_in, _ptr(x),
                             group_size, n_grid, flags, _ptr(err))
    return err


def threads() -> int:
    """Threads the OpenMP parts of the oracle use on this host."""
    return int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
