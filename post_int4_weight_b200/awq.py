"""Python binding of libawq_b200.so (the C ABI of include/awq.h).

Argument marshalling only: every step of the path runs in the library's CUDA
kernels.  Tensors are ``torch`` CUDA tensors; PyTorch provides the device
memory and the stream (the current stream of the tensors' device).  There is
no CPU fallback: without the built library or a CUDA device these functions
raise.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence, Tuple

import torch

from . import build as _build

SCALE_FP16 = 0
SCALE_FP32 = 1
OP_ACT_STATS = 0
OP_SCALE_SEARCH = 1
OP_OUTPUT_ERROR = 2
OP_CLIP_SEARCH = 3
OP_SCALE_SEARCH_DUO = 4
OP_CLIP_SEARCH_OUTPUT = 5
DUO_SCALING = 2
ASYMMETRIC = 4
ZERO_POINT_ASYM = -1
# test hook of scale_search: one weight load that never completes (see
# AWQ_TEST_STALL_WAIT in include/awq.h); only for the failure-path test
TEST_STALL_WAIT = 0x40000000
CLIP_DEN = 20
MAX_SEGMENTS = 8
# sticky device-side condition bits (awq_last_device_flags)
FLAG_NONFINITE_X = 0x1
FLAG_NONFINITE_SCORE = 0x2
FLAG_NONFINITE_GROUP = 0x4
FLAG_NONFINITE_SCALE = 0x8
FLAG_WAIT_TIMEOUT = 0x10

LIB_PATH = _build.LIB

_lib = None


class AwqError(RuntimeError):
    """A non-zero awq_status returned by the library."""

    def __init__(self, status: int, where: str):
        self.status = status
        detail = ""
        if status == 5:   # AWQ_ERR_CUDA
            detail = " [" + lib().awq_last_error().decode() + "]"
        super().__init__(f"{where}: {string(status)}{detail}")


def lib() -> ctypes.CDLL:
    """Load the library (building it first if it is missing or stale)."""
    global _lib
    if _lib is None:
        if not _build.up_to_date():
            _build.build()
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"CUDA library missing: {LIB_PATH}")
        L = ctypes.CDLL(LIB_PATH)
        i32, i64, sz = ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
        p = ctypes.c_void_p
        L.awq_status_string.argtypes = [i32]
        L.awq_status_string.restype = ctypes.c_char_p
        L.awq_abi_version.restype = i32
        L.awq_last_error.restype = ctypes.c_char_p
        L.awq_workspace_size.argtypes = [i32, i64, i64, i64, i32, i32, ctypes.POINTER(sz)]
        L.awq_workspace_size.restype = i32
        L.awq_act_stats.argtypes = [p, i64, i64, i64, p, p, sz, p]
        L.awq_act_stats.restype = i32
        L.awq_scale_search.argtypes = [i32, p, p, i64, p, i32, i32, i32, p, p, p, p, sz, p]
        L.awq_scale_search.restype = i32
        L.awq_quantize_pack.argtypes = [p, i64, i64, p, p, i32, i32, p, p, p, p]
        L.awq_quantize_pack.restype = i32
        L.awq_clip_search.argtypes = [p, i64, i64, p, p, i32, i32, i32, p, p, p, sz, p]
        L.awq_clip_search.restype = i32
        L.awq_norm_group_scale.argtypes = [i32, p, i64, p, p]
        L.awq_norm_group_scale.restype = i32
        L.awq_clip_search.restype = i32
        L.awq_output_error.argtypes = [p, i64, p, i64, i64, p, i32, i32, i32, p, p, p, p, sz, p]
        L.awq_output_error.restype = i32
        L.awq_clip_search_output.argtypes = [p, i64, i64, p, i64, i64, p, i32, i32, i32, p, p,
                                             p, sz, p]
        L.awq_clip_search_output.restype = i32
        L.awq_last_device_flags.argtypes = [ctypes.POINTER(ctypes.c_uint32), i32]
        L.awq_last_device_flags.restype = i32
        _lib = L
    return _lib


def string(status: int) -> str:
    return lib().awq_status_string(int(status)).decode()


def _check(status: int, where: str):
    if status != 0:
        raise AwqError(status, where)


def _cuda(t: torch.Tensor, dtype, name: str) -> torch.Tensor:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def _stream(device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def last_device_flags(clear: bool = True) -> Tuple[int, int]:
    """awq_last_device_flags on the current device: (status, AWQ_FLAG_* bits
    raised since the last clearing read).  Synchronises the device.  Status 6
    (AWQ_ERR_NONFINITE) and 7 (AWQ_ERR_DEVICE_TIMEOUT) are returned, not
    raised; any other non-zero status raises AwqError."""
    bits = ctypes.c_uint32(0)
    st = lib().awq_last_device_flags(ctypes.byref(bits), 1 if clear else 0)
    if st not in (0, 6, 7):
        raise AwqError(st, "awq_last_device_flags")
    return st, int(bits.value)


def workspace_size(op: int, T: int, d_out_total: int, d_in: int, group_size: int,
                   n_grid: int) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().awq_workspace_size(op, T, d_out_total, d_in, group_size, n_grid,
                                    ctypes.byref(n)), "awq_workspace_size")
    return int(n.value)


def workspace(op: int, device, T: int = 1, d_out_total: int = 8, d_in: int = 128,
              group_size: int = 128, n_grid: int = 20) -> torch.Tensor:
    n = workspace_size(op, T, d_out_total, d_in, group_size, n_grid)
    return torch.empty(max(n, 1), dtype=torch.uint8, device=device)


def act_stats(X: torch.Tensor, out: Optional[torch.Tensor] = None,
              ws: Optional[torch.Tensor] = None) -> torch.Tensor:
    """x[j] = mean_t |X[t, j]| (exact mean, fp32) of fp16 X [T, d_in]."""
    _cuda(X, torch.float16, "X")
    T, d_in = X.shape
    if out is None:
        out = torch.empty(d_in, dtype=torch.float32, device=X.device)
    if ws is None:
        ws = workspace(OP_ACT_STATS, X.device, T, 8, d_in)
    _check(lib().awq_act_stats(X.data_ptr(), T, d_in, d_in, out.data_ptr(),
                               ws.data_ptr(), ws.numel(), _stream(X.device)),
           "awq_act_stats")
    return out


def scale_search(Ws: Sequence[torch.Tensor], x: torch.Tensor, group_size: int = 128,
                 n_grid: int = 20, flags: int = SCALE_FP16,
                 out: Optional[Tuple[torch.Tensor, torch.Tensor, torch.Tensor]] = None,
                 ws: Optional[torch.Tensor] = None):
    """Fused alpha-grid search over weight segments sharing input x.

    Returns (err fp64[n_grid], best_idx int32[1], s_best fp32[d_in]), all on
    the device (no synchronisation)."""
    Ws = [_cuda(W, torch.float16, "W") for W in Ws]
    _cuda(x, torch.float32, "x")
    d_in = x.shape[0]
    for W in Ws:
        if W.dim() != 2 or W.shape[1] != d_in:
            raise ValueError("every W must be [d_out, d_in] with d_in = len(x)")
    dev = x.device
    if out is None:
        out = (torch.empty(n_grid, dtype=torch.float64, device=dev),
               torch.empty(1, dtype=torch.int32, device=dev),
               torch.empty(d_in, dtype=torch.float32, device=dev))
    err, best, s_best = out
    if ws is None:
        op = OP_SCALE_SEARCH_DUO if flags & DUO_SCALING else OP_SCALE_SEARCH
        ws = workspace(op, dev, 1, 8, d_in, group_size, n_grid)
    n = len(Ws)
    ptrs = (ctypes.c_void_p * n)(*[W.data_ptr() for W in Ws])
    d_out = (ctypes.c_int64 * n)(*[W.shape[0] for W in Ws])
    _check(lib().awq_scale_search(n, ptrs, d_out, d_in, x.data_ptr(), group_size, n_grid,
                                  flags, err.data_ptr(), best.data_ptr(), s_best.data_ptr(),
                                  ws.data_ptr(), ws.numel(), _stream(dev)),
           "awq_scale_search")
    return err, best, s_best


def quantize_pack(W: torch.Tensor, s: Optional[torch.Tensor] = None, group_size: int = 128,
                  zero_point: int = 8, out=None, clip_idx: Optional[torch.Tensor] = None):
    """AutoAWQ GEMM packing: (qweight int32 [d_in, d_out/8],
    scales fp16 [d_in/g, d_out], qzeros int32 [d_in/g, d_out/8]).
    clip_idx: optional uint8 [d_out, d_in/g] from clip_search."""
    _cuda(W, torch.float16, "W")
    d_out, d_in = W.shape
    if s is not None:
        _cuda(s, torch.float32, "s")
    if clip_idx is not None:
        _cuda(clip_idx, torch.uint8, "clip_idx")
        if tuple(clip_idx.shape) != (d_out, d_in // group_size):
            raise ValueError("clip_idx must be [d_out, d_in / group_size]")
    dev = W.device
    G = d_in // group_size
    if out is None:
        out = (torch.empty(d_in, d_out // 8, dtype=torch.int32, device=dev),
               torch.empty(G, d_out, dtype=torch.float16, device=dev),
               torch.empty(G, d_out // 8, dtype=torch.int32, device=dev))
    qw, sc, qz = out
    _check(lib().awq_quantize_pack(W.data_ptr(), d_out, d_in,
                                   None if s is None else s.data_ptr(),
                                   None if clip_idx is None else clip_idx.data_ptr(),
                                   group_size, zero_point, qw.data_ptr(), sc.data_ptr(),
                                   qz.data_ptr(), _stream(dev)),
           "awq_quantize_pack")
    return qw, sc, qz


def norm_group_scale(ss: Sequence[torch.Tensor], out: Optional[torch.Tensor] = None):
    """Per-channel geometric mean of the member linears' scales (fp32)."""
    ss = [_cuda(x, torch.float32, "s") for x in ss]
    d_in = ss[0].shape[0]
    for x in ss:
        if x.dim() != 1 or x.shape[0] != d_in:
            raise ValueError("every scale must be [d_in]")
    dev = ss[0].device
    if out is None:
        out = torch.empty(d_in, dtype=torch.float32, device=dev)
    n = len(ss)
    ptrs = (ctypes.c_void_p * n)(*[x.data_ptr() for x in ss])
    _check(lib().awq_norm_group_scale(n, ptrs, d_in, out.data_ptr(), _stream(dev)),
           "awq_norm_group_scale")
    return out


def clip_search(W: torch.Tensor, x: torch.Tensor, s: Optional[torch.Tensor] = None,
                group_size: int = 128, n_clip: int = 10, flags: int = SCALE_FP16,
                out: Optional[Tuple[torch.Tensor, torch.Tensor]] = None,
                ws: Optional[torch.Tensor] = None):
    """Per (row, group) clip ratio search at scale s: (clip_idx uint8
    [d_out, d_in/g], err fp64[2] = (no clipping, chosen ratios))."""
    _cuda(W, torch.float16, "W")
    _cuda(x, torch.float32, "x")
    if s is not None:
        _cuda(s, torch.float32, "s")
    d_out, d_in = W.shape
    dev = W.device
    if out is None:
        out = (torch.empty(d_out, d_in // group_size, dtype=torch.uint8, device=dev),
               torch.empty(2, dtype=torch.float64, device=dev))
    idx, err = out
    if ws is None:
        ws = workspace(OP_CLIP_SEARCH, dev, 1, d_out, d_in, group_size, 1)
    _check(lib().awq_clip_search(W.data_ptr(), d_out, d_in, x.data_ptr(),
                                 None if s is None else s.data_ptr(), group_size, n_clip, flags,
                                 idx.data_ptr(), err.data_ptr(), ws.data_ptr(), ws.numel(),
                                 _stream(dev)),
           "awq_clip_search")
    return idx, err


def clip_search_output(X: torch.Tensor, W: torch.Tensor, s: Optional[torch.Tensor] = None,
                       group_size: int = 128, n_clip: int = 10, flags: int = SCALE_FP16,
                       out: Optional[Tuple[torch.Tensor, torch.Tensor]] = None,
                       ws: Optional[torch.Tensor] = None):
    """Clip search scored in output space (each group's share of
    ||X (W - W_hat)^T||^2): (clip_idx uint8 [d_out, d_in/g], err fp64[2])."""
    _cuda(X, torch.float16, "X")
    _cuda(W, torch.float16, "W")
    if s is not None:
        _cuda(s, torch.float32, "s")
    T, d_in = X.shape
    d_out = W.shape[0]
    dev = W.device
    if out is None:
        out = (torch.empty(d_out, d_in // group_size, dtype=torch.uint8, device=dev),
               torch.empty(2, dtype=torch.float64, device=dev))
    idx, err = out
    if ws is None:
        ws = workspace(OP_CLIP_SEARCH_OUTPUT, dev, T, d_out, d_in, group_size, 1)
    _check(lib().awq_clip_search_output(X.data_ptr(), T, d_in, W.data_ptr(), d_out, d_in,
                                        None if s is None else s.data_ptr(), group_size, n_clip,
                                        flags, idx.data_ptr(), err.data_ptr(), ws.data_ptr(),
                                        ws.numel(), _stream(dev)),
           "awq_clip_search_output")
    return idx, err


def output_error(X: torch.Tensor, W: torch.Tensor, x: torch.Tensor, group_size: int = 128,
                 n_grid: int = 20, flags: int = SCALE_FP16,
                 out: Optional[Tuple[torch.Tensor, torch.Tensor, torch.Tensor]] = None,
                 ws: Optional[torch.Tensor] = None):
    """Output-space score ||X (W - W_hat_i)^T||^2 per grid point:
    (err fp64[n_grid], best_idx int32[1], s_best fp32[d_in])."""
    _cuda(X, torch.float16, "X")
    _cuda(W, torch.float16, "W")
    _cuda(x, torch.float32, "x")
    T, d_in = X.shape
    d_out = W.shape[0]
    dev = X.device
    if out is None:
        out = (torch.empty(n_grid, dtype=torch.float64, device=dev),
               torch.empty(1, dtype=torch.int32, device=dev),
               torch.empty(d_in, dtype=torch.float32, device=dev))
    err, best, s_best = out
    if ws is None:
        ws = workspace(OP_OUTPUT_ERROR, dev, T, d_out, d_in, group_size, n_grid)
    _check(lib().awq_output_error(X.data_ptr(), T, W.data_ptr(), d_out, d_in, x.data_ptr(),
                                  group_size, n_grid, flags, err.data_ptr(), best.data_ptr(),
                                  s_best.data_ptr(), ws.data_ptr(), ws.numel(), _stream(dev)),
           "awq_output_error")
    return err, best, s_best


def quantize_group(Ws: Sequence[torch.Tensor], X: torch.Tensor, group_size: int = 128,
                   n_grid: int = 20, zero_point: int = 8):
    """The whole hot path for linears sharing the input X: activation stats,
    the fused scale search, then quantise-and-pack of every member with the
    chosen scale.  Returns (err, best_idx, s_best, [(qweight, scales, qzeros)])
    on the device."""
    x = act_stats(X)
    err, best, s_best = scale_search(Ws, x, group_size, n_grid)
    packed = [quantize_pack(W, s_best, group_size, zero_point) for W in Ws]
    return err, best, s_best, packed


_noalloc_fn = None


def _noalloc_entry():
    """ctypes handle of awq_scale_search_noalloc with its argument types."""
    global _noalloc_fn
    if _noalloc_fn is None:
        fn = lib().awq_scale_search_noalloc
        p = ctypes.c_void_p
        fn.argtypes = [ctypes.c_int, p, p, ctypes.c_int64, p, ctypes.c_int, ctypes.c_int,
                       ctypes.c_int, p, p, p, p]
        fn.restype = ctypes.c_int
        _noalloc_fn = fn
    return _noalloc_fn


def scale_search_noalloc(Ws: Sequence[torch.Tensor], x: torch.Tensor, group_size: int = 128,
                         n_grid: int = 20, flags: int = SCALE_FP16):
    """awq_scale_search_noalloc: the same search with the library's static
    per-device scratch instead of a caller workspace.  Only the outputs are
    allocated here (by torch); the library allocates nothing."""
    fn = _noalloc_entry()
    Ws = [_cuda(W, torch.float16, "W") for W in Ws]
    _cuda(x, torch.float32, "x")
    d_in = x.shape[0]
    dev = x.device
    err = torch.empty(n_grid, dtype=torch.float64, device=dev)
    best = torch.empty(1, dtype=torch.int32, device=dev)
    s_best = torch.empty(d_in, dtype=torch.float32, device=dev)
    n = len(Ws)
    ptrs = (ctypes.c_void_p * n)(*[W.data_ptr() for W in Ws])
    d_out = (ctypes.c_int64 * n)(*[W.shape[0] for W in Ws])
    _check(fn(n, ptrs, d_out, d_in, x.data_ptr(), group_size, n_grid, flags,
              err.data_ptr(), best.data_ptr(), s_best.data_ptr(), _stream(dev)),
           "awq_scale_search_noalloc")
    return err, best, s_best
