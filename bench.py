#!/usr/bin/env python
"""Benchmark of the AWQ INT4 hot path (activation stats + fused alpha-grid
scale search + quantise-and-pack) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--group-size G]

One step = one pass of the whole hot path over the workload: for every
search group (linears sharing one input), awq_act_stats on its X,
awq_scale_search over the 20-point alpha grid (or awq_output_error for the
output-space workload), and awq_quantize_pack of every member at the chosen
scale.  Workloads (post_int4_weight_b200/workloads.py):

  q_proj_4096x4096        (default) one 4096x4096 linear, 4096 tokens, g128
  qwen3_8b_block          one decoder block, 7 linears in 4 groups, 16384
                          tokens, g128 (or --group-size 64)
  down_proj_output_error  4096x12288 down_proj scored in output space,
                          8192 tokens, on the tensor cores
  qwen3_8b_stack36        36 such blocks (6.95 B weights), 2048 tokens per
                          layer, streamed layer by layer

Inputs are seeded synthetic and resident in HBM when the timed region
starts.  Workloads whose inputs fit in the 126 MB L2 get a 256 MB buffer
written between timed steps (outside the per-step CUDA events); larger ones
are not flushed.  The end-to-end number ("e2e") streams the same work from
pinned host memory: copies in, kernels, results out, overlapped layer by
layer on three streams.

Scaling: one-layer workloads give every rank its own independent layer (weak
scaling); the 36-layer stack is split over the ranks by layer (strong
scaling).  No data-path collective either way; the time is the max over
ranks.

Prints one JSON line (rank 0).  --impl reference times the CPU oracle on the
host cores instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "AWQ search+pack Gparam/s per layer"
UNIT = "Gparam/s"
# Algorithmic work of the search per (weight, alpha) pair, as the scope of the
# path counts it (an FMA counts once): multiply w*s, |.| and max, divide by
# q_scale, round, two clamps, multiply q*q_scale, divide by s, subtract,
# multiply by x, square-accumulate.
ALG_OPS_PER_PAIR = 11
# FMA-pipe lane operations the search kernel actually executes per pair:
# w*s, the rounding addition and its removal, the residual, the square, and
# half of the weighted accumulate that a lane's two rows share -- reported
# beside it.
FMA_OPS_PER_PAIR = 5.5
# dram__bytes_read.sum + dram__bytes_write.sum of one launch of the dominant
# kernel from the committed ncu captures (profiles/), for the kernels as they
# stand; None where no capture of the current kernel exists.
# DRAM bytes (read + write) of one launch of the dominant kernel, from an ncu
# capture of the current kernel: (workload, asymmetric grid) -> bytes.
# (workload, asymmetric grid, group size) -> DRAM bytes of one launch of the
# dominant kernel, read + written, from one ncu capture of the current kernel
NCU_TRAFFIC = {("q_proj_4096x4096", False, 128): 34258432,        # search_kernel<8,0,0>
               ("q_proj_4096x4096", True, 128): 34260224,         # search_kernel<8,0,1>
               ("down_proj_output_error", False, 128): 1506610176}  # oe_gemm_kernel, per alpha
FP32_LANES_PER_SM = 128
HBM_SPEC_GBS = 8000.0     # the B200's HBM3e bandwidth as specified (the measured copy rate is the peak)
DEFAULT_STEPS = {"single_linear_256x512": 1000, "q_proj_4096x4096": 1000,
                 "qwen3_8b_block": 100, "down_proj_output_error": 10,
                 "qwen3_8b_stack36": 20}


def _args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None,
                    help="timed steps (default: about a second or more of work per workload)")
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="q_proj_4096x4096")
    ap.add_argument("--group-size", type=int, default=0,
                    help="group size (default: the workload's first)")
    ap.add_argument("--scale-mode", choices=["joint", "geomean"], default="joint",
                    help="joint: one search over a shared-input group's linears; geomean: "
                         "one search per linear, then their geometric mean (norm group)")
    ap.add_argument("--asym", action="store_true",
                    help="asymmetric INT4 grid (per-group zero points) in search and pack")
    ap.add_argument("--duo", action="store_true",
                    help="duo scaling candidates (weights' row-normalised mean) in the search")
    ap.add_argument("--clip", type=int, default=0,
                    help="also run the clip search with this many ratios per member "
                         "(0: off, the method's default path)")
    ap.add_argument("--clip-space", choices=["weight", "output"], default="weight",
                    help="score the clip search's ratios on the activation-weighted weight "
                         "error (weight) or on each group's share of the output error (output)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-graph", action="store_true",
                    help="launch each step eagerly instead of replaying a CUDA graph")
    a = ap.parse_args()
    if a.steps is None:
        a.steps = DEFAULT_STEPS.get(a.workload, 20)
    return a


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return json.load(f), "measured"
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "sm_max_mhz": 1965.0}, "fallback"


# ----------------------------------------------------------------- clocks --

class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML every 2 ms."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, torch_device):
        self.samples = []
        self.reasons = 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._h = None
        try:
            import pynvml as nv
            self.nv = nv
            nv.nvmlInit()
            props = __import__("torch").cuda.get_device_properties(torch_device)
            h = None
            uuid = getattr(props, "uuid", None)
            if uuid is not None:
                try:
                    h = nv.nvmlDeviceGetHandleByUUID(("GPU-" + str(uuid)).encode())
                except Exception:
                    h = None
            if h is None:
                h = nv.nvmlDeviceGetHandleByIndex(torch_device.index or 0)
            self._h = h
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
        except Exception:
            self._h = None

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                self.reasons |= int(nv.nvmlDeviceGetCurrentClocksEventReasons(self._h))
            except Exception:
                pass
            time.sleep(0.002)

    def __enter__(self):
        if self._h is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        if self._h is not None:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"]}
        names = [n for b, n in self.REASONS.items() if self.reasons & b and b != 0x1]
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": names, "samples": len(self.samples)}


def fp32_rate_probe(dev):
    """Measured FP32 FMA rate of this GPU from the probe library
    (libawq_probe.so): lane-ops per second for scalar FFMA, packed FFMA2 and
    a half-and-half mix, best of 5 launches each, with the SM clock sampled
    meanwhile.  None if the probe is unavailable."""
    import ctypes
    import torch
    from post_int4_weight_b200 import build as b
    try:
        L = ctypes.CDLL(b.PROBE_LIB)
    except OSError:
        return None
    fn = L.awq_probe_fp32_rate
    fn.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_void_p,
                   ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_double)]
    fn.restype = ctypes.c_int
    n_sms = torch.cuda.get_device_properties(dev).multi_processor_count
    out = torch.empty(n_sms * 8 * 256, dtype=torch.float32, device=dev)
    rates = {}
    ck = ClockSampler(dev)
    with ck:
        for mode, name in ((0, "scalar_ffma"), (1, "packed_ffma2"), (2, "half_packed")):
            ops, t = ctypes.c_double(0), ctypes.c_double(0)
            if fn(mode, 32768, 5, out.data_ptr(), ctypes.byref(ops), ctypes.byref(t)) != 0:
                return None
            rates[name] = ops.value / (t.value * 1e-3)
    summ = ck.summary()
    mhz = summ["sm_mhz"] or summ["sm_max_mhz"]
    best = max(rates.values())
    return {"lane_op_per_s": rates, "best": best, "sm_mhz": mhz,
            "samples": summ.get("samples", 0),
            "lane_op_per_clk_per_sm": best / (n_sms * mhz * 1e6) if mhz else None}


def launch_stream_times(jobs, wss, dev, stream, target_bytes=768 << 20, reps=20):
    """Average launch duration of awq_act_stats and of awq_quantize_pack in a
    steady stream: one CUDA graph of back-to-back calls, each on its own copy
    of the inputs (copies rotate, more bytes than the 126 MB L2 in all, so
    every call reads cold data), timed with CUDA events around the replay and
    divided by the number of calls.  Returns {"stats": ms, "pack": ms,
    "copies": n, "rot_bytes": bytes}."""
    import torch
    from post_int4_weight_b200 import awq
    in_bytes = sum(j.X.numel() * 2 + sum(W.numel() * 2 for W in j.Ws) for j in jobs)
    n = max(2, min(16, -(-target_bytes // max(in_bytes, 1))))
    if n * in_bytes > (6 << 30):
        return {}
    Xs = [[j.X.clone() for j in jobs] for _ in range(n)]
    Ws = [[[W.clone() for W in j.Ws] for j in jobs] for _ in range(n)]

    def stats_all():
        for c in range(n):
            for j, X in zip(jobs, Xs[c]):
                awq.act_stats(X, out=j.x, ws=wss.stats)

    def pack_all():
        for c in range(n):
            for j, Wl in zip(jobs, Ws[c]):
                for W, pk in zip(Wl, j.packs):
                    awq.quantize_pack(W, j.s_best, j.g, j.zero_point, out=pk)

    out = {"copies": n, "rot_bytes": n * in_bytes}
    calls = {"stats": (stats_all, n * len(jobs)),
             "pack": (pack_all, n * sum(len(j.Ws) for j in jobs))}
    for name, (fn, n_calls) in calls.items():
        fn()
        torch.cuda.synchronize(dev)
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr):
            fn()
        ts = []
        for _ in range(reps):
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            gr.replay()
            e1.record(stream)
            torch.cuda.synchronize(dev)
            ts.append(e0.elapsed_time(e1))
        out[name] = statistics.median(ts) / n_calls
        del gr
    del Xs, Ws
    return out


def h2d_bound_GBps(host_layer, dev, passes=5):
    """Pinned host -> device copy rate of one layer's input buffers: one
    cudaMemcpyAsync (torch non-blocking copy) per buffer, back to back on one
    stream, best of `passes` passes."""
    import torch
    bufs = [t for Ws, X in host_layer for t in (*Ws, X)]
    dst = [torch.empty_like(t, device=dev) for t in bufs]
    nbytes = sum(t.numel() * t.element_size() for t in bufs)
    st = torch.cuda.Stream(dev)
    best = None
    with torch.cuda.stream(st):
        for _ in range(passes + 1):
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(st)
            for d, h in zip(dst, bufs):
                d.copy_(h, non_blocking=True)
            e1.record(st)
            e1.synchronize()
            t = e0.elapsed_time(e1)
            best = t if best is None else min(best, t)
    del dst
    return nbytes / (best * 1e-3) / 1e9


# ---------------------------------------------------------------- our arm --

def _group_size(a, work):
    g = a.group_size or work.group_sizes[0]
    if g not in work.group_sizes:
        raise SystemExit(f"--group-size {g}: workload {work.name} is defined for "
                         f"{list(work.group_sizes)}")
    return g


def _layer_ids(work, world, rank):
    """(layers this rank runs, input seed override per layer, scaling)."""
    from post_int4_weight_b200 import pipeline
    if work.layers > 1:
        return pipeline.shard_layers(work.layers, world, rank), [], "strong"
    return [0], [work.seed + 1000 * rank], "weak"


def _inputs(work, layer, seed, device):
    from post_int4_weight_b200 import workloads as wl
    return [(Ws, X) for _, Ws, X in wl.group_inputs(work, layer, device, seed)]


def run_ours(a):
    import torch
    import torch.distributed as dist
    from post_int4_weight_b200 import pipeline
    from post_int4_weight_b200 import workloads as wl

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)

    work = wl.WORKLOADS[a.workload]
    g = _group_size(a, work)
    n_grid = work.n_grid
    layers, seeds, scaling = _layer_ids(work, world, rank)
    # one-layer workloads: generated on the CPU (the same tensors the parity
    # tests and the CPU baseline use); the stack: generated on the device
    gen_dev = "cpu" if work.layers == 1 else dev
    layer_inputs = []
    for i, l in enumerate(layers):
        seed = seeds[i] if i < len(seeds) else None
        layer_inputs.append([(Ws, X) for Ws, X in _inputs(work, l, seed, gen_dev)])
    jobs = []
    for li in layer_inputs:
        for Ws, X in li:
            jobs.append(pipeline.GroupJob([W.to(dev) for W in Ws], X.to(dev), g, n_grid,
                                          work.output_mode, n_clip=a.clip,
                                          scale_mode=a.scale_mode, duo=a.duo,
                                          asym=a.asym, clip_space=a.clip_space))
    if work.layers == 1:
        host_layer = [([W.pin_memory() for W in Ws], X.pin_memory()) for Ws, X in layer_inputs[0]]
    else:
        host_layer = None
    wss = pipeline.Workspaces(jobs, dev)
    params = sum(j.params for j in jobs)
    in_bytes = sum(j.X.numel() * 2 + sum(W.numel() * 2 for W in j.Ws) for j in jobs)
    flush_l2 = in_bytes < (512 << 20)
    flush = torch.empty(256 << 20 if flush_l2 else 1, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    launches_per_step = sum(j.launches for j in jobs)

    def call_stats():
        for j in jobs:
            j.stats(wss.stats)

    def call_search():
        for j in jobs:
            j.search(wss.search)

    def call_pack():
        for j in jobs:
            j.pack()

    def call_clip():
        for j in jobs:
            j.clip(wss.clip)

    def step():
        for j in jobs:
            j.run(wss)

    def do_flush():
        if flush_l2:
            flush.zero_()

    # eager warm-up (first calls do the one-time per-device set-up), then the
    # step and each call are captured into CUDA graphs and replayed
    for _ in range(max(a.warmup, 3)):
        do_flush()
        step()
    torch.cuda.synchronize(dev)
    graphs = None
    if not a.no_graph:
        graphs = {}
        calls = [("step", step), ("stats", call_stats), ("search", call_search),
                 ("pack", call_pack)] + ([("clip", call_clip)] if a.clip > 0 else [])
        for name, fn in calls:
            gr = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gr):
                fn()
            graphs[name] = gr
        for _ in range(3):
            do_flush()
            graphs["step"].replay()
        torch.cuda.synchronize(dev)
    run = {k: (graphs[k].replay if graphs else f) for k, f in
           (("step", step), ("stats", call_stats), ("search", call_search), ("pack", call_pack),
            ("clip", call_clip))
           if a.clip > 0 or k != "clip"}

    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(a.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    clk = ClockSampler(dev)
    with clk:
        for k in range(a.steps):
            do_flush()
            evs[k][0].record(stream)
            run["step"]()
            evs[k][1].record(stream)
        torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    t_step = [e0.elapsed_time(e1) for e0, e1 in evs]
    ms = pipeline.max_over_ranks(sum(t_step) / len(t_step), dev)

    # per-call breakdown (separately timed passes, L2 flushed before each);
    # about 0.2 s of passes, 3 to 200 of them; the clock sampler keeps
    # running over them (their kernels are the step's)
    n_br = max(3, min(200, int(200.0 / max(ms, 1e-3))))
    names = ["stats", "search"] + (["clip"] if a.clip > 0 else []) + ["pack"]
    br = {k: [] for k in names}
    clk_br = ClockSampler(dev)
    with clk_br:
        for _ in range(n_br):
            do_flush()
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(len(names) + 1)]
            ev[0].record(stream)
            for i, k in enumerate(names):
                run[k]()
                ev[i + 1].record(stream)
            torch.cuda.synchronize(dev)
            for i, k in enumerate(names):
                br[k].append(ev[i].elapsed_time(ev[i + 1]))
    ms_stats = sum(br["stats"]) / n_br
    ms_search = sum(br["search"]) / n_br
    ms_pack = sum(br["pack"]) / n_br
    ms_clip = sum(br["clip"]) / n_br if a.clip > 0 else None
    del graphs
    stream_ms = launch_stream_times(jobs, wss, dev, stream) if work.layers == 1 else {}

    # --- end to end: the same work streamed from pinned host memory
    template = layer_inputs[0]
    streamer = pipeline.LayerStreamer(template, dev, g, n_grid, work.output_mode,
                                      n_clip=a.clip, scale_mode=a.scale_mode, duo=a.duo,
                                      asym=a.asym, clip_space=a.clip_space)
    if work.layers == 1:
        n_e2e = max(20, min(50, a.steps // 20))
        host_layers = [host_layer] * n_e2e
        out_one = streamer.host_outputs()
        host_out = [out_one] * n_e2e
        e2e_units = n_e2e
    else:
        # this rank's layers, copied once to pinned host memory (not timed)
        def pinned(t):
            return torch.empty(t.shape, dtype=t.dtype, pin_memory=True).copy_(t)
        host_layers = [[([pinned(W) for W in Ws], pinned(X)) for Ws, X in li]
                       for li in layer_inputs]
        host_out = [streamer.host_outputs() for _ in host_layers]
        e2e_units = 1
    del layer_inputs
    for _ in range(2):   # warm-up passes over at most two layers
        streamer.run(host_layers[:2], host_out[:2])
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    streamer.run(host_layers, host_out, after=e0)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    ms_e2e = pipeline.max_over_ranks(e0.elapsed_time(e1) / e2e_units, dev)
    h2d_l, d2h_l = streamer.bytes_per_layer()
    h2d_bound = h2d_bound_GBps(host_layers[0], dev)
    per_step_layers = len(host_layers) // e2e_units
    e2e = {"value": _total_params(work, world, params) / (ms_e2e * 1e-3) / 1e9, "unit": UNIT,
           "ms_per_step": ms_e2e, "h2d_bytes_per_step": int(h2d_l * per_step_layers),
           "d2h_bytes_per_step": int(d2h_l * per_step_layers), "steps": e2e_units,
           # the copies bound this number: host->device bytes over the step time
           "h2d_GBps": h2d_l * per_step_layers / (ms_e2e * 1e-3) / 1e9,
           "h2d_bound_GBps": h2d_bound,
           "h2d_frac": (h2d_l * per_step_layers / (ms_e2e * 1e-3) / 1e9) / h2d_bound,
           "h2d_bound_basis": "the same pinned host buffers copied to the device with one "
                              "cudaMemcpyAsync each, back to back, best of 5 passes",
           "pipeline": "pinned host -> 2-slot device ring; H2D, kernels and D2H on three "
                       "streams, overlapped across layers"}

    if rank != 0:
        if world > 1:
            dist.destroy_process_group()
        return

    peaks, peak_src = _peaks()
    clocks = clk.summary()
    clocks_br = clk_br.summary()
    clocks["breakdown_sm_mhz"] = clocks_br["sm_mhz"]
    clocks["breakdown_samples"] = clocks_br.get("samples", 0)
    clocks["breakdown_reasons"] = clocks_br["reasons"]
    n_sms = torch.cuda.get_device_properties(dev).multi_processor_count
    # the per-call times (ms_search and the others) come from the breakdown
    # passes: their peaks use the clock sampled over those passes
    clk_mhz = (clocks_br["sm_mhz"] or clocks["sm_mhz"] or peaks.get("sm_max_mhz", 1965.0))
    hbm = peaks["hbm_gbs"]
    bytes_stats = sum(j.X.numel() * 2 for j in jobs)
    bytes_pack = sum(W.numel() * 2 for j in jobs for W in j.Ws) + \
        sum(t.numel() * t.element_size() for j in jobs for pk in j.packs for t in pk)
    def hbm_entry(name, nbytes, ms_single):
        # per-launch time of a stream of back-to-back calls where measured,
        # else the single-call replay (which carries the graph launch)
        ms_l = stream_ms.get(name, ms_single)
        return {"ms": ms_l, "GB/s": nbytes / (ms_l * 1e-3) / 1e9,
                "hbm_frac": nbytes / (ms_l * 1e-3) / 1e9 / hbm,
                "hbm_frac_spec": nbytes / (ms_l * 1e-3) / 1e9 / HBM_SPEC_GBS,
                "ms_single_call": ms_single,
                "basis": ("average launch of a CUDA graph of back-to-back calls on "
                          f"{stream_ms.get('copies')} rotating input copies "
                          f"({stream_ms.get('rot_bytes', 0) / 1e6:.0f} MB in all, > L2); "
                          "ms_single_call: one call per graph replay, with the graph "
                          "launch" if name in stream_ms else
                          "one call per graph replay (graph launch included)")}
    kernels = {
        "act_stats": hbm_entry("stats", bytes_stats, ms_stats),
        "quantize_pack": hbm_entry("pack", bytes_pack, ms_pack),
        "hbm_peak_GBs": hbm, "peak_source": peak_src, "hbm_spec_GBs": HBM_SPEC_GBS}
    if work.output_mode:
        flops = sum(2.0 * j.X.shape[0] * W.numel() * n_grid for j in jobs for W in j.Ws)
        achieved = flops / (ms_search * 1e-3)
        peak_t = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]) * 1e12
        roof = {"bound": "tensor",
                "kernel": "awq_output_error (scale table + per alpha: dW builder + tcgen05 "
                          "GEMM with fused square-sum + finalize)",
                "achieved": achieved / 1e12, "peak": peak_t / 1e12, "unit": "TFLOP/s",
                "frac": achieved / peak_t,
                "traffic": (NCU_TRAFFIC[(a.workload, bool(a.asym), g)] * n_grid
                            if (a.workload, bool(a.asym), g) in NCU_TRAFFIC else None),
                "traffic_basis": "DRAM bytes of the n_grid GEMM launches of one call "
                                 "(ncu, per launch x n_grid)",
                "flops_per_step": flops, "executed_flops_per_step": 2 * flops,
                "peak_basis": "measured bf16 dense GEMM, sustained (fp16 has the same "
                              "nominal tensor rate); algorithmic FLOPs 2*T*d_out*d_in per "
                              "alpha, the tensor cores execute twice that (hi and lo "
                              "fp16 parts of W - W_hat)"}
        kernels["output_error"] = {"ms": ms_search, "TFLOP/s": achieved / 1e12,
                                   "ms_median": statistics.median(br["search"]),
                                   "ms_best": min(br["search"]),
                                   "executed_TFLOP/s": 2 * achieved / 1e12}
    else:
        peak_ops = n_sms * FP32_LANES_PER_SM * clk_mhz * 1e6          # lane-ops / s
        ops = params * n_grid * ALG_OPS_PER_PAIR
        achieved = ops / (ms_search * 1e-3)
        executed = params * n_grid * FMA_OPS_PER_PAIR / (ms_search * 1e-3)
        roof = {"bound": "alu",
                "kernel": "awq_scale_search (table kernel + fused search kernel with finalize)",
                "achieved": achieved / 1e12, "peak": peak_ops / 1e12, "unit": "Top/s",
                "frac": achieved / peak_ops,
                "traffic": NCU_TRAFFIC.get((a.workload, bool(a.asym), g)),
                "ops_per_weight_alpha": ALG_OPS_PER_PAIR,
                "executed_fma_pipe_ops_per_weight_alpha": FMA_OPS_PER_PAIR,
                "executed_frac": executed / peak_ops,
                "peak_basis": f"{n_sms} SMs x {FP32_LANES_PER_SM} FP32 lanes x "
                              f"{clk_mhz:.0f} MHz (median SM clock sampled over the "
                              f"per-call passes that time the search)"}
        probe = fp32_rate_probe(dev)
        if probe and probe["lane_op_per_clk_per_sm"]:
            peak_meas = probe["lane_op_per_clk_per_sm"] * n_sms * clk_mhz * 1e6
            roof["peak_measured"] = peak_meas / 1e12
            roof["frac_measured"] = achieved / peak_meas
            roof["executed_frac_measured"] = executed / peak_meas
            roof["measured_probe"] = {
                "lane_op_per_clk_per_sm": probe["lane_op_per_clk_per_sm"],
                "Tlane_op_per_s": {k: v / 1e12 for k, v in probe["lane_op_per_s"].items()},
                "probe_sm_mhz": probe["sm_mhz"], "probe_clock_samples": probe["samples"],
                "basis": "FP32 FMA stream (libawq_probe.so, best of scalar / packed / mixed), "
                         "per SM per clock, scaled to the search passes' clock"}
        if a.clip > 0 and a.clip_space == "output":
            # Gram matrices (2 T g d_in per group set) + quadratic forms (2 g^2 per row,
            # group and ratio)
            gram = sum(2.0 * j.X.shape[0] * g * j.X.shape[1] for j in jobs for _ in j.Ws)
            forms = sum(2.0 * g * g * (W.numel() // g) * a.clip for j in jobs for W in j.Ws)
            kernels["clip_search"] = {"ms": ms_clip, "n_clip": a.clip, "space": "output",
                                      "flop": gram + forms,
                                      "TFLOP/s": (gram + forms) / (ms_clip * 1e-3) / 1e12}
        elif a.clip > 0:
            clip_ops = params * a.clip * ALG_OPS_PER_PAIR
            kernels["clip_search"] = {"ms": ms_clip, "n_clip": a.clip,
                                      "Top/s": clip_ops / (ms_clip * 1e-3) / 1e12,
                                      "frac_of_alu_peak": clip_ops / (ms_clip * 1e-3) / peak_ops}
        kernels["scale_search"] = {"ms": ms_search, "Top/s": achieved / 1e12,
                                   "ms_median": statistics.median(br["search"]),
                                   "ms_best": min(br["search"]),
                                   "executed_Tlane-op/s": executed / 1e12,
                                   "W_GB/s": params * 2 / (ms_search * 1e-3) / 1e9}
    if work.layers == 1:
        par = f"independent layer per rank x{world}"
    else:
        par = f"layers split over {world} rank(s), {len(layers)} on rank 0"
    out = {
        "metric": METRIC, "value": _total_params(work, world, params) / (ms * 1e-3) / 1e9,
        "unit": UNIT, "n_gpus": world, "steps": a.steps, "warmup": a.warmup,
        "ms_per_step": ms, "higher_is_better": True, "scaling": scaling,
        "ms_per_step_stats": {"rank0_median": statistics.median(t_step),
                              "rank0_best": min(t_step), "n": len(t_step)},
        "vs_baseline": None, "dtype": "f16" if work.output_mode else "f32",
        "data": "synthetic",
        "config": {"workload": a.workload, "layers": work.layers, "tokens": work.tokens,
                   "group_size": g, "n_grid": n_grid, "n_clip": a.clip,
                   "scale_mode": a.scale_mode, "duo": a.duo, "asym": a.asym,
                   "clip_space": a.clip_space,
                   "params_per_step": _total_params(work, world, params),
                   "params_rank0": params,
                   "l2": ("flushed (256 MB write) between timed steps" if flush_l2 else
                          f"not flushed: {in_bytes / 1e9:.2f} GB of inputs per step "
                          f"(> 126 MB L2)"),
                   "parallelism": par},
        "roofline": roof,
        "kernels": kernels,
        "clocks": clocks,
        "e2e": e2e,
        "gpu_launches": launches_per_step * a.steps,
        "launch": "CUDA graph per step" if not a.no_graph else "eager",
    }
    if world == 1 and not a.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(work, g, a.cpu_seconds, a.clip, a.scale_mode,
                                           a.duo, a.asym, a.clip_space)
    print(json.dumps(out), flush=True)
    if world > 1:
        dist.destroy_process_group()


def _total_params(work, world, params_rank0):
    """Weights quantised per step by all ranks together."""
    if work.layers > 1:
        return work.params          # the stack is split, not replicated
    return world * params_rank0


# ----------------------------------------------------------- CPU oracle --

def oracle_sample(work, g, row_cap=256, out_rows=16, out_tokens=None):
    """A bounded sample of layer 0 of the workload for the CPU oracle.

    Weight-space workloads: the first rows of every member (all of a linear
    up to 2^24 weights, else ``row_cap`` rows in proportion to the members'
    sizes) with the same share of the tokens, so the stats : search : pack
    costs keep the full layer's ratio.  The output-space workload:
    ``out_rows`` rows of the linear with ``out_tokens`` tokens (all by
    default); its cost per weight grows with the tokens, so the sample's
    weights are counted times tokens / T.
    Returns ([(Ws, X)], weights counted, description)."""
    from post_int4_weight_b200 import workloads as wl
    groups = wl.group_inputs(work, 0)
    out, params, parts = [], 0.0, []
    for grp, Ws, X in groups:
        d_out = sum(W.shape[0] for W in Ws)
        T = X.shape[0]
        if work.output_mode:
            rows, tok = out_rows, min(T, out_tokens or T)
        else:
            rows = d_out if d_out * grp.d_in <= (1 << 24) and row_cap >= 256 else row_cap
            tok = max(1, T * rows // d_out)
        Ws_s = [W[:max(8, W.shape[0] * rows // d_out)].numpy() for W in Ws]
        out.append((Ws_s, X[:tok].numpy()))
        n = sum(W.size for W in Ws_s)
        params += n * tok / T if work.output_mode else n
        parts.append(f"{grp.name}: {sum(W.shape[0] for W in Ws_s)} rows x {grp.d_in}, "
                     f"{tok} tokens")
    if work.output_mode:
        mode = "stats + 20-point output-space search + pack; weights counted x tokens/T"
    else:
        mode = "stats + 20-point search + pack"
    return out, params, "; ".join(parts) + f" ({mode})"


def _oracle_pass(sample, g, n_grid, output_mode, n_clip=0, scale_mode="joint", duo=False,
                 asym=False, clip_space="weight"):
    import oracle
    fl = (oracle.DUO if duo else 0) | (oracle.ASYM if asym else 0)
    zp = -1 if asym else 8
    for Ws, X in sample:
        x = oracle.act_stats(X)
        if output_mode:
            err = oracle.output_error(X, Ws[0], x, g, n_grid)
            s = oracle.scale_table(x, n_grid)[int(err.argmin())]
        elif scale_mode == "geomean" and len(Ws) > 1:
            s = oracle.geomean_scales([oracle.scale_search([W], x, g, n_grid, fl)[2]
                                       for W in Ws])
        else:
            err, best, s = oracle.scale_search(Ws, x, g, n_grid, fl)
        for W in Ws:
            if n_clip > 0 and clip_space == "output":
                idx = oracle.clip_search_output(X, W, s, g, n_clip)[0]
            else:
                idx = oracle.clip_search(W, x, s, g, n_clip)[0] if n_clip > 0 else None
            oracle.quantize_pack(W, s, g, zp, idx)


def cpu_baseline(work, g, seconds, n_clip=0, scale_mode="joint", duo=False, asym=False,
                 clip_space="weight"):
    """Passes of the CPU oracle over a bounded sample of the workload until
    `seconds` have elapsed."""
    import oracle
    sample, params, text = oracle_sample(work, g)
    if n_clip > 0:
        text += f" + {n_clip}-ratio clip search"
    n = 0
    t0 = time.perf_counter()
    while True:
        _oracle_pass(sample, g, work.n_grid, work.output_mode, n_clip, scale_mode, duo, asym,
                     clip_space)
        n += 1
        if time.perf_counter() - t0 >= seconds:
            break
    dt = time.perf_counter() - t0
    return {"value": n * params / dt / 1e9, "unit": UNIT, "cores": oracle.threads(),
            "kind": "oracle", "sample": f"{n} pass(es) over {text}"}


def run_reference(a):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    import oracle
    from post_int4_weight_b200 import workloads as wl
    work = wl.WORKLOADS[a.workload]
    g = _group_size(a, work)
    # a small sample per step, so that even thousands of steps end in minutes
    sample, params, text = oracle_sample(work, g, row_cap=64, out_rows=8, out_tokens=1024)
    if a.clip > 0:
        text += f" + {a.clip}-ratio clip search"
    for _ in range(max(a.warmup, 3)):
        _oracle_pass(sample, g, work.n_grid, work.output_mode, a.clip, a.scale_mode, a.duo,
                     a.asym, a.clip_space)
    t0 = time.perf_counter()
    for _ in range(a.steps):
        _oracle_pass(sample, g, work.n_grid, work.output_mode, a.clip, a.scale_mode, a.duo,
                     a.asym, a.clip_space)
    dt = time.perf_counter() - t0
    v = a.steps * params / dt / 1e9
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": world,
        "steps": a.steps, "warmup": a.warmup, "ms_per_step": dt / a.steps * 1e3,
        "higher_is_better": True, "scaling": "strong" if work.layers > 1 else "weak",
        "vs_baseline": None, "dtype": "f64" if work.output_mode else "f32",
        "data": "synthetic", "config": {"workload": a.workload, "group_size": g,
                                        "n_grid": work.n_grid, "n_clip": a.clip,
                                        "scale_mode": a.scale_mode, "duo": a.duo,
                                        "asym": a.asym},
        "cpu_baseline": {"value": v, "unit": UNIT, "cores": oracle.threads(),
                         "kind": "oracle", "sample": f"per step, one pass over {text}"},
        "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


if __name__ == "__main__":
    args = _args()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)
