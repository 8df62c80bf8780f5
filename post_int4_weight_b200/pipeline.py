"""Orchestration of the AWQ hot path over search groups, layers and stacks.

Host plumbing only: output buffers, shared workspaces, CUDA streams, events
and the split of a stack's layers over ranks.  Every step of the method runs
in the library's kernels through the calls of :mod:`awq`.

The unit of work is a *search group*: the linears that read one input X
(q/k/v, gate/up, or a linear alone).  Its path is awq_act_stats on X, the
scale search (weight-space, or output-space with ``output_mode``) over all
members at once -- or, with ``scale_mode="geomean"``, one search per member
and the geometric mean of their scales (the Qwen3-8B page's exporter steps
1-2: one scale per norm group) -- optionally a clip search per member (``n_clip`` > 0; the
architecture page's pipeline step 5), then awq_quantize_pack of every member
at the chosen scale (and clip ratios)
("From-Scratch AWQ INT4 Quantization on Qwen3-8B", pipeline and AWQ scaling
sections; "AWQ architecture, in depth", section "The scale search as code").
"""
from __future__ import annotations

from typing import List, Sequence, Tuple

import torch

from . import awq

# kernels each call launches (the library's own count, used for reporting)
LAUNCHES_STATS = 1
LAUNCHES_SEARCH = 2            # scale table + fused search with finalize
LAUNCHES_CLIP = 2              # per member: (x / s)^2 + clip search (plus the memset)
LAUNCHES_CLIP_OUTPUT = 3       # per member: Gram slices + their sum + scoring (plus the memset)


def launches_output_error(n_grid: int) -> int:
    """Scale table + one dW builder and one GEMM per grid point + finalize."""
    return 1 + 2 * n_grid + 1


def shard_layers(n_layers: int, world: int, rank: int) -> List[int]:
    """Layers of a stack that one rank quantises: layer l goes to rank l % world.

    Layers are independent units of the path (each has its own inputs and
    outputs), so the split needs no exchange between ranks."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside world of {world}")
    return list(range(rank, n_layers, world))


def max_over_ranks(value: float, device=None) -> float:
    """Maximum of a per-rank number over all ranks of the default process
    group (the rank's own value when there is no group)."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    if device is None:
        device = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


class GroupJob:
    """One search group on the device with its output buffers.

    Ws: fp16 [d_out_k, d_in] device tensors sharing the input X fp16 [T, d_in].
    After :meth:`run`: ``x`` (activation magnitude), ``err`` (per grid point),
    ``best``, ``s_best`` and ``packs`` [(qweight, scales, qzeros) per member].
    """

    def __init__(self, Ws: Sequence[torch.Tensor], X: torch.Tensor, group_size: int = 128,
                 n_grid: int = 20, output_mode: bool = False, zero_point: int = 8,
                 n_clip: int = 0, scale_mode: str = "joint", duo: bool = False,
                 asym: bool = False, clip_space: str = "weight"):
        if output_mode and len(Ws) != 1:
            raise ValueError("the output-space score takes one linear per call")
        if scale_mode not in ("joint", "geomean"):
            raise ValueError("scale_mode is 'joint' or 'geomean'")
        self.Ws = list(Ws)
        self.X = X
        self.g = group_size
        self.n_grid = n_grid
        self.output_mode = output_mode
        self.n_clip = n_clip
        if clip_space not in ("weight", "output"):
            raise ValueError("clip_space is 'weight' or 'output'")
        self.clip_space = clip_space
        self.flags = (awq.DUO_SCALING if duo else 0) | (awq.ASYMMETRIC if asym else 0)
        if (duo or asym) and output_mode:
            raise ValueError("duo scaling and the asymmetric grid are weight-space options")
        if asym and n_clip > 0:
            raise ValueError("the clip search is defined on the symmetric grid")
        if asym:
            zero_point = awq.ZERO_POINT_ASYM
        self.zero_point = zero_point
        # geomean with one member is the joint search
        self.geomean = scale_mode == "geomean" and len(self.Ws) > 1
        dev = X.device
        T, d_in = X.shape
        M = len(self.Ws)
        self.x = torch.empty(d_in, dtype=torch.float32, device=dev)
        if self.geomean:
            # per member: errors, chosen index and scale; s_best is their
            # geometric mean
            # (rows padded to 16 bytes: the library wants aligned outputs)
            self.err = torch.empty(M, (n_grid + 1) // 2 * 2, dtype=torch.float64, device=dev)
            self.best = torch.empty(M, 4, dtype=torch.int32, device=dev)
            self.member_s = torch.empty(M, d_in, dtype=torch.float32, device=dev)
        else:
            self.err = torch.empty(n_grid, dtype=torch.float64, device=dev)
            self.best = torch.empty(1, dtype=torch.int32, device=dev)
        self.s_best = torch.empty(d_in, dtype=torch.float32, device=dev)
        G = d_in // group_size
        self.packs = [(torch.empty(d_in, W.shape[0] // 8, dtype=torch.int32, device=dev),
                       torch.empty(G, W.shape[0], dtype=torch.float16, device=dev),
                       torch.empty(G, W.shape[0] // 8, dtype=torch.int32, device=dev))
                      for W in self.Ws]
        # clip ratio indices and (unclipped, clipped) error totals per member
        self.clips = [(torch.zeros(W.shape[0], G, dtype=torch.uint8, device=dev),
                       torch.zeros(2, dtype=torch.float64, device=dev))
                      for W in self.Ws] if n_clip > 0 else []

    @property
    def params(self) -> int:
        return sum(W.numel() for W in self.Ws)

    @property
    def launches(self) -> int:
        if self.output_mode:
            search = launches_output_error(self.n_grid)
        elif self.flags & awq.DUO_SCALING:
            # weight mean (2) + duo table (2) + search, per search call
            n = len(self.Ws) if self.geomean else 1
            search = 5 * n + (1 if self.geomean else 0)
        elif self.geomean:
            search = LAUNCHES_SEARCH * len(self.Ws) + 1
        else:
            search = LAUNCHES_SEARCH
        per_clip = LAUNCHES_CLIP_OUTPUT if self.clip_space == "output" else LAUNCHES_CLIP
        clip = per_clip * len(self.Ws) if self.n_clip > 0 else 0
        return LAUNCHES_STATS + search + clip + len(self.Ws)

    def workspace_bytes(self) -> Tuple[int, int, int]:
        """(act_stats, search, clip) workspace bytes of this job."""
        T, d_in = self.X.shape
        d_out = sum(W.shape[0] for W in self.Ws)
        st = awq.workspace_size(awq.OP_ACT_STATS, T, 8, d_in, self.g, self.n_grid)
        op = awq.OP_OUTPUT_ERROR if self.output_mode else (
            awq.OP_SCALE_SEARCH_DUO if self.flags & awq.DUO_SCALING else awq.OP_SCALE_SEARCH)
        se = awq.workspace_size(op, T, d_out, d_in, self.g, self.n_grid)
        cl_op = awq.OP_CLIP_SEARCH_OUTPUT if self.clip_space == "output" else awq.OP_CLIP_SEARCH
        d_max = max(W.shape[0] for W in self.Ws)
        cl = awq.workspace_size(cl_op, T, d_max, d_in, self.g, 1) if self.n_clip > 0 else 0
        return st, se, cl

    def stats(self, ws: torch.Tensor):
        awq.act_stats(self.X, out=self.x, ws=ws)

    def search(self, ws: torch.Tensor):
        if self.geomean:
            for m, W in enumerate(self.Ws):
                awq.scale_search([W], self.x, self.g, self.n_grid, self.flags,
                                 out=(self.err[m, :self.n_grid], self.best[m, :1],
                                      self.member_s[m]), ws=ws)
            awq.norm_group_scale(list(self.member_s), out=self.s_best)
            return
        out = (self.err, self.best, self.s_best)
        if self.output_mode:
            awq.output_error(self.X, self.Ws[0], self.x, self.g, self.n_grid,
                             self.flags & awq.ASYMMETRIC, out=out, ws=ws)
        else:
            awq.scale_search(self.Ws, self.x, self.g, self.n_grid, self.flags, out=out, ws=ws)

    def clip(self, ws: torch.Tensor):
        for W, cl in zip(self.Ws, self.clips):
            if self.clip_space == "output":
                awq.clip_search_output(self.X, W, self.s_best, self.g, self.n_clip, out=cl,
                                       ws=ws)
            else:
                awq.clip_search(W, self.x, self.s_best, self.g, self.n_clip, out=cl, ws=ws)

    def pack(self):
        for m, (W, pk) in enumerate(zip(self.Ws, self.packs)):
            awq.quantize_pack(W, self.s_best, self.g, self.zero_point, out=pk,
                              clip_idx=self.clips[m][0] if self.n_clip > 0 else None)

    def run(self, ws: "Workspaces"):
        self.stats(ws.stats)
        self.search(ws.search)
        if self.n_clip > 0:
            self.clip(ws.clip)
        self.pack()


class Workspaces:
    """One workspace per call kind, sized for the largest of ``jobs``.  Jobs
    that run one after another on one stream may share it; jobs that run
    concurrently need their own."""

    def __init__(self, jobs: Sequence[GroupJob], device):
        sizes = [j.workspace_bytes() for j in jobs]
        st = max([b[0] for b in sizes] + [1])
        se = max([b[1] for b in sizes] + [1])
        cl = max([b[2] for b in sizes] + [1])
        self.stats = torch.empty(st, dtype=torch.uint8, device=device)
        self.search = torch.empty(se, dtype=torch.uint8, device=device)
        self.clip = torch.empty(cl, dtype=torch.uint8, device=device)


def _pinned_like(t: torch.Tensor) -> torch.Tensor:
    return torch.empty(t.shape, dtype=t.dtype, pin_memory=True)


class LayerStreamer:
    """Quantises layers held in pinned host memory, end to end.

    A ring of ``depth`` device slots (each slot: the inputs and outputs of one
    layer) is driven by three streams: host-to-device copies of layer l+1 run
    on one, the kernels of layer l on another, and the device-to-host copies
    of layer l-1's results on a third, ordered by events per slot.  A layer is
    given as [(Ws, X) per search group] of pinned CPU tensors; all layers have
    the shapes of ``template`` (the same list with device or CPU tensors).
    """

    def __init__(self, template, device, group_size: int = 128, n_grid: int = 20,
                 output_mode: bool = False, zero_point: int = 8, depth: int = 2,
                 n_clip: int = 0, scale_mode: str = "joint", duo: bool = False,
                 asym: bool = False, clip_space: str = "weight"):
        self.device = torch.device(device)
        self.depth = depth
        self.slots = []
        for _ in range(depth):
            jobs = []
            for Ws, X in template:
                dWs = [torch.empty(W.shape, dtype=torch.float16, device=self.device) for W in Ws]
                dX = torch.empty(X.shape, dtype=torch.float16, device=self.device)
                jobs.append(GroupJob(dWs, dX, group_size, n_grid, output_mode, zero_point,
                                     n_clip, scale_mode, duo, asym, clip_space))
            self.slots.append(jobs)
        self.ws = Workspaces(self.slots[0], self.device)
        self.h2d = torch.cuda.Stream(self.device)
        self.compute = torch.cuda.Stream(self.device)
        self.d2h = torch.cuda.Stream(self.device)
        self.loaded = [torch.cuda.Event() for _ in range(depth)]
        self.computed = [torch.cuda.Event() for _ in range(depth)]
        self.drained = [torch.cuda.Event() for _ in range(depth)]
        cur = torch.cuda.current_stream(self.device)
        for evs in (self.loaded, self.computed, self.drained):
            for e in evs:
                e.record(cur)

    @property
    def launches_per_layer(self) -> int:
        return sum(j.launches for j in self.slots[0])

    def host_outputs(self):
        """Pinned host buffers for one layer's results:
        [(err, best, s_best, [(qweight, scales, qzeros[, clip_idx]) per member])
        per group]."""
        out = []
        for j in self.slots[0]:
            packs = []
            for m, pk in enumerate(j.packs):
                ts = list(pk) + ([j.clips[m][0]] if j.n_clip > 0 else [])
                packs.append(tuple(_pinned_like(t) for t in ts))
            out.append((_pinned_like(j.err), _pinned_like(j.best), _pinned_like(j.s_best),
                        packs))
        return out

    def bytes_per_layer(self) -> Tuple[int, int]:
        """(host-to-device, device-to-host) bytes copied per layer."""
        jobs = self.slots[0]
        h2d = sum(j.X.numel() * 2 + sum(W.numel() * 2 for W in j.Ws) for j in jobs)
        d2h = sum(j.err.numel() * 8 + j.best.numel() * 4 + j.s_best.numel() * 4 +
                  sum(t.numel() * t.element_size() for pk in j.packs for t in pk) +
                  sum(c[0].numel() for c in j.clips)
                  for j in jobs)
        return h2d, d2h

    def run(self, host_layers, host_out, after=None):
        """Enqueue every layer of ``host_layers``; results land in the matching
        entries of ``host_out``.  ``after``: an event the copies must wait
        for.  Returns with the work enqueued; the current stream waits for all
        of it."""
        if after is not None:
            for s in (self.h2d, self.compute, self.d2h):
                s.wait_event(after)
        for l, layer in enumerate(host_layers):
            k = l % self.depth
            jobs = self.slots[k]
            self.h2d.wait_event(self.computed[k])     # the slot's inputs are free
            with torch.cuda.stream(self.h2d):
                for job, (Ws, X) in zip(jobs, layer):
                    job.X.copy_(X, non_blocking=True)
                    for dW, W in zip(job.Ws, Ws):
                        dW.copy_(W, non_blocking=True)
            self.loaded[k].record(self.h2d)
            self.compute.wait_event(self.loaded[k])
            self.compute.wait_event(self.drained[k])  # the slot's outputs are free
            with torch.cuda.stream(self.compute):
                for job in jobs:
                    job.run(self.ws)
            self.computed[k].record(self.compute)
            self.d2h.wait_event(self.computed[k])
            with torch.cuda.stream(self.d2h):
                for job, (err, best, s_best, packs) in zip(jobs, host_out[l]):
                    err.copy_(job.err, non_blocking=True)
                    best.copy_(job.best, non_blocking=True)
                    s_best.copy_(job.s_best, non_blocking=True)
                    for m, (pk_h, pk) in enumerate(zip(packs, job.packs)):
                        src = list(pk) + ([job.clips[m][0]] if job.n_clip > 0 else [])
                        for th, t in zip(pk_h, src):
                            th.copy_(t, non_blocking=True)
            self.drained[k].record(self.d2h)
        cur = torch.cuda.current_stream(self.device)
        for s in (self.h2d, self.compute, self.d2h):
            cur.wait_stream(s)
