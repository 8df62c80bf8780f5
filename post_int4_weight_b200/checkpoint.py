"""Checkpoint and resume of a long layer-by-layer quantisation run.

Quantising a 36-layer stack streams every layer through the device once; a
run that stops part way (a crash, a preempted job, a lost node) should not
redo the layers it finished.  ``StackCheckpoint`` keeps each finished
layer's results on disk, written atomically (a temporary file renamed into
place, then the manifest rewritten the same way), with a SHA-256 of the
file, and a fingerprint of the run's configuration.  ``run_layers`` calls a
per-layer compute function for every layer that is not already done and
saves its results; on a rerun with the same directory and configuration it
skips the layers whose files verify and recomputes any whose file is
missing or damaged.  A manifest written under a different configuration is
refused rather than mixed in.

Host-side plumbing only: the compute function is whatever produces a
layer's results (for the device path, the library's calls through
``pipeline.GroupJob`` and a copy back to the host).
"""
from __future__ import annotations

import hashlib
import json
import os
from typing import Callable, Dict, Iterable, Mapping, Optional

import torch

MANIFEST = "manifest.json"


class CheckpointMismatch(RuntimeError):
    """The directory holds a checkpoint of a different configuration."""


def _sha256(path: str) -> str:
    h = hashlib.sha256()
    with open(path, "rb") as f:
        for block in iter(lambda: f.read(1 << 20), b""):
            h.update(block)
    return h.hexdigest()


def _atomic_write(path: str, write: Callable[[str], None]):
    tmp = path + ".tmp"
    write(tmp)
    with open(tmp, "rb") as f:
        os.fsync(f.fileno())
    os.replace(tmp, path)


class StackCheckpoint:
    """Finished layers of one run, under ``directory``.

    ``config``: a JSON-serialisable description of everything that decides
    the results (workload, group size, grid, flags, library ABI version...);
    it is stored with the first save and must match on every later open.
    """

    def __init__(self, directory: str, config: Mapping):
        self.dir = directory
        os.makedirs(directory, exist_ok=True)
        self.config = json.loads(json.dumps(dict(config), sort_keys=True))
        self._path = os.path.join(directory, MANIFEST)
        if os.path.exists(self._path):
            with open(self._path) as f:
                m = json.load(f)
            if m.get("config") != self.config:
                raise CheckpointMismatch(
                    f"{directory} holds a checkpoint of another configuration: "
                    f"{m.get('config')} != {self.config}")
            self.layers: Dict[str, Dict] = m.get("layers", {})
        else:
            self.layers = {}

    def _file(self, layer: int) -> str:
        return os.path.join(self.dir, f"layer_{layer:04d}.pt")

    def _write_manifest(self):
        body = json.dumps({"config": self.config, "layers": self.layers}, sort_keys=True,
                          indent=1)

        def write(tmp):
            with open(tmp, "w") as f:
                f.write(body)
        _atomic_write(self._path, write)

    def done(self, layer: int) -> bool:
        """True when the layer's file exists and matches its recorded hash."""
        rec = self.layers.get(str(layer))
        path = self._file(layer)
        return rec is not None and os.path.exists(path) and _sha256(path) == rec["sha256"]

    def completed(self, layers: Iterable[int]):
        return [l for l in layers if self.done(l)]

    def save(self, layer: int, results: Mapping[str, torch.Tensor]):
        """Stores a layer's results (host tensors) and records it as done."""
        path = self._file(layer)
        cpu = {k: v.detach().cpu().contiguous() for k, v in results.items()}
        _atomic_write(path, lambda tmp: torch.save(cpu, tmp))
        self.layers[str(layer)] = {"sha256": _sha256(path),
                                   "keys": sorted(cpu.keys())}
        self._write_manifest()

    def load(self, layer: int) -> Dict[str, torch.Tensor]:
        if not self.done(layer):
            raise KeyError(f"layer {layer} is not a verified part of this checkpoint")
        return torch.load(self._file(layer), map_location="cpu", weights_only=True)


def run_layers(layers: Iterable[int], compute: Callable[[int], Mapping[str, torch.Tensor]],
               ckpt: StackCheckpoint,
               on_layer: Optional[Callable[[int, bool], None]] = None) -> Dict[int, Dict]:
    """Runs ``compute(layer)`` for every layer not already done in ``ckpt``
    (in the given order), saving each result as soon as it is computed, and
    returns every layer's results (loaded from disk for the skipped ones).
    ``on_layer(layer, computed)`` is told about each layer as it is handled.
    An exception from ``compute`` propagates after the layers before it were
    saved, so a rerun resumes at the failed layer."""
    out: Dict[int, Dict] = {}
    for l in layers:
        if ckpt.done(l):
            out[l] = ckpt.load(l)
            if on_layer:
                on_layer(l, False)
            continue
        res = compute(l)
        ckpt.save(l, res)
        out[l] = {k: v.detach().cpu() for k, v in res.items()}
        if on_layer:
            on_layer(l, True)
    return out
