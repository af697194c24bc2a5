"""Checkpoint and resume of an optimizer run, continuing bit for bit.

The whole state of a run is device tensors and step counters: the weights,
every simulated worker's momentum (or LionMuon EMA), the step count t that
selects Muon steps and the counter-based gradient streams, and for CacheMuon
the cached transform Q, the current momentum and the counters. Nothing else
carries over between steps, so restoring those bytes into the same buffers
and continuing gives exactly the run that never stopped.

snapshot() copies the state to host memory; restore() copies it back in place
(the tensors keep their addresses, so prepared plans stay valid); save() and
load() put a snapshot in a file with torch.save.
"""
from __future__ import annotations

import torch

from . import CacheMuon, LionMuon


def _sync(named) -> None:
    if any(t.is_cuda for t in named.values()):
        torch.cuda.synchronize()


def _host(t: torch.Tensor) -> torch.Tensor:
    return t.detach().to("cpu", copy=True)


def _put(dst: torch.Tensor, src: torch.Tensor, name: str) -> None:
    if dst.shape != src.shape or dst.dtype != src.dtype:
        raise ValueError(f"checkpoint entry {name}: {tuple(src.shape)} {src.dtype} does not fit "
                         f"{tuple(dst.shape)} {dst.dtype}")
    dst.copy_(src.to(dst.device), non_blocking=False)


def _tensors(obj):
    """(kind, named tensors, counters) of an optimizer object or a dict of tensors."""
    if isinstance(obj, LionMuon):
        named = {f"W.{l}": w for l, w in enumerate(obj.W)}
        named.update({f"mom.{l}.{k}": m for l, layer in enumerate(obj.mom) for k, m in enumerate(layer)})
        return "lionmuon", named, {"t": int(obj.state.t)}
    if isinstance(obj, CacheMuon):
        named = {"M": obj.M, "D": obj.D, "Q": obj.Q, "err": obj.err, "accept": obj.accept, "counters": obj.cnt}
        return "cachemuon", named, {"steps": int(obj.steps)}
    if isinstance(obj, dict):
        return "tensors", dict(obj), {}
    raise TypeError(f"cannot checkpoint a {type(obj).__name__}")


def snapshot(obj) -> dict:
    """Host copy of the state (waits for the device work that produced it)."""
    kind, named, counters = _tensors(obj)
    _sync(named)
    return {"kind": kind, "tensors": {k: _host(v) for k, v in named.items()}, "counters": counters}


def restore(obj, snap: dict) -> None:
    """Copies a snapshot back into the object's own tensors and counters."""
    kind, named, _ = _tensors(obj)
    if snap["kind"] != kind:
        raise ValueError(f"checkpoint of a {snap['kind']} run cannot resume a {kind} run")
    if set(snap["tensors"]) != set(named):
        raise ValueError("checkpoint and run hold different tensors")
    for k, v in named.items():
        _put(v, snap["tensors"][k], k)
    if kind == "lionmuon":
        obj.state.t = snap["counters"]["t"]
    elif kind == "cachemuon":
        obj.steps = snap["counters"]["steps"]
    _sync(named)


def save(path: str, obj) -> None:
    torch.save(snapshot(obj), path)


def load(path: str, obj) -> None:
    restore(obj, torch.load(path, map_location="cpu", weights_only=True))
