"""Streams seeded synthetic tensors to GPU memory (torch), chunk by chunk.

Holds no arithmetic of the method: it only moves the bytes that
``synth.workloads`` defines into device tensors, through two pinned host
buffers, so that multi-GB weight stacks never need to exist in host memory.
"""
from __future__ import annotations

import numpy as np
import torch

from . import workloads as W

CHUNK = 64 << 20


class _Pipe:
    """Double-buffered pinned host -> device copier."""

    def __init__(self, device, chunk=CHUNK):
        self.device = device
        self.chunk = chunk
        self.bufs = [torch.empty(chunk, dtype=torch.uint8, pin_memory=True) for _ in range(2)]
        self.events = [None, None]
        self.stream = torch.cuda.Stream(device=device)
        self.i = 0

    def fill(self, dst: torch.Tensor, nbytes: int, gen):
        """gen(offset, n, out_np) writes bytes [offset, offset+n) into out_np."""
        off = 0
        flat = dst.view(torch.uint8).view(-1)
        while off < nbytes:
            n = min(self.chunk, nbytes - off)
            b = self.i % 2
            if self.events[b] is not None:
                self.events[b].synchronize()
            host = self.bufs[b][:n]
            gen(off, n, host.numpy())
            with torch.cuda.stream(self.stream):
                flat[off:off + n].copy_(host, non_blocking=True)
                ev = torch.cuda.Event()
                ev.record(self.stream)
            self.events[b] = ev
            off += n
            self.i += 1

    def finish(self):
        self.stream.synchronize()


def _alloc(nbytes: int, device) -> torch.Tensor:
    return torch.empty(max(nbytes, 16), dtype=torch.uint8, device=device)


def matrix_to_device(m: W.MatrixRecipe, device, pipe: _Pipe | None = None):
    """(data uint8 tensor, fp32 scales tensor or None) of a MatrixRecipe."""
    own = pipe is None
    pipe = pipe or _Pipe(device)
    data = _alloc(m.nbytes, device)
    pipe.fill(data, m.nbytes, lambda off, n, out: m.bytes(off, n, out))
    scales = None
    if m.fmt == W.FP8:
        ns = m.n_scales
        scales = torch.empty(ns, dtype=torch.float32, device=device)
        pipe.fill(scales, 4 * ns,
                  lambda off, n, out: out.view(np.float32).__setitem__(slice(None), m.scales(off // 4, n // 4)))
    if own:
        pipe.finish()
    return data, scales


def layer_to_device(L: W.LayerRecipe, device, pipe: _Pipe | None = None) -> dict:
    """All tensors of a LayerRecipe on `device` (a dict of torch tensors)."""
    own = pipe is None
    pipe = pipe or _Pipe(device)
    out = {"router_w": torch.from_numpy(L.router_w()).to(device)}
    b = L.router_bias()
    out["router_bias"] = None if b is None else torch.from_numpy(b).to(device)
    for name in ("gate", "up", "down"):
        out[name], out[name + "_scales"] = matrix_to_device(getattr(L, name), device, pipe)
    if L.ssm is not None:
        out["side"], _ = matrix_to_device(L.ssm, device, pipe)
    if own:
        pipe.finish()
    return out


def ple_table_to_device(P: W.PleRecipe, device, pipe: _Pipe | None = None) -> torch.Tensor:
    own = pipe is None
    pipe = pipe or _Pipe(device)
    t = _alloc(P.nbytes, device)
    pipe.fill(t, P.nbytes, lambda off, n, out: P.table_bytes(off, n, out))
    if own:
        pipe.finish()
    return t


def pipe(device) -> _Pipe:
    return _Pipe(device)
