"""Overlapped host <-> device streaming of chunks through the library.

A streaming caller produces one chunk after another on the host and wants
each chunk's output back on the host.  Run serially, every chunk pays its
host-to-device copy, its compute and its device-to-host copy one after the
other.  ``ChunkPipeline`` runs them on three CUDA streams instead: chunk n's
inputs are copied in while chunk n - 1 computes and chunk n - 2's outputs are
copied out, with ``depth`` (>= 2) device staging slots for the inputs and
outputs.  The compute stream runs the chunks in submission order, so the
rolling window sees its appends in stream order.

Only plumbing lives here (torch streams, events and device buffers); every
step of the computation is the caller's ``step`` function, which issues the
library calls on the stream it is given.
"""
from __future__ import annotations

from typing import Callable, Dict, Tuple

import torch

Spec = Dict[str, Tuple[Tuple[int, ...], torch.dtype]]


class ChunkPipeline:
    """Three-stream executor for per-chunk device steps.

    inputs / outputs: name -> (shape, dtype) of the per-chunk device tensors.
    step(dev_in, dev_out, stream): enqueues the chunk's work on ``stream``,
    reading ``dev_in`` and writing ``dev_out`` (dicts of device tensors).
    """

    def __init__(self, inputs: Spec, outputs: Spec, step: Callable, depth: int = 2, device="cuda"):
        if depth < 2:
            raise ValueError("depth must be >= 2")
        self.step = step
        self.depth = depth
        self.device = torch.device(device)
        self.h2d = torch.cuda.Stream(self.device)
        self.compute = torch.cuda.Stream(self.device)
        self.d2h = torch.cuda.Stream(self.device)
        self.dev_in = [{n: torch.empty(s, dtype=d, device=self.device) for n, (s, d) in inputs.items()}
                       for _ in range(depth)]
        self.dev_out = [{n: torch.empty(s, dtype=d, device=self.device) for n, (s, d) in outputs.items()}
                        for _ in range(depth)]
        self.h2d_done = [torch.cuda.Event() for _ in range(depth)]
        self.comp_done = [torch.cuda.Event() for _ in range(depth)]
        self.d2h_done = [torch.cuda.Event() for _ in range(depth)]
        self.n = 0

    def submit(self, host_in: Dict[str, torch.Tensor], host_out: Dict[str, torch.Tensor]) -> None:
        """Queue one chunk: copy ``host_in`` in, run the step, copy the outputs
        into ``host_out``.  Host tensors should be pinned (for asynchronous
        copies) and must stay untouched until ``synchronize`` (or until a
        later ``d2h_done`` event of their slot) has passed."""
        slot = self.n % self.depth
        reuse = self.n >= self.depth
        din, dout = self.dev_in[slot], self.dev_out[slot]
        # inputs: the slot's previous chunk has finished computing
        if reuse:
            self.h2d.wait_event(self.comp_done[slot])
        with torch.cuda.stream(self.h2d):
            for name, t in din.items():
                t.copy_(host_in[name], non_blocking=True)
            self.h2d_done[slot].record(self.h2d)
        # compute: inputs landed, and the slot's previous outputs have left
        self.compute.wait_event(self.h2d_done[slot])
        if reuse:
            self.compute.wait_event(self.d2h_done[slot])
        with torch.cuda.stream(self.compute):
            self.step(din, dout, self.compute)
            self.comp_done[slot].record(self.compute)
        # outputs
        self.d2h.wait_event(self.comp_done[slot])
        with torch.cuda.stream(self.d2h):
            for name, t in dout.items():
                host_out[name].copy_(t, non_blocking=True)
            self.d2h_done[slot].record(self.d2h)
        self.n += 1

    def synchronize(self) -> None:
        self.h2d.synchronize()
        self.compute.synchronize()
        self.d2h.synchronize()
