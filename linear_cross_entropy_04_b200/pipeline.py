"""Fused linear cross-entropy over inputs and results that live in host memory.

HostPipeline runs a stream of steps whose X, W and target sit in pinned host
memory and whose loss, grad_X and grad_W must come back to pinned host memory.
Each step's host-to-device copies, compute and device-to-host copies run on
three CUDA streams ordered by events, with two device slots, so step i's
upload overlaps step i-1's compute and step i-2's download (PCIe copies in the
two directions run concurrently). Every step still copies all of its inputs
in and all of its results out; the compute is the library's fused call, or
`step` (for instance the data-parallel call, whose grad_W may come back as
this rank's rows only).
"""
from __future__ import annotations

from typing import Callable, List, Optional, Tuple

import torch

from .api import fused_linear_cross_entropy


class HostPipeline:
    def __init__(self, BT: int, H: int, V: int, dtype=torch.bfloat16, device=None, slots: int = 2,
                 step: Optional[Callable] = None, **flce_kw):
        """step(X, W, t, out) -> (loss, grad_X, grad_W), run on the compute stream,
        replaces the fused call; the tensors it returns are the ones copied back."""
        self.dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
        self.kw = flce_kw
        self.step = step
        self.slots = slots
        mk = lambda *s, dt=dtype: [torch.empty(*s, dtype=dt, device=self.dev) for _ in range(slots)]  # noqa: E731
        self.X, self.W, self.gX, self.gW = mk(BT, H), mk(V, H), mk(BT, H), mk(V, H)
        self.t = mk(BT, dt=torch.int64)
        self.loss = mk((), dt=torch.float32)
        self.s_in = torch.cuda.Stream(self.dev)
        self.s_run = torch.cuda.Stream(self.dev)
        self.s_out = torch.cuda.Stream(self.dev)
        ev = lambda: [torch.cuda.Event() for _ in range(slots)]  # noqa: E731
        self.in_done, self.run_done, self.out_done = ev(), ev(), ev()
        self.used = [False] * slots
        self.i = 0

    def submit(self, X_h: torch.Tensor, W_h: torch.Tensor, t_h: torch.Tensor,
               out_h: Tuple[torch.Tensor, torch.Tensor, torch.Tensor]):
        """Enqueue one step; results land in the pinned host tensors out_h = (loss, grad_X, grad_W)."""
        s = self.i % self.slots
        self.i += 1
        with torch.cuda.stream(self.s_in):
            if self.used[s]:
                self.s_in.wait_event(self.run_done[s])  # the slot's inputs are no longer read
            self.X[s].copy_(X_h, non_blocking=True)
            self.W[s].copy_(W_h, non_blocking=True)
            self.t[s].copy_(t_h, non_blocking=True)
            self.in_done[s].record(self.s_in)
        with torch.cuda.stream(self.s_run):
            self.s_run.wait_event(self.in_done[s])
            if self.used[s]:
                self.s_run.wait_event(self.out_done[s])  # the slot's results were copied out
            out = (self.loss[s], self.gX[s], self.gW[s])
            if self.step is None:
                fused_linear_cross_entropy(self.X[s], self.W[s], self.t[s], out=out, stream=self.s_run, **self.kw)
                res = out
            else:
                res = self.step(self.X[s], self.W[s], self.t[s], out)
            self.run_done[s].record(self.s_run)
        with torch.cuda.stream(self.s_out):
            self.s_out.wait_event(self.run_done[s])
            for h, d in zip(out_h, res):
                d.record_stream(self.s_out)  # a tensor the step allocated stays alive for the copy
                h.copy_(d, non_blocking=True)
            self.out_done[s].record(self.s_out)
        self.used[s] = True
        return self.out_done[s]

    def synchronize(self):
        for st in (self.s_in, self.s_run, self.s_out):
            st.synchronize()
