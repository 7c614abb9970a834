"""Training steps whose inputs and results live in pinned host memory.

HostStepper drives an MoELayer over a sequence of steps whose per-step
inputs (x, dY and, in random-routing mode, the expert ids) arrive in pinned
host memory and whose results (y and dX) go back to pinned host memory.
It overlaps the copies with the layer's kernels on three CUDA streams:

  copy-in  : host -> device copy of step i+1's inputs (double-buffered on
             the device) while step i computes;
  compute  : the layer's calls (router ... permute backward) of step i;
  copy-out : device -> host copy of step i's y as soon as its forward ends,
             and of dX after its backward (double-buffered outputs).

Events order every buffer reuse, so results are identical to running the
steps one after another.  Nothing here computes: it only schedules copies
around the C-ABI calls that MoELayer issues.
"""
from __future__ import annotations

import torch

from .layer import MoELayer


class HostStepper:
    def __init__(self, layer: MoELayer, with_route: bool = False):
        self.L = layer
        dev = layer.device
        T, d, k = layer.T, layer.d, layer.k
        bf = torch.bfloat16
        self.compute = torch.cuda.current_stream(dev)
        self.copy_in = torch.cuda.Stream(dev)
        self.copy_out = torch.cuda.Stream(dev)
        self.x = [torch.empty(T, d, dtype=bf, device=dev) for _ in range(2)]
        self.dy = [torch.empty(T, d, dtype=bf, device=dev) for _ in range(2)]
        self.route = ([torch.empty(T, k, dtype=torch.int32, device=dev) for _ in range(2)]
                      if with_route else [None, None])
        self.y = [torch.empty(T, d, dtype=bf, device=dev) for _ in range(2)]
        self.dx = [torch.empty(T, d, dtype=bf, device=dev) for _ in range(2)]
        ev = lambda: torch.cuda.Event()
        self.in_ready = [ev(), ev()]    # inputs of buffer b copied in
        self.in_free = [ev(), ev()]     # compute finished reading inputs of buffer b
        self.fwd_done = [ev(), ev()]    # y of buffer b written
        self.bwd_done = [ev(), ev()]    # dx of buffer b written
        self.y_out = [ev(), ev()]       # y of buffer b copied out
        self.dx_out = [ev(), ev()]      # dx of buffer b copied out
        self.started = [False, False]

    def _copy_in(self, b, x_h, dy_h, route_h):
        with torch.cuda.stream(self.copy_in):
            if self.started[b]:
                self.copy_in.wait_event(self.in_free[b])
            self.x[b].copy_(x_h, non_blocking=True)
            self.dy[b].copy_(dy_h, non_blocking=True)
            if route_h is not None:
                self.route[b].copy_(route_h, non_blocking=True)
            self.in_ready[b].record(self.copy_in)

    def run(self, steps, w_r, w_gu, w_d, bias=None, after: torch.cuda.Event | None = None,
            shared=None):
        """steps: list of dicts with pinned host tensors "x", "dy", "y", "dx"
        (and "route" in random-routing mode).  Results land in each step's
        "y" and "dx" host tensors; the call returns after enqueuing
        everything (synchronise the device to read them).  `after`: an event
        that the first copy waits for.  `shared`: (w_gu_s, w_d_s) for a layer
        with a shared expert."""
        ws = {} if shared is None else {"w_gu_s": shared[0], "w_d_s": shared[1]}
        L = self.L
        n = len(steps)
        if n == 0:
            return
        if after is not None:
            self.copy_in.wait_event(after)
            self.copy_out.wait_event(after)
        s0 = steps[0]
        self._copy_in(0, s0["x"], s0["dy"], s0.get("route"))
        for i, st in enumerate(steps):
            b = i & 1
            if i + 1 < n:   # prefetch the next step's inputs into the other buffer
                nx = steps[i + 1]
                self._copy_in(b ^ 1, nx["x"], nx["dy"], nx.get("route"))
            c = self.compute
            c.wait_event(self.in_ready[b])
            if self.started[b]:   # output buffers of b are free once copied out
                c.wait_event(self.y_out[b])
                c.wait_event(self.dx_out[b])
            L.y, L.dx = self.y[b], self.dx[b]
            x, dy, route = self.x[b], self.dy[b], self.route[b]
            L.forward(x, w_r, w_gu, w_d, bias, route, **ws)
            self.fwd_done[b].record(c)
            L.backward(dy, x, w_r, w_gu, w_d, **ws)
            self.bwd_done[b].record(c)
            self.in_free[b].record(c)
            with torch.cuda.stream(self.copy_out):
                self.copy_out.wait_event(self.fwd_done[b])
                st["y"].copy_(self.y[b], non_blocking=True)
                self.y_out[b].record(self.copy_out)
                self.copy_out.wait_event(self.bwd_done[b])
                st["dx"].copy_(self.dx[b], non_blocking=True)
                self.dx_out[b].record(self.copy_out)
            self.started[b] = True

    def done_event(self):
        """An event on the compute stream after which every enqueued copy is
        complete."""
        self.compute.wait_stream(self.copy_out)
        self.compute.wait_stream(self.copy_in)
        ev = torch.cuda.Event(enable_timing=True)
        ev.record(self.compute)
        return ev
