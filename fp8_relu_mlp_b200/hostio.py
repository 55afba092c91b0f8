"""Steps fed from and drained to pinned host memory, with the copies overlapped.

A training step whose inputs arrive from the host and whose results go back
to it spends most of its time on PCIe, not in the kernels (at M=16384 the
MLP block moves 50 MB in and 50 MB out per step against 0.35 ms of compute).
The link is full duplex, so :class:`HostPipeline` keeps two sets of device
buffers and three streams: while step t computes on set t % 2, the
host-to-device copy of step t+1's inputs fills the other set and the
device-to-host copy of step t-1's results drains it.  Each set's step runs
as one CUDA graph.  The order of the steps and their results are those of
running them one after another; only the copies overlap.
"""
from __future__ import annotations

import torch


class HostPipeline:
    """Runs ``step(k)`` (k = 0 or 1: the buffer set) over a stream of steps.

    ``dev_in[k]`` / ``dev_out[k]``: the device tensors step k reads / writes
    (same shapes in both sets); the host side is one list of pinned tensors
    per direction, matching them in order.  ``step(k)`` must issue its work
    on the current stream; with ``graph=True`` it is launched once per set
    and then captured into a CUDA graph (``graph=False`` launches it
    eagerly at every step instead)."""

    def __init__(self, step, dev_in, dev_out, device=None, graph=True):
        self.step = step
        self.dev_in = dev_in
        self.dev_out = dev_out
        self.device = torch.device(device) if device is not None else dev_in[0][0].device
        self.s_in = torch.cuda.Stream(self.device)
        self.s_out = torch.cuda.Stream(self.device)
        self.main = torch.cuda.current_stream(self.device)
        self.graphs = [None, None]
        if graph:
            for k in (0, 1):
                step(k)  # warm-up launch, outside the capture
                torch.cuda.synchronize(self.device)
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g):
                    step(k)
                self.graphs[k] = g

    def _run(self, k):
        if self.graphs[k] is not None:
            self.graphs[k].replay()
        else:
            self.step(k)

    def run(self, host_in, host_out, steps, timer=None):
        """``steps`` steps, each copying ``host_in`` in and ``dev_out`` back
        to ``host_out``.  With ``timer = (start, end)`` CUDA events, start is
        recorded before the first copy and end after the last result is on
        the host side of the copy."""
        h2d = [torch.cuda.Event(), torch.cuda.Event()]
        done = [torch.cuda.Event(), torch.cuda.Event()]
        d2h = [torch.cuda.Event(), torch.cuda.Event()]
        used_in = [False, False]   # set k's inputs were read by an issued step
        used_out = [False, False]  # set k's outputs have a copy-out issued

        def copy_in(k):
            with torch.cuda.stream(self.s_in):
                if used_in[k]:
                    self.s_in.wait_event(done[k])
                for dst, src in zip(self.dev_in[k], host_in):
                    dst.copy_(src, non_blocking=True)
                h2d[k].record(self.s_in)

        if timer is not None:
            timer[0].record(self.s_in)
        copy_in(0)
        for t in range(steps):
            k = t & 1
            if t + 1 < steps:
                copy_in(k ^ 1)
            self.main.wait_event(h2d[k])
            if used_out[k]:
                self.main.wait_event(d2h[k])
            self._run(k)
            used_in[k] = True
            done[k].record(self.main)
            with torch.cuda.stream(self.s_out):
                self.s_out.wait_event(done[k])
                for dst, src in zip(host_out, self.dev_out[k]):
                    dst.copy_(src, non_blocking=True)
                d2h[k].record(self.s_out)
            used_out[k] = True
        self.main.wait_stream(self.s_out)
        if timer is not None:
            timer[1].record(self.main)


def block_pipeline(blk, side, graph=True, step_fn=None):
    """A :class:`HostPipeline` over an :class:`MLPBlock` training step
    (``train_step_overlapped``: forward, backward, scale update and W2 cache
    refresh; or ``step_fn()``, e.g. a data-parallel step of the same block);
    inputs x and dOut, results out and dX.  The block's own buffers are set
    0; set 1 starts as a copy of them.  With ``graph=True`` building the
    pipeline runs one training step on each set (the launch before each
    capture), so the block's delayed scale advances by two steps."""
    sets = [dict(x=blk.x, dOut=blk.dOut, out=blk.out, dX=blk.dX)]
    sets.append({k: v.clone() for k, v in sets[0].items()})

    def step(k):
        for name, t in sets[k].items():
            setattr(blk, name, t)
        if step_fn is not None:
            step_fn()
        else:
            blk.train_step_overlapped(side)

    pipe = HostPipeline(step, [[s["x"], s["dOut"]] for s in sets], [[s["out"], s["dX"]] for s in sets],
                        device=blk.device, graph=graph)
    for name, t in sets[0].items():
        setattr(blk, name, t)
    return pipe
