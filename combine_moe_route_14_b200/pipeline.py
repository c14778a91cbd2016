"""Host-buffer pipelining for a layer: host->device copies, the forward and
device->host copies of consecutive batches overlap.

The layer itself runs entirely in the library's kernels; this module only
orders copies and launches on three CUDA streams:

    h2d stream      X[i] (and logits[i]) pinned host -> device buffer s = i % depth
    compute stream  the layer forward on buffer s (waits for its inputs, and for
                    the device->host copy that last read output buffer s)
    d2h stream      Y[i] device buffer s -> pinned host (waits for the forward)

With depth >= 2 the copies of batch i+1 and i-1 run while batch i computes,
so a step costs the slowest of the three instead of their sum.  Every batch's
copies still happen; nothing is cached.
"""
from __future__ import annotations

import torch

__all__ = ["HostPipeline"]


class HostPipeline:
    """Run `layer` (a MoeLayer) over batches held in pinned host memory.

    submit(X_pin, Y_pin, logits_pin=None) enqueues one batch and returns at
    once; Y_pin is complete after synchronize() (or once a later submit has
    gone `depth` batches past it).  X_pin [T, d] bf16, Y_pin [T, d] bf16 and
    logits_pin [T, E] fp32 must be pinned host tensors of the shapes given here.
    """

    def __init__(self, layer, T: int, d: int, E: int | None = None, with_logits: bool = False,
                 device=None, depth: int = 2):
        if depth < 1:
            raise ValueError("depth must be >= 1")
        dev = torch.device(device) if device is not None else layer.W1.device
        self.layer, self.depth, self.device = layer, depth, dev
        self.h2d = torch.cuda.Stream(device=dev)
        self.comp = torch.cuda.Stream(device=dev)
        self.d2h = torch.cuda.Stream(device=dev)
        self.X = [torch.empty((T, d), dtype=torch.bfloat16, device=dev) for _ in range(depth)]
        self.Y = [torch.empty((T, d), dtype=torch.bfloat16, device=dev) for _ in range(depth)]
        self.L = ([torch.empty((T, E), dtype=torch.float32, device=dev) for _ in range(depth)]
                  if with_logits else None)
        mk = lambda: [torch.cuda.Event() for _ in range(depth)]  # noqa: E731
        self.x_ready, self.x_free, self.y_ready, self.y_free = mk(), mk(), mk(), mk()
        self.n = 0

    def submit(self, X_pin, Y_pin, logits_pin=None):
        s = self.n % self.depth
        reuse = self.n >= self.depth  # buffer s was used by batch n - depth
        with torch.cuda.stream(self.h2d):
            if reuse:
                self.h2d.wait_event(self.x_free[s])
            self.X[s].copy_(X_pin, non_blocking=True)
            if self.L is not None:
                self.L[s].copy_(logits_pin, non_blocking=True)
            self.x_ready[s].record(self.h2d)
        with torch.cuda.stream(self.comp):
            self.comp.wait_event(self.x_ready[s])
            if reuse:
                self.comp.wait_event(self.y_free[s])
            self.layer(self.X[s], logits=None if self.L is None else self.L[s], Y=self.Y[s],
                       stream=self.comp)
            self.x_free[s].record(self.comp)
            self.y_ready[s].record(self.comp)
        with torch.cuda.stream(self.d2h):
            self.d2h.wait_event(self.y_ready[s])
            Y_pin.copy_(self.Y[s], non_blocking=True)
            self.y_free[s].record(self.d2h)
        self.n += 1

    def synchronize(self):
        for st in (self.h2d, self.comp, self.d2h):
            st.synchronize()
