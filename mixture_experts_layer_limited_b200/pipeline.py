"""Forwards over batches that live in pinned host memory, with the copies
hidden behind the computation.

A batch's tokens go host -> device on one copy stream while the previous
batch is still being computed, and a finished batch's output goes device ->
host on a second copy stream while the next batch is computed. The device
input is double-buffered (a copy into one buffer may start once the forward
two batches back has finished reading it); the layer's output buffer is
single, so a forward's combine waits until the previous output has left the
device. Ordering is by CUDA events only: no host synchronisation inside the
loop. torch provides the streams, events and buffers; every step of the
forward is a libmoe launch.
"""
from typing import Callable, Optional, Sequence

import torch

from .layer import MoELayer

# stages that read the forward's input x, and the stage that writes its output y
_READS_X = ("route", "permute", "gate_up", "gate_up_routed", "gate_up_shared", "ffn")
_WRITES_Y = ("combine", "down_combine")


class HostPipeline:
    def __init__(self, layer: MoELayer, T: int):
        if T > layer.T_max:
            raise ValueError(f"T={T} exceeds the layer's T_max={layer.T_max}")
        self.layer = layer
        self.T = T
        dev = layer.dev
        self.x_dev = [torch.empty(T, layer.spec.H, dtype=torch.bfloat16, device=dev) for _ in range(2)]
        self.stages = [layer.stages(x) for x in self.x_dev]
        last = [max(i for i, (n, _) in enumerate(st) if n in _READS_X) for st in self.stages]
        self.last_x_reader = last
        self.h2d = torch.cuda.Stream(device=dev)
        self.d2h = torch.cuda.Stream(device=dev)
        self.x_loaded = [torch.cuda.Event() for _ in range(2)]
        self.x_free = [torch.cuda.Event() for _ in range(2)]
        self.y_ready = torch.cuda.Event()
        self.y_free = torch.cuda.Event()

    def run(self, x_host: Sequence[torch.Tensor], y_host: Sequence[torch.Tensor],
            after_forward: Optional[Callable[[int], None]] = None):
        """Computes y_host[i] = layer(x_host[i]) for every i, in order.

        x_host[i] / y_host[i]: pinned [T, H] bf16 host tensors. after_forward(i),
        if given, is called on the compute stream right after forward i (e.g.
        the bias step); its work is ordered before forward i + 1. Returns
        without waiting for the device; synchronise before reading y_host."""
        compute = torch.cuda.current_stream(self.layer.dev)
        y = self.layer.y[:self.T]
        for i, (xh, yh) in enumerate(zip(x_host, y_host)):
            b = i % 2
            # input: into buffer b once forward i-2 has finished reading it
            self.h2d.wait_event(self.x_free[b])
            with torch.cuda.stream(self.h2d):
                self.x_dev[b].copy_(xh, non_blocking=True)
            self.x_loaded[b].record(self.h2d)
            compute.wait_event(self.x_loaded[b])
            for j, (name, fn) in enumerate(self.stages[b]):
                if name in _WRITES_Y:
                    compute.wait_event(self.y_free)        # the previous output has left y
                fn()
                if j == self.last_x_reader[b]:
                    self.x_free[b].record(compute)
            if after_forward is not None:
                after_forward(i)
            self.y_ready.record(compute)
            # output: device -> host while the next forward runs
            self.d2h.wait_event(self.y_ready)
            with torch.cuda.stream(self.d2h):
                yh.copy_(y, non_blocking=True)
            self.y_free.record(self.d2h)
        # the caller's stream sees every copy finished
        compute.wait_stream(self.h2d)
        compute.wait_stream(self.d2h)
