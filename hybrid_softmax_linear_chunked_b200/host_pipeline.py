"""Batches from pinned host memory through a device computation with the copies overlapped.

For a run of steps whose inputs live in host memory, step i's computation runs on the caller's
stream while the upload of step i+1's inputs runs on an upload stream and the download of step
i-1's output on a download stream (PCIe carries the two directions at once).  Device inputs and
outputs are double-buffered, and events order each buffer's reuse:
  * upload i+1 waits for compute i-1 (the last reader of that input buffer);
  * compute i waits for upload i and for download i-2 (the last reader of its output buffer);
  * download i waits for compute i.
The caller's stream waits for the last download before `run` returns (nothing is synchronised on
the host), so events recorded on it around `run` bracket every copy and every computation.
"""
from __future__ import annotations

from typing import Callable, Sequence

import torch


class HostPipeline:
    """`compute(i, dev_inputs, dev_out)` enqueues step i on the current stream; `in_like` and
    `out_like` give the shapes and dtypes of one step's device inputs and output (the same for
    every step).  `out_like` may be a list: `dev_out` and each step's host output are then lists
    in the same order."""

    def __init__(self, compute: Callable[[int, list, object], None],
                 in_like: Sequence[torch.Tensor], out_like, device):
        self.compute = compute
        self.device = torch.device(device)
        self.multi = not isinstance(out_like, torch.Tensor)
        outs = list(out_like) if self.multi else [out_like]
        self.inputs = [[torch.empty(t.shape, dtype=t.dtype, device=self.device) for t in in_like]
                       for _ in range(2)]
        self.outputs = [[torch.empty(t.shape, dtype=t.dtype, device=self.device) for t in outs]
                        for _ in range(2)]
        self.up = torch.cuda.Stream(self.device)
        self.down = torch.cuda.Stream(self.device)
        self.ev_up = [torch.cuda.Event() for _ in range(2)]
        self.ev_comp = [torch.cuda.Event() for _ in range(2)]
        self.ev_down = [torch.cuda.Event() for _ in range(2)]

    def _upload(self, i: int, host_inputs: Sequence[torch.Tensor]) -> None:
        b = i % 2
        with torch.cuda.stream(self.up):
            if i >= 2:
                self.up.wait_event(self.ev_comp[b])
            for dst, src in zip(self.inputs[b], host_inputs):
                dst.copy_(src, non_blocking=True)
            self.ev_up[b].record(self.up)

    def run(self, host_inputs: Sequence[Sequence[torch.Tensor]], host_outputs: Sequence) -> None:
        """Step i reads host_inputs[i] (pinned tensors) and writes host_outputs[i] (pinned; a list
        when the outputs are)."""
        n = len(host_inputs)
        if len(host_outputs) != n:
            raise ValueError("one host output per step")
        if n == 0:
            return
        main = torch.cuda.current_stream(self.device)
        # nothing of this run starts before the work already on the caller's stream
        self.up.wait_stream(main)
        self.down.wait_stream(main)
        self._upload(0, host_inputs[0])
        for i in range(n):
            b = i % 2
            if i + 1 < n:
                self._upload(i + 1, host_inputs[i + 1])
            main.wait_event(self.ev_up[b])
            if i >= 2:
                main.wait_event(self.ev_down[b])
            outs = self.outputs[b]
            self.compute(i, self.inputs[b], outs if self.multi else outs[0])
            self.ev_comp[b].record(main)
            with torch.cuda.stream(self.down):
                self.down.wait_event(self.ev_comp[b])
                dst = host_outputs[i] if self.multi else [host_outputs[i]]
                for h, d in zip(dst, self.outputs[b]):
                    h.copy_(d, non_blocking=True)
                self.ev_down[b].record(self.down)
        main.wait_event(self.ev_down[(n - 1) % 2])
        if n >= 2:
            main.wait_event(self.ev_down[(n - 2) % 2])
