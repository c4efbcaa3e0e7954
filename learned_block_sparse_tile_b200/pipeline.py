"""Host-to-host execution of consecutive, independent Veda layer calls with the transfers overlapped.

A layer call on host-resident inputs moves 3 S H D bf16 in and S H D bf16 out over PCIe, which at 104k
tokens takes longer than the layer itself. ``HostPipeline`` keeps two device copies of the inputs and
outputs and runs three streams: uploads, the layer's kernels, downloads. While call i computes, call
i + 1's Q/K/V are uploaded and call i - 1's output is downloaded, so a sequence of calls (independent
requests; each call's inputs must not depend on an earlier call's output) costs per call about the
largest of the three, not their sum. The arithmetic is the layer's own (``VedaLayer.forward``); this
module only orders copies and launches with CUDA events.
"""
from __future__ import annotations

import torch


class HostPipeline:
    """Double-buffered upload / compute / download of ``VedaLayer`` calls on pinned host tensors."""

    def __init__(self, layer, seq_len, heads, dim, device="cuda"):
        self.layer = layer
        self.device = torch.device(device)
        shape = (seq_len, heads, dim)
        self.d_in = [[torch.empty(shape, dtype=torch.bfloat16, device=self.device) for _ in range(3)]
                     for _ in range(2)]
        self.d_out = [torch.empty(shape, dtype=torch.bfloat16, device=self.device) for _ in range(2)]
        self.up = torch.cuda.Stream(self.device)
        self.down = torch.cuda.Stream(self.device)
        # per slot: inputs uploaded / inputs consumed by the layer / output written / output downloaded
        self._ev = [{k: torch.cuda.Event() for k in ("in_ready", "in_free", "out_ready", "out_free")}
                    for _ in range(2)]

    def run(self, inputs, outputs, stream=None):
        """Enqueues one layer call per element of ``inputs`` and returns without waiting.

        inputs: sequence of (q, k, v) bf16 [S, H, D] pinned host tensors; outputs: same-length sequence of
        pinned host bf16 [S, H, D] tensors, written in order (the same tensor may repeat: its downloads are
        ordered). ``stream`` (default: the current stream) runs the layer's kernels and, when this returns,
        is ordered after the last download, so work enqueued on it later sees every output."""
        if len(inputs) != len(outputs):
            raise ValueError("HostPipeline.run: one output tensor per call")
        for t in [x for qkv in inputs for x in qkv] + list(outputs):
            if t.device.type != "cpu" or not t.is_pinned():
                raise ValueError("HostPipeline.run: host tensors must be pinned CPU memory")
            if t.dtype != torch.bfloat16 or tuple(t.shape) != tuple(self.d_out[0].shape):
                raise ValueError("HostPipeline.run: tensors must be bf16 of the pipeline's [S, H, D] shape")
        comp = stream if stream is not None else torch.cuda.current_stream(self.device)
        start = torch.cuda.Event()
        start.record(comp)
        self.up.wait_event(start)
        self.down.wait_event(start)
        for i, (qkv, hout) in enumerate(zip(inputs, outputs)):
            s, ev = i & 1, self._ev[i & 1]
            if i >= 2:
                self.up.wait_event(ev["in_free"])  # call i - 2 no longer reads this slot's inputs
            with torch.cuda.stream(self.up):
                for d, h in zip(self.d_in[s], qkv):
                    d.copy_(h, non_blocking=True)
            ev["in_ready"].record(self.up)
            comp.wait_event(ev["in_ready"])
            if i >= 2:
                comp.wait_event(ev["out_free"])  # call i - 2's output has left this slot
            dq, dk, dv = self.d_in[s]
            self.layer.forward(dq, dk, dv, self.d_out[s], stream=comp)
            ev["in_free"].record(comp)
            ev["out_ready"].record(comp)
            self.down.wait_event(ev["out_ready"])
            with torch.cuda.stream(self.down):
                hout.copy_(self.d_out[s], non_blocking=True)
            ev["out_free"].record(self.down)
        end = torch.cuda.Event()
        end.record(self.down)
        comp.wait_event(end)
        self.up.wait_event(end)
