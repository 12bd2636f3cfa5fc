"""Rowwise quantization of a batch that lives in pinned host memory, with the
outputs returned to pinned host memory.

The batch moves in chunks of entries on three CUDA streams, so that the
host-to-device copy of chunk k + 1, the quantization of chunk k and the
device-to-host copy of chunk k - 1 are in flight together (PCIe carries both
directions at once).  This module only orders copies and launches; every
step of the quantization runs in libfos.so's kernels through fos.quantize,
one call per chunk.  Each batch entry has its own per-tensor scale and the
stochastic-rounding counters follow the global element index (elem_offset),
so the results equal one fos.quantize call over the whole batch.

Source of the method: Hugging Face transformers doc "Four Over Six"
(introduction: NVFP4 with a per-block choice of 4 or 6); Ultralytics glossary
"FP4", "Como funciona FP4" (E4M3 block scales, FP32 per-tensor scale).
"""
from __future__ import annotations

from typing import List, Optional, Tuple

import torch

from . import fos


class HostQuantizer:
    """Quantizes [batch, rows, cols] bf16 from pinned host memory into pinned
    host codes [batch, rows, cols/2], scales [batch, rows, cols/bs] and (NVFP4)
    S_t [batch].  Device buffers, streams and events are made once here and
    reused by every call.  fmt: "nvfp4_46", "nvfp4_6" or "mxfp4"; rounding:
    "rne" or "sr" (Philox keyed on seed and the element index); chunk:
    entries per pipeline stage."""

    def __init__(self, batch: int, rows: int, cols: int, fmt: str = "nvfp4_46", rounding: str = "rne",
                 seed: int = 0, chunk: int = 4, device="cuda"):
        if batch < 1 or chunk < 1:
            raise ValueError("batch and chunk must be positive")
        self.batch, self.rows, self.cols = batch, rows, cols
        self.fmt, self.rounding, self.seed = fmt, rounding, seed
        self.block = "1x32" if fmt == "mxfp4" else "1x16"
        bs = 32 if fmt == "mxfp4" else 16
        dev = torch.device(device)
        self.x = torch.empty(batch, rows, cols, dtype=torch.bfloat16, device=dev)
        self.codes = torch.empty(batch, rows, cols // 2, dtype=torch.uint8, device=dev)
        self.scales = torch.empty(batch, rows, cols // bs, dtype=torch.uint8, device=dev)
        self.ts = torch.empty(batch, dtype=torch.float32, device=dev) if fmt != "mxfp4" else None
        self.chunks: List[Tuple[int, int]] = [(c, min(c + chunk, batch)) for c in range(0, batch, chunk)]
        self.ws = torch.empty(fos.workspace_size(chunk, rows, cols), dtype=torch.uint8, device=dev)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        self.streams = [torch.cuda.Stream(device=dev) for _ in range(3)]
        n = len(self.chunks)
        self.ev_in = [torch.cuda.Event() for _ in range(n)]
        self.ev_q = [torch.cuda.Event() for _ in range(n)]

    def host_outputs(self) -> Tuple[torch.Tensor, torch.Tensor, Optional[torch.Tensor]]:
        """Pinned host buffers of the right shapes for __call__."""
        pin = dict(pin_memory=True)
        return (torch.empty(self.codes.shape, dtype=torch.uint8, **pin),
                torch.empty(self.scales.shape, dtype=torch.uint8, **pin),
                torch.empty(self.ts.shape, dtype=torch.float32, **pin) if self.ts is not None else None)

    def __call__(self, h_x: torch.Tensor, h_codes: torch.Tensor, h_scales: torch.Tensor,
                 h_ts: Optional[torch.Tensor] = None) -> None:
        """Enqueue one pass: h_x (pinned host bf16) -> h_codes, h_scales, h_ts
        (pinned host).  Ordered after the current stream's earlier work; the
        current stream waits for the last copy, so synchronizing it (or an
        event recorded on it) means the host outputs are complete.  The status
        word (self.status) collects the kernels' data-error bits."""
        if h_x.shape != self.x.shape or h_x.dtype != torch.bfloat16 or not h_x.is_pinned():
            raise ValueError("h_x must be pinned host bf16 of shape %s" % (tuple(self.x.shape),))
        for h, d in ((h_codes, self.codes), (h_scales, self.scales), (h_ts, self.ts)):
            if d is not None and (h is None or h.shape != d.shape or not h.is_pinned()):
                raise ValueError("host outputs must be pinned and shaped like host_outputs()")
        main = torch.cuda.current_stream(self.x.device)
        s_in, s_q, s_out = self.streams
        for s in self.streams:
            s.wait_stream(main)
        per_entry = self.rows * self.cols
        for k, (c0, c1) in enumerate(self.chunks):
            with torch.cuda.stream(s_in):
                self.x[c0:c1].copy_(h_x[c0:c1], non_blocking=True)
                self.ev_in[k].record(s_in)
            s_q.wait_event(self.ev_in[k])
            with torch.cuda.stream(s_q):
                q = fos.QTensor(self.codes[c0:c1], self.scales[c0:c1],
                                self.ts[c0:c1] if self.ts is not None else None, None, c1 - c0,
                                self.rows, self.cols, self.fmt, self.block, 0)
                fos.quantize(self.x[c0:c1], fmt=self.fmt, rounding=self.rounding, seed=self.seed,
                             elem_offset=c0 * per_entry, out_row=q, workspace=self.ws, status=self.status)
                self.ev_q[k].record(s_q)
            s_out.wait_event(self.ev_q[k])
            with torch.cuda.stream(s_out):
                h_codes[c0:c1].copy_(self.codes[c0:c1], non_blocking=True)
                h_scales[c0:c1].copy_(self.scales[c0:c1], non_blocking=True)
                if self.ts is not None:
                    h_ts[c0:c1].copy_(self.ts[c0:c1], non_blocking=True)
        main.wait_stream(s_out)
