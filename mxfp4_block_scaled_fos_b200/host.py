"""Rowwise quantization of a batch that lives in pinned host memory, with the
outputs returned to pinned host memory: the binding of fos_quantize_host
(include/fos.h).

The library moves the batch in chunks of entries on three CUDA streams, so
that the host-to-device copy of chunk k + 1, the quantization of chunk k and
the device-to-host copy of chunk k - 1 are in flight together (PCIe carries
both directions at once).  This module owns the device staging buffers, the
streams and the events the call needs, and marshals the arguments.  Each
batch entry has its own per-tensor scale and the stochastic-rounding
counters follow the global element index, so the results equal one
fos_quantize over the whole batch.

Source of the method: Hugging Face transformers doc "Four Over Six"
(introduction: NVFP4 with a per-block choice of 4 or 6); Ultralytics glossary
"FP4", "Como funciona FP4" (E4M3 block scales, FP32 per-tensor scale).
"""
from __future__ import annotations

import ctypes
from typing import Optional, Tuple

import torch

from . import fos


class HostQuantizer:
    """Quantizes [batch, rows, cols] bf16 from pinned host memory into pinned
    host codes [batch, rows, cols/2], scales [batch, rows, cols/bs] and (NVFP4)
    S_t [batch].  The device buffers, streams and events are made once here
    and reused by every call.  fmt: "nvfp4_46", "nvfp4_6" or "mxfp4";
    rounding: "rne" or "sr" (Philox keyed on seed and the element index);
    chunk: batch entries per pipeline stage."""

    def __init__(self, batch: int, rows: int, cols: int, fmt: str = "nvfp4_46", rounding: str = "rne",
                 seed: int = 0, chunk: int = 4, device="cuda"):
        if batch < 1 or chunk < 1:
            raise ValueError("batch and chunk must be positive")
        self.batch, self.rows, self.cols, self.chunk = batch, rows, cols, chunk
        self.fmt = fmt
        block = "1x32" if fmt == "mxfp4" else "1x16"
        self.opts = fos.Options(fos.FMT[fmt], fos.BLK[block], fos.RND[rounding], 0, seed, 0)
        bs = 32 if fmt == "mxfp4" else 16
        dev = torch.device(device)
        self.x = torch.empty(batch, rows, cols, dtype=torch.bfloat16, device=dev)
        self.codes = torch.empty(batch, rows, cols // 2, dtype=torch.uint8, device=dev)
        self.scales = torch.empty(batch, rows, cols // bs, dtype=torch.uint8, device=dev)
        self.ts = torch.empty(batch, dtype=torch.float32, device=dev) if fmt != "mxfp4" else None
        self.ws = torch.empty(fos.workspace_size(chunk, rows, cols), dtype=torch.uint8, device=dev)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        self.streams = [torch.cuda.Stream(device=dev) for _ in range(3)]
        nchunks = (batch + chunk - 1) // chunk
        self.events = [torch.cuda.Event() for _ in range(2 * nchunks)]
        for e in self.events:   # create the driver events now (torch creates them on first record)
            e.record(self.streams[0])
        self.events_c = (ctypes.c_void_p * len(self.events))(*[e.cuda_event for e in self.events])
        self.dev_q = fos.QTensorC(self.codes.data_ptr(), self.scales.data_ptr(),
                                  self.ts.data_ptr() if self.ts is not None else None, None, cols // 2, cols // bs)
        torch.cuda.synchronize(dev)

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
        for s in self.streams:
            s.wait_stream(main)
        host_q = fos.QTensorC(h_codes.data_ptr(), h_scales.data_ptr(),
                              h_ts.data_ptr() if self.ts is not None else None, None,
                              self.codes.shape[2], self.scales.shape[2])
        st = fos.lib().fos_quantize_host(
            ctypes.c_void_p(h_x.data_ptr()), self.batch, self.rows, self.cols, ctypes.byref(self.opts), None,
            ctypes.byref(host_q), ctypes.c_void_p(self.x.data_ptr()), ctypes.byref(self.dev_q),
            ctypes.c_void_p(self.ws.data_ptr()), self.ws.numel(), ctypes.c_void_p(self.status.data_ptr()),
            self.chunk, ctypes.c_void_p(self.streams[0].cuda_stream),
            ctypes.c_void_p(self.streams[1].cuda_stream), ctypes.c_void_p(self.streams[2].cuda_stream),
            self.events_c)
        if st != 0:
            raise fos.FosError(st, "fos_quantize_host")
        main.wait_stream(self.streams[2])
