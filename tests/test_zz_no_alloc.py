"""fos_quantize_static: the quantizer for callers that cannot allocate device
memory (code inside a stream capture, serving paths that must not allocate,
hosts whose allocator hands out no scratch).  Its scratch lives in a fixed
array inside the library instead of a caller workspace.

Checked through the C ABI against fos_quantize with its own workspace, on two
calls in a row whose inputs differ, so that anything the first call left in
the shared array would show in the second.  This file is collected last and
needs no state from other tests.
"""
import ctypes

import numpy as np
import pytest
import torch

import mxfp4_block_scaled_fos_b200 as F
from mxfp4_block_scaled_fos_b200.fos import Options

from helpers import require_gpu, zeroed_out

pytestmark = pytest.mark.gpu

FOS_STATIC_MAX_BATCH = 4096  # include/fos.h


def _input(shape, seed, scale, dev):
    g = torch.Generator().manual_seed(seed)
    z = torch.randn(shape, generator=g)
    c = sum(torch.randn(shape, generator=g) ** 2 for _ in range(3))
    return (z / torch.sqrt(c / 3) * scale).to(torch.bfloat16).to(dev)


def _run(x, opts, static, colwise, block):
    """One call through the C ABI; returns (row, col) output tensors."""
    batch, rows, cols = x.shape
    nb = batch * (rows // 16) * (cols // 16) if block == "16x16" else batch * rows * (cols // 16)
    nbc = nb if block == "16x16" else batch * cols * (rows // 16)
    r = zeroed_out(batch, rows, cols, "nvfp4_46", block, 0, x.device, nb)
    c = zeroed_out(batch, cols, rows, "nvfp4_46", block, 0, x.device, nbc) if colwise else None
    rc = r.c_struct()
    cc = c.c_struct() if c is not None else None
    status = torch.zeros(1, dtype=torch.int32, device=x.device)
    L = F.lib()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    args = (ctypes.c_void_p(x.data_ptr()), batch, rows, cols, x.stride(1), ctypes.byref(opts), None,
            ctypes.byref(rc), ctypes.byref(cc) if cc is not None else None)
    if static:
        st = L.fos_quantize_static(*args, ctypes.c_void_p(status.data_ptr()), stream)
    else:
        ws = torch.empty(F.workspace_size(batch, rows, cols), dtype=torch.uint8, device=x.device)
        st = L.fos_quantize(*args, ctypes.c_void_p(ws.data_ptr()), ws.numel(),
                            ctypes.c_void_p(status.data_ptr()), stream)
    assert st == 0, F.status_string(st)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return r, c


def _same(a, b):
    for name in ("codes", "scales", "tensor_scale", "choice"):
        ta, tb = getattr(a, name), getattr(b, name)
        assert torch.equal(ta.view(torch.uint8), tb.view(torch.uint8)), name


@pytest.mark.parametrize("block,rounding,colwise", [("1x16", "rne", False), ("1x16", "sr", True),
                                                    ("16x16", "rne", True)])
def test_static_scratch_matches_workspace_twice(block, rounding, colwise):
    dev = require_gpu()
    opts = Options(0, {"1x16": 0, "16x16": 1}[block], {"rne": 0, "sr": 1}[rounding], 0, 7, 0)
    # the first input has much larger amaxes than the second: stale amax
    # words in the shared array would change the second call's scales
    for seed, scale in ((1, 10.0), (2, 1e-3)):
        x = _input((3, 64, 256), seed, scale, dev)
        got = _run(x, opts, True, colwise, block)
        want = _run(x, opts, False, colwise, block)
        _same(got[0], want[0])
        if colwise:
            _same(got[1], want[1])


def test_static_scratch_rejects_batch_beyond_limit():
    dev = require_gpu()
    x = torch.zeros(FOS_STATIC_MAX_BATCH + 1, 16, 16, dtype=torch.bfloat16, device=dev)
    r = zeroed_out(x.shape[0], 16, 16, "nvfp4_46", "1x16", 0, dev, x.shape[0] * 16)
    rc = r.c_struct()
    st = F.lib().fos_quantize_static(ctypes.c_void_p(x.data_ptr()), x.shape[0], 16, 16, 16,
                                     ctypes.byref(Options(0, 0, 0, 0, 0, 0)), None,
                                     ctypes.byref(rc), None, None,
                                     ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 5  # FOS_ERR_WORKSPACE


def test_static_scratch_limit_applies_only_to_calls_that_use_scratch():
    """MXFP4 calls and calls with a caller-supplied amax need no scratch, so
    they take a batch beyond the limit and match fos_quantize."""
    dev = require_gpu()
    batch = FOS_STATIC_MAX_BATCH + 3
    x = _input((batch, 16, 32), 5, 1.0, dev)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    amax = F.amax(x)
    for fmt, blk, use_amax in ((2, 2, False), (0, 0, True)):
        name = "mxfp4" if fmt == 2 else "nvfp4_46"
        block = "1x32" if fmt == 2 else "1x16"
        outs = []
        for static in (True, False):
            r = zeroed_out(batch, 16, 32, name, block, 0, dev, batch * 16 * 2)
            rc = r.c_struct()
            args = (ctypes.c_void_p(x.data_ptr()), batch, 16, 32, 32, ctypes.byref(Options(fmt, blk, 0, 0, 0, 0)),
                    ctypes.c_void_p(amax.data_ptr()) if use_amax else None, ctypes.byref(rc), None)
            if static:
                st = F.lib().fos_quantize_static(*args, None, stream)
            else:
                st = F.lib().fos_quantize(*args, None, 0, None, stream)
            assert st == 0, F.status_string(st)
            outs.append(r)
        torch.cuda.synchronize()
        for name_ in ("codes", "scales"):
            assert torch.equal(getattr(outs[0], name_), getattr(outs[1], name_)), name_
        if fmt == 0:
            assert torch.equal(outs[0].tensor_scale, outs[1].tensor_scale)
            assert torch.equal(outs[0].choice, outs[1].choice)
