"""The fused amax + quantize kernel's bounded waits give up and report
FOS_STATUS_TIMEOUT instead of hanging.  The failure is planted on the host
(include/fos_testing.h): one batch entry's amax never counts in, and the
spin limit is set to a few thousand polls.  The launch must end, the status
word must carry the timeout bit, the entries before the stalled one must
still be exact against the oracle, and the context must stay usable."""
import ctypes
import time

import numpy as np
import pytest
import torch

import oracle
import mxfp4_block_scaled_fos_b200 as F
from mxfp4_block_scaled_fos_b200.fos import Options

from helpers import assert_bytes_equal, check_quantize, np_bits, require_gpu, zeroed_out

pytestmark = pytest.mark.gpu


def _input(batch, rows, cols, dev):
    g = torch.Generator().manual_seed(41)
    s = torch.exp2(torch.randint(-6, 6, (batch, 1, 1), generator=g).float())
    return (torch.randn(batch, rows, cols, generator=g) * s).to(torch.bfloat16).to(dev)


def _stalled(x, out, ws, status, stall_entry, spin_limit, fmt=0, blk=0):
    batch, rows, cols = x.shape
    rc = out.c_struct()
    return F.lib().fos_testing_quantize_stalled(
        ctypes.c_void_p(x.data_ptr()), batch, rows, cols, cols, ctypes.byref(Options(fmt, blk, 0, 0, 0, 0)),
        ctypes.byref(rc), ctypes.c_void_p(ws.data_ptr()), ws.numel(), ctypes.c_void_p(status.data_ptr()),
        stall_entry, spin_limit, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def test_fused_wait_runs_out_and_reports_timeout():
    dev = require_gpu()
    batch, rows, cols, stall = 6, 96, 512, 3
    x = _input(batch, rows, cols, dev)
    nblk = rows * cols // 16
    out = zeroed_out(batch, rows, cols, "nvfp4_46", "1x16", 0, dev, batch * nblk)
    ws = torch.zeros(F.workspace_size(batch, rows, cols), dtype=torch.uint8, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    t0 = time.time()
    assert _stalled(x, out, ws, status, stall, 2000) == 0
    torch.cuda.synchronize()
    assert time.time() - t0 < 60
    assert int(status.item()) & F.STATUS_TIMEOUT, "no timeout reported"
    ref = oracle.quantize(np_bits(x))
    keep = list(range(stall))
    assert_bytes_equal(out.codes.cpu().numpy()[keep], ref["r_codes"][keep], "codes")
    assert_bytes_equal(out.scales.cpu().numpy()[keep], ref["r_scales"][keep], "scales")
    assert_bytes_equal(out.tensor_scale.cpu().numpy()[keep].view(np.uint32),
                       ref["tensor_scale"][keep].view(np.uint32), "S_t")
    got = np.unpackbits(out.choice.cpu().numpy(), bitorder="little")[: batch * nblk].reshape(batch, nblk)
    want = np.unpackbits(ref["r_choice"], bitorder="little")[: batch * nblk].reshape(batch, nblk)
    assert np.array_equal(got[keep], want[keep])
    # the context is still usable and a normal call is exact, with no status
    check_quantize(x)


def test_stall_hook_argument_errors():
    dev = require_gpu()
    x = _input(2, 16, 64, dev)
    out = zeroed_out(2, 16, 64, "nvfp4_46", "1x16", 0, dev, 128)
    ws = torch.zeros(F.workspace_size(2, 16, 64), dtype=torch.uint8, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    assert _stalled(x, out, ws, status, 2, 100) == 7      # entry out of range
    assert _stalled(x, out, ws, status, 0, 0) == 7        # no polls
    assert _stalled(x, out, ws, status, 0, 100, blk=1) == 4
    torch.cuda.synchronize()
    assert int(status.item()) == 0
