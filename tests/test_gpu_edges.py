"""GPU edge cases through the C ABI: empty tensors, one block, many tiny
batch entries (the fused amax + quantize queue with one item of each kind
per entry), a few entries with several ragged items each in dense,
strided and swizzled layouts, and the largest block counts a 16-bit batch
index allows with small entries.  Checked bit for bit against the oracle
where there is output."""
import ctypes

import numpy as np
import pytest
import torch

import mxfp4_block_scaled_fos_b200 as F
from mxfp4_block_scaled_fos_b200.fos import Options

from helpers import check_quantize, np_bits, require_gpu, zeroed_out

pytestmark = pytest.mark.gpu


def _call(x, batch, rows, cols, out, fmt=0, blk=0):
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws = torch.zeros(F.workspace_size(max(batch, 1), max(rows, 1), max(cols, 1)), dtype=torch.uint8,
                     device="cuda")
    rc = out.c_struct()
    st = F.lib().fos_quantize(ctypes.c_void_p(x.data_ptr()), batch, rows, cols, max(cols, 16),
                              ctypes.byref(Options(fmt, blk, 0, 0, 0, 0)), None, ctypes.byref(rc), None,
                              ctypes.c_void_p(ws.data_ptr()), ws.numel(), ctypes.c_void_p(status.data_ptr()),
                              ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    torch.cuda.synchronize()
    return st, int(status.item())


@pytest.mark.parametrize("batch,rows,cols", [(0, 16, 32), (2, 0, 32), (2, 16, 0)])
def test_empty_tensors_are_a_no_op(batch, rows, cols):
    require_gpu()
    x = torch.zeros(max(batch, 1) * max(rows, 1) * max(cols, 16), dtype=torch.bfloat16, device="cuda")
    out = zeroed_out(max(batch, 1), max(rows, 1), max(cols, 16), "nvfp4_46", "1x16", 0, x.device, 64)
    out.codes.fill_(0xA5)
    out.scales.fill_(0xA5)
    st, status = _call(x, batch, rows, cols, out)
    assert st == 0 and status == 0
    assert bool((out.codes == 0xA5).all()) and bool((out.scales == 0xA5).all())


@pytest.mark.parametrize("fmt", ["nvfp4_46", "nvfp4_6", "mxfp4"])
def test_single_block(fmt):
    require_gpu()
    g = torch.Generator().manual_seed(5)
    cols = 32 if fmt == "mxfp4" else 16
    x = (torch.randn(1, 1, cols, generator=g) * 3).to(torch.bfloat16).cuda()
    check_quantize(x, fmt=fmt)


@pytest.mark.parametrize("rounding", ["rne", "sr"])
def test_many_tiny_entries_through_the_fused_queue(rounding):
    """300 entries of 2 x 32: one amax item and one quantize item each, so
    the queue runs 600 items over hundreds of lag phases; the per-entry
    scales span 2^-20 .. 2^20."""
    require_gpu()
    g = torch.Generator().manual_seed(6)
    x = torch.randn(300, 2, 32, generator=g)
    x *= torch.exp2(torch.randint(-20, 21, (300, 1, 1), generator=g).float())
    check_quantize(x.to(torch.bfloat16).cuda(), rounding=rounding, seed=3)


def test_entries_with_all_zero_and_all_tiny_values_in_one_batch():
    """Entry amaxes of 0, a bf16 subnormal-range value and a normal value in
    one fused call: S_t = 0 for the zero entry, subnormal-range S_t for the
    tiny one."""
    require_gpu()
    g = torch.Generator().manual_seed(7)
    x = torch.randn(3, 16, 64, generator=g)
    x[0] = 0.0
    x[1] *= 1e-39
    check_quantize(x.to(torch.bfloat16).cuda())


@pytest.mark.parametrize("layout", ["dense", "ragged_words", "strided", "swizzled"])
@pytest.mark.parametrize("fmt", ["nvfp4_46", "nvfp4_6"])
def test_fused_queue_several_items_per_entry(layout, fmt):
    """Three entries with several amax and quantize items each and a ragged
    last item, so that with a lag of two entries the middle entry's items
    interleave with both neighbours' in the queue.  dense: 72 x 1024 (4608
    blocks, whole choice words per entry: the dense loop); ragged_words:
    70 x 1040 (4550 blocks, choice words that straddle entries); strided:
    the same rows read with ld = 1104; swizzled: swizzled scales.  The
    per-entry scales differ by up to 2^12."""
    require_gpu()
    g = torch.Generator().manual_seed(8)
    rows, cols = (72, 1024) if layout == "dense" else (70, 1040)
    big = torch.randn(3, rows, 1104, generator=g)
    big *= torch.exp2(torch.randint(-6, 7, (3, 1, 1), generator=g).float())
    big = big.to(torch.bfloat16).cuda()
    if layout == "strided":
        x = big[:, :, :cols]
        assert x.stride(1) == 1104
        check_quantize(x, fmt=fmt, x_bits=np_bits(x.contiguous()))
    else:
        check_quantize(big[:, :, :cols].contiguous(), fmt=fmt, swizzle=layout == "swizzled")
