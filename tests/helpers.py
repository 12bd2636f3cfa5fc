"""Shared helpers for the GPU parity tests: run the CUDA path through the
C ABI binding and the CPU oracle on the same bf16 bytes, compare bit for bit."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import mxfp4_block_scaled_fos_b200 as F
from mxfp4_block_scaled_fos_b200 import workloads

FMT_O = {"nvfp4_46": oracle.FMT_NVFP4_46, "nvfp4_6": oracle.FMT_NVFP4_6, "mxfp4": oracle.FMT_MXFP4}
BLK_O = {"1x16": oracle.BLK_1X16, "16x16": oracle.BLK_16X16, "1x32": oracle.BLK_1X32}
RND_O = {"rne": oracle.RND_RNE, "sr": oracle.RND_SR}


def require_gpu():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return torch.device("cuda:0")


def np_bits(t: torch.Tensor) -> np.ndarray:
    return workloads.bits(t)


def n_blocks(batch, R, C, block):
    if block == "16x16":
        return batch * (R // 16) * (C // 16)
    return batch * R * (C // (32 if block == "1x32" else 16))


def compare_choice(gpu: torch.Tensor, ref: np.ndarray, nblocks: int, what=""):
    g = np.unpackbits(gpu.cpu().numpy(), bitorder="little")[:nblocks]
    r = np.unpackbits(ref, bitorder="little")[:nblocks]
    bad = np.nonzero(g != r)[0]
    assert bad.size == 0, "%s choice bits differ at %s" % (what, bad[:8])


def assert_bytes_equal(gpu: np.ndarray, ref: np.ndarray, what: str):
    gpu = np.asarray(gpu)
    ref = np.asarray(ref)
    assert gpu.shape == ref.shape, (what, gpu.shape, ref.shape)
    bad = np.argwhere(gpu != ref)
    assert bad.size == 0, "%s differs at %d positions, first %s: gpu %s ref %s" % (
        what, len(bad), bad[:4].tolist(), gpu[tuple(bad[0])], ref[tuple(bad[0])])


def zeroed_out(batch, R, C, fmt, block, flags, device, nblocks, choice=True):
    """Pre-zeroed output buffers (so unwritten swizzle padding compares as 0)."""
    bs = 32 if fmt == "mxfp4" else 16
    codes = torch.zeros(batch, R, C // 2, dtype=torch.uint8, device=device)
    if flags & F.FLAG_SCALE_SWIZZLED:
        scales = torch.zeros(batch, F.scales_size(R, C // bs, flags), dtype=torch.uint8, device=device)
    else:
        scales = torch.zeros(batch, R, C // bs, dtype=torch.uint8, device=device)
    ts = torch.zeros(batch, dtype=torch.float32, device=device) if fmt != "mxfp4" else None
    ch = None
    if choice and fmt == "nvfp4_46":
        ch = torch.zeros(8 * ((nblocks + 63) // 64), dtype=torch.uint8, device=device)
    return F.QTensor(codes, scales, ts, ch, batch, R, C, fmt, block, flags)


def quantize_2d_strip(x3, opts, amax, orow, ocol, status, nsub):
    """fos_testing_quantize_2d_strip (include/fos_testing.h): fos_quantize
    with the 2D kernel's strip length forced to nsub sub-tiles."""
    import ctypes
    batch, R, C = x3.shape
    ws = torch.zeros(F.workspace_size(batch, R, C), dtype=torch.uint8, device=x3.device)
    rc = orow.c_struct() if orow is not None else None
    cc = ocol.c_struct() if ocol is not None else None
    st = F.lib().fos_testing_quantize_2d_strip(
        ctypes.c_void_p(x3.data_ptr()), batch, R, C, x3.stride(1), ctypes.byref(opts),
        ctypes.c_void_p(amax.data_ptr()) if amax is not None else None,
        ctypes.byref(rc) if rc is not None else None, ctypes.byref(cc) if cc is not None else None,
        ctypes.c_void_p(ws.data_ptr()), ws.numel(), ctypes.c_void_p(status.data_ptr()), nsub,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, F.ERRORS.get(st, st)


def check_quantize(x: torch.Tensor, fmt="nvfp4_46", block=None, rounding="rne", rht=False,
                   swizzle=False, seed=0, elem_offset=0, rowwise=True, colwise=False,
                   amax=None, x_bits=None, rht_col=False, strip_2d=None):
    """Quantize x on the GPU and with the oracle; assert bit equality of
    codes, scales, tensor scales and choice bits.  Returns the GPU outputs.
    strip_2d: run the 16x16 kernel with that many sub-tiles per strip."""
    block = block or ("1x32" if fmt == "mxfp4" else "1x16")
    x3 = x if x.dim() == 3 else x.unsqueeze(0)
    batch, R, C = x3.shape
    flags = (F.FLAG_RHT16 if rht else 0) | (F.FLAG_SCALE_SWIZZLED if swizzle else 0) | \
        (F.FLAG_RHT16_COL if rht_col else 0)
    orow = zeroed_out(batch, R, C, fmt, block, flags, x.device, n_blocks(batch, R, C, block)) \
        if rowwise else None
    ocol = zeroed_out(batch, C, R, fmt, block, flags, x.device,
                      n_blocks(batch, C, R, "1x16") if block == "1x16" else n_blocks(batch, R, C, block)) \
        if colwise else None
    status = torch.zeros(1, dtype=torch.int32, device=x.device)
    if strip_2d is None:
        F.quantize(x3, fmt=fmt, block=block, rounding=rounding, rht=rht, swizzle=swizzle, seed=seed,
                   elem_offset=elem_offset, rowwise=rowwise, colwise=colwise, amax=amax,
                   status=status, out_row=orow, out_col=ocol, rht_col=rht_col)
    else:
        from mxfp4_block_scaled_fos_b200.fos import BLK, FMT, RND, Options
        opts = Options(FMT[fmt], BLK[block], RND[rounding], flags, seed, elem_offset)
        quantize_2d_strip(x3, opts, amax, orow, ocol, status, strip_2d)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    xb = x_bits if x_bits is not None else np_bits(x3.contiguous() if x3.stride(1) != C else x3)
    ain = amax.cpu().numpy() if amax is not None else None
    ref = oracle.quantize(xb, fmt=FMT_O[fmt], blk=BLK_O[block], rnd=RND_O[rounding], rht=rht,
                          seed=seed, elem_offset=elem_offset, rowwise=rowwise, colwise=colwise,
                          amax_in=ain, rht_col=rht_col)
    for tag, q in (("r", orow), ("c", ocol)):
        if q is None:
            continue
        assert_bytes_equal(q.codes.cpu().numpy(), ref[tag + "_codes"], tag + "_codes")
        sc = ref[tag + "_scales"]
        if swizzle:
            sc = oracle.swizzle_scales(sc).reshape(batch, -1)
        assert_bytes_equal(q.scales.cpu().numpy(), sc, tag + "_scales")
        if fmt != "mxfp4":
            assert_bytes_equal(q.tensor_scale.cpu().numpy().view(np.uint32),
                               ref["tensor_scale" if tag == "r" else "c_tensor_scale"].view(np.uint32),
                               tag + "_tensor_scale")
        if q.choice is not None:
            nb = n_blocks(batch, q.rows, q.cols, block) if block != "16x16" else n_blocks(batch, R, C, block)
            compare_choice(q.choice, ref[tag + "_choice"], nb, tag)
    return orow, ocol, ref
