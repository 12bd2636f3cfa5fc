"""GPU parity at the full workload sizes, in the launch configuration the
benchmark times.  Where the oracle cannot redo the whole tensor in seconds,
sampled slices are compared: the oracle computes the tensor amax itself
(a cheap full pass), then quantizes the sampled rows or experts with that
amax and the matching element offset, and the GPU's outputs for those
slices must equal it bit for bit."""
import numpy as np
import pytest
import torch

import oracle
import mxfp4_block_scaled_fos_b200 as F
from mxfp4_block_scaled_fos_b200 import workloads

from helpers import assert_bytes_equal, compare_choice, require_gpu

pytestmark = pytest.mark.gpu


def _slice_check(q_gpu, ref, r0, r1, tag, block_cols, fmt_mx=False):
    """Compare rows [r0, r1) of a GPU orientation with the oracle slice."""
    assert_bytes_equal(q_gpu.codes[0, r0:r1].cpu().numpy(), ref[tag + "_codes"][0], tag + "_codes")
    assert_bytes_equal(q_gpu.scales[0, r0:r1].cpu().numpy(), ref[tag + "_scales"][0], tag + "_scales")


def test_weight_normal_2d_full():
    """14336x4096 N(0, 0.02^2): 16x16 2D 4/6, rowwise + transposed, whole tensor."""
    dev = require_gpu()
    x = workloads.weight_normal(14336, 4096, device=dev)
    r, c = F.quantize(x, block="16x16", colwise=True)
    torch.cuda.synchronize()
    ref = oracle.quantize(workloads.bits(x), blk=oracle.BLK_16X16, colwise=True)
    assert_bytes_equal(r.codes.cpu().numpy(), ref["r_codes"], "r_codes")
    assert_bytes_equal(r.scales.cpu().numpy(), ref["r_scales"], "r_scales")
    assert_bytes_equal(c.codes.cpu().numpy(), ref["c_codes"], "c_codes")
    assert_bytes_equal(c.scales.cpu().numpy(), ref["c_scales"], "c_scales")
    assert r.tensor_scale.cpu().numpy().view(np.uint32)[0] == ref["tensor_scale"].view(np.uint32)[0]
    compare_choice(r.choice, ref["r_choice"], (14336 // 16) * (4096 // 16), "r")
    compare_choice(c.choice, ref["c_choice"], (14336 // 16) * (4096 // 16), "c")


def test_gradient_student_t_sr_dual_sampled():
    """16384x8192 Student-t(3)*1e-3, SR (seed 0), both orientations; three
    512-row strips compared (rowwise rows and the matching colwise blocks)."""
    dev = require_gpu()
    R, C = 16384, 8192
    x = workloads.gradient_student_t(R, C, device=dev)
    r, c = F.quantize(x, rounding="sr", seed=0, colwise=True)
    torch.cuda.synchronize()
    xb = workloads.bits(x)
    A = oracle.amax(xb)
    assert r.tensor_scale.cpu().numpy().view(np.uint32)[0] == \
        np.float32(A[0] / np.float32(1792)).view(np.uint32)
    for r0 in (0, 7680, R - 512):
        sl = np.ascontiguousarray(xb[:, r0:r0 + 512])
        ref = oracle.quantize(sl, rnd=oracle.RND_SR, seed=0, elem_offset=r0 * C, colwise=True,
                              amax_in=A)
        assert_bytes_equal(r.codes[0, r0:r0 + 512].cpu().numpy(), ref["r_codes"][0], "r_codes")
        assert_bytes_equal(r.scales[0, r0:r0 + 512].cpu().numpy(), ref["r_scales"][0], "r_scales")
        # colwise: every column, row groups r0/16 .. r0/16 + 31
        assert_bytes_equal(c.codes[0, :, r0 // 2:(r0 + 512) // 2].cpu().numpy(), ref["c_codes"][0], "c_codes")
        assert_bytes_equal(c.scales[0, :, r0 // 16:(r0 + 512) // 16].cpu().numpy(), ref["c_scales"][0], "c_scales")
        g = np.unpackbits(r.choice.cpu().numpy(), bitorder="little")[r0 * (C // 16):(r0 + 512) * (C // 16)]
        w = np.unpackbits(ref["r_choice"], bitorder="little")[:512 * (C // 16)]
        assert np.array_equal(g, w)


def test_activation_rht_full():
    """8192x4096 activations with 1% outlier channels, RHT16 seed 0, whole tensor."""
    dev = require_gpu()
    x = workloads.activation_outliers(8192, 4096, device=dev)
    r, _ = F.quantize(x, rht=True, seed=0)
    torch.cuda.synchronize()
    ref = oracle.quantize(workloads.bits(x), rht=True, seed=0)
    assert_bytes_equal(r.codes.cpu().numpy(), ref["r_codes"], "r_codes")
    assert_bytes_equal(r.scales.cpu().numpy(), ref["r_scales"], "r_scales")
    compare_choice(r.choice, ref["r_choice"], 8192 * 4096 // 16, "r")


@pytest.fixture(scope="module")
def moe():
    dev = require_gpu()
    x = workloads.moe_experts(128, 2880, 2880, device=dev)
    return x


@pytest.mark.parametrize("fmt", ["nvfp4_46", "nvfp4_6", "mxfp4"])
def test_moe_experts_sampled(moe, fmt):
    """128x2880x2880 experts: the full GPU launch, three experts compared."""
    x = moe
    r, _ = F.quantize(x, fmt=fmt)
    y = F.dequantize(r)
    torch.cuda.synchronize()
    fo = {"nvfp4_46": oracle.FMT_NVFP4_46, "nvfp4_6": oracle.FMT_NVFP4_6, "mxfp4": oracle.FMT_MXFP4}[fmt]
    blk = oracle.BLK_1X32 if fmt == "mxfp4" else oracle.BLK_1X16
    for e in (0, 63, 127):
        xe = workloads.bits(x[e:e + 1])
        ref = oracle.quantize(xe, fmt=fo, blk=blk)
        assert_bytes_equal(r.codes[e:e + 1].cpu().numpy(), ref["r_codes"], "codes e%d" % e)
        assert_bytes_equal(r.scales[e:e + 1].cpu().numpy(), ref["r_scales"], "scales e%d" % e)
        if fmt != "mxfp4":
            assert r.tensor_scale[e].cpu().numpy().view(np.uint32) == ref["tensor_scale"].view(np.uint32)[0]
        yref = oracle.dequantize(ref["r_codes"], ref["r_scales"], ref["tensor_scale"], fmt=fo)
        assert_bytes_equal(workloads.bits(y[e:e + 1]), yref, "dequant e%d" % e)
        if fmt == "nvfp4_46":
            n = 2880 * 180
            g = np.unpackbits(r.choice.cpu().numpy(), bitorder="little")[e * n:(e + 1) * n]
            assert np.array_equal(g, np.unpackbits(ref["r_choice"], bitorder="little")[:n])
