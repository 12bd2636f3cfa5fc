"""Fake quantization (fos_fake_quantize): quantize and dequantize in one
kernel, bf16 out, without writing codes or scales -- the simulated-FP4 path
of the Hugging Face transformers doc "Four Over Six" (introduction).  Every
output must equal the oracle's dequantize of the oracle's quantize of the
same bf16 input, bit for bit."""
import numpy as np
import pytest
import torch

import oracle
import mxfp4_block_scaled_fos_b200 as F

from helpers import FMT_O, RND_O, assert_bytes_equal, np_bits, require_gpu

pytestmark = pytest.mark.gpu


def _input(shape, seed, dev):
    g = torch.Generator().manual_seed(seed)
    s = torch.exp2(torch.randint(-10, 10, shape[:-1] + (1,), generator=g).float())
    x = torch.randn(shape, generator=g) * s
    x.view(-1)[::53] *= 25
    return x.to(torch.bfloat16).to(dev)


def _reference(xb, fmt, rounding, rht, seed, elem_offset=0, amax=None):
    blk = oracle.BLK_1X32 if fmt == "mxfp4" else oracle.BLK_1X16
    q = oracle.quantize(xb, fmt=FMT_O[fmt], blk=blk, rnd=RND_O[rounding], rht=rht, seed=seed,
                        elem_offset=elem_offset, amax_in=amax)
    return oracle.dequantize(q["r_codes"], q["r_scales"], q["tensor_scale"], FMT_O[fmt])


@pytest.mark.parametrize("shape", [(1, 64, 256), (3, 48, 400), (2, 1, 16 * 37), (1, 300, 1024)])
@pytest.mark.parametrize("fmt,rounding,rht", [("nvfp4_46", "rne", False), ("nvfp4_6", "rne", False),
                                              ("nvfp4_46", "sr", False), ("nvfp4_46", "rne", True),
                                              ("nvfp4_6", "sr", True)])
@pytest.mark.parametrize("supply_amax", [False, True])
def test_fake_quant_equals_dequantize_of_quantize(shape, fmt, rounding, rht, supply_amax):
    dev = require_gpu()
    x = _input(shape, shape[1] * 31 + shape[2], dev)
    amax = F.amax(x, rht=rht, seed=7) if supply_amax else None
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    y = F.fake_quantize(x, fmt=fmt, rounding=rounding, rht=rht, seed=7, amax=amax, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    want = _reference(np_bits(x), fmt, rounding, rht, 7, amax=amax.cpu().numpy() if amax is not None else None)
    assert_bytes_equal(np_bits(y), want, "fake-quantized bf16")


@pytest.mark.parametrize("shape", [(1, 64, 256), (2, 33, 320)])
def test_fake_quant_mxfp4(shape):
    dev = require_gpu()
    x = _input(shape, 5, dev)
    y = F.fake_quantize(x, fmt="mxfp4")
    torch.cuda.synchronize()
    assert_bytes_equal(np_bits(y), _reference(np_bits(x), "mxfp4", "rne", False, 0), "MXFP4 fake-quantized")


def test_fake_quant_strided_rows_and_sr_offset():
    dev = require_gpu()
    xf = _input((2, 40, 384), 9, dev)
    x = xf[:, :, :256]
    yf = torch.full((2, 40, 320), 7.0, dtype=torch.bfloat16, device=dev)
    y = yf[:, :, :256]
    F.fake_quantize(x, rounding="sr", seed=3, elem_offset=16 * 999, out=y)
    torch.cuda.synchronize()
    want = _reference(np_bits(x.contiguous()), "nvfp4_46", "sr", False, 3, elem_offset=16 * 999)
    assert_bytes_equal(np_bits(y.contiguous()), want, "strided fake-quantized")
    assert torch.all(yf[:, :, 256:] == 7.0), "wrote past the row"


def test_fake_quant_moe_experts_sampled():
    """The full 128 x 2880 x 2880 expert batch through the fused kernel;
    three experts checked against the oracle."""
    dev = require_gpu()
    from mxfp4_block_scaled_fos_b200 import workloads
    x = workloads.moe_experts(128, 2880, 2880, device=dev)
    y = F.fake_quantize(x)
    torch.cuda.synchronize()
    for e in (0, 77, 127):
        want = _reference(np_bits(x[e:e + 1]), "nvfp4_46", "rne", False, 0)
        assert_bytes_equal(np_bits(y[e:e + 1]), want, "expert %d" % e)
