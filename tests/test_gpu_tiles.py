"""GPU parity of the two-orientation quantizers against the oracle:
1x16 rowwise + colwise (x and x^T from one read) and 16x16 2D block scaling
with its exact transposed copy.  Shapes cover whole and ragged 64x128
sub-tiles, strips shorter and longer than 512 rows, batches, and the
bitmap layouts whose words are owned by one CTA or shared."""
import numpy as np
import pytest
import torch

import oracle
import mxfp4_block_scaled_fos_b200 as F

from helpers import check_quantize, np_bits, require_gpu

pytestmark = pytest.mark.gpu

SHAPES = [(1, 16, 16), (1, 64, 128), (2, 80, 272), (1, 512, 256), (1, 528, 400), (3, 1040, 128),
          (1, 1024, 1024)]


def _rand(shape, seed, dev, kind="heavy"):
    g = torch.Generator().manual_seed(seed)
    if kind == "heavy":
        z = torch.randn(shape, generator=g)
        c = sum(torch.randn(shape, generator=g) ** 2 for _ in range(3))
        x = z / torch.sqrt(c / 3) * 1e-3
    else:
        x = torch.randn(shape, generator=g) * torch.exp2(
            torch.randint(-12, 12, shape[:-1] + (1,), generator=g).float())
    return x.to(torch.bfloat16).to(dev)


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("rounding", ["rne", "sr"])
@pytest.mark.parametrize("fmt", ["nvfp4_46", "nvfp4_6"])
def test_dual_1x16(shape, rounding, fmt):
    dev = require_gpu()
    x = _rand(shape, shape[1] * 7 + shape[2], dev)
    check_quantize(x, fmt=fmt, rounding=rounding, seed=99, rowwise=True, colwise=True)


@pytest.mark.parametrize("shape", [(1, 64, 128), (2, 528, 400)])
def test_colwise_only_and_swizzled(shape):
    dev = require_gpu()
    x = _rand(shape, 5, dev, "scaled")
    check_quantize(x, rowwise=False, colwise=True)
    check_quantize(x, rowwise=True, colwise=True, swizzle=True, rounding="sr", seed=3)


def test_dual_sr_element_offset():
    dev = require_gpu()
    x = _rand((1, 96, 160), 8, dev)
    check_quantize(x, rounding="sr", seed=17, elem_offset=16 * 12345, colwise=True)


@pytest.mark.parametrize("shape", [(1, 16, 16), (2, 80, 272), (1, 528, 400), (3, 1040, 128)])
@pytest.mark.parametrize("rounding", ["rne", "sr"])
@pytest.mark.parametrize("fmt", ["nvfp4_46", "nvfp4_6"])
def test_dual_with_colwise_transform(shape, rounding, fmt):
    """FOS_FLAG_RHT16_COL: the colwise blocks transformed along rows, with
    their own S_t (R21); the rowwise copy of the same call untransformed.
    Outlier rows make the transform change the codes."""
    dev = require_gpu()
    x = _rand(shape, shape[1] * 3 + shape[2] + 1, dev, "scaled")
    x[..., ::9, :] *= 16
    check_quantize(x, fmt=fmt, rounding=rounding, seed=21, rowwise=True, colwise=True, rht_col=True)


def test_colwise_transform_options():
    dev = require_gpu()
    x = _rand((2, 96, 160), 12, dev, "scaled")
    # colwise only, swizzled scales, SR with an element offset
    check_quantize(x, rowwise=False, colwise=True, rht_col=True, swizzle=True, rounding="sr", seed=4,
                   elem_offset=16 * 777)
    # the rowwise amax supplied: the colwise amax is still computed in the call
    am = F.amax(x)
    check_quantize(x, rowwise=True, colwise=True, rht_col=True, amax=am)
    # refused combinations
    for kw in (dict(rht_col=True), dict(rht_col=True, block="16x16", colwise=True),
               dict(rht_col=True, rht=True, colwise=True)):
        with pytest.raises(F.FosError):
            F.quantize(x, **kw)


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("rounding", ["rne", "sr"])
@pytest.mark.parametrize("fmt", ["nvfp4_46", "nvfp4_6"])
def test_2d_16x16(shape, rounding, fmt):
    dev = require_gpu()
    x = _rand(shape, shape[1] + 3 * shape[2], dev, "scaled")
    check_quantize(x, fmt=fmt, block="16x16", rounding=rounding, seed=5, rowwise=True, colwise=True)


@pytest.mark.parametrize("nsub", range(1, 9))
def test_2d_every_strip_length(nsub):
    """The 2D kernel's results do not depend on how many 64-row sub-tiles a
    CTA strip holds (the library picks it per launch).  1040 rows end strips
    of every length early; 2048 rows make the transposed bitmap's 32-bit
    words whole, which strips of 8 store directly."""
    dev = require_gpu()
    for shape, seed in (((2, 1040, 400), 3), ((1, 2048, 384), 4)):
        x = _rand(shape, seed, dev, "scaled")
        check_quantize(x, block="16x16", rowwise=True, colwise=True, strip_2d=nsub)
        check_quantize(x, block="16x16", rowwise=True, colwise=True, swizzle=True, rounding="sr", seed=9,
                       strip_2d=nsub)
    x = _rand((1, 528, 272), 5, dev, "scaled")
    check_quantize(x, fmt="nvfp4_6", block="16x16", rowwise=False, colwise=True, strip_2d=nsub)


@pytest.mark.parametrize("row,col", [(True, False), (False, True)])
def test_2d_one_orientation_and_swizzle(row, col):
    dev = require_gpu()
    x = _rand((2, 272, 400), 12, dev)
    check_quantize(x, block="16x16", rowwise=row, colwise=col)
    check_quantize(x, block="16x16", rowwise=row, colwise=col, swizzle=True)


def test_2d_transposed_dequant_is_transpose():
    dev = require_gpu()
    x = _rand((1, 256, 384), 21, dev)
    r, c = F.quantize(x, block="16x16", colwise=True)
    yr = F.dequantize(r)
    yc = F.dequantize(c)
    torch.cuda.synchronize()
    assert torch.equal(yr[0].t().contiguous().view(torch.int16), yc[0].contiguous().view(torch.int16))
