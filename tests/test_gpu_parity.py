"""GPU parity: the sm_100a kernels (through the C ABI) against the CPU oracle,
bit for bit, on seeded inputs.  Small shapes span several CTAs, ragged tails
(odd block counts, single rows), batches, strided rows and the degenerate
cases (zero tensors, zero blocks, ties, tiny values)."""
import numpy as np
import pytest
import torch

import oracle
import mxfp4_block_scaled_fos_b200 as F
from mxfp4_block_scaled_fos_b200 import workloads

from helpers import check_quantize, np_bits, require_gpu, zeroed_out, assert_bytes_equal

pytestmark = pytest.mark.gpu


def _rand(shape, kind, seed, device):
    g = torch.Generator(device="cpu").manual_seed(seed)
    if kind == "normal":
        x = torch.randn(shape, generator=g)
    elif kind == "heavy":
        z = torch.randn(shape, generator=g)
        c = sum(torch.randn(shape, generator=g) ** 2 for _ in range(3))
        x = z / torch.sqrt(c / 3)
    elif kind == "outliers":
        x = torch.randn(shape, generator=g)
        x.view(-1)[::97] *= 40
    elif kind == "tiny":
        x = torch.randn(shape, generator=g) * 1e-38
    elif kind == "mixed_scale":
        x = torch.randn(shape, generator=g) * torch.exp2(torch.randint(-30, 30, shape[:-1] + (1,), generator=g).float())
    elif kind == "zeros":
        x = torch.zeros(shape)
        x.view(-1)[::7] = -0.0
    else:
        raise KeyError(kind)
    return x.to(torch.bfloat16).to(device)


def _ties(device):
    """S_t = 1 (tensor max 1792); a block with max 24 has e6 = 4 and e4 = 6,
    so w = 4*m hits every E2M1 midpoint m for the 6-candidate and w = 6*m for
    the 4-candidate."""
    mids = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 0.5, 1.0, 3.0]
    rows = []
    r0 = [0.0] * 32
    r0[0] = 1792.0
    rows.append(r0)
    for mult in (4.0, 6.0):
        for sign in (1.0, -1.0):
            r = [0.0] * 32
            r[0] = 24.0
            r[16] = -24.0
            for i, m in enumerate(mids):
                r[1 + i] = sign * mult * m
                r[17 + i] = -sign * mult * m * 0.5
            rows.append(r)
    rows.append([-0.0] * 32)
    return torch.tensor(rows, dtype=torch.float32).to(torch.bfloat16).to(device)


def test_outlier_vector_full_size():
    """The page example's generator at 128x256: 4/6, 1x16, RNE, rowwise."""
    dev = require_gpu()
    x = workloads.outlier_vector(128, 256).to(dev)
    check_quantize(x)


SHAPES = [(1, 1, 16), (1, 3, 48), (2, 5, 32), (3, 17, 80), (1, 64, 1024), (2, 33, 2880)]


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("kind", ["normal", "heavy", "outliers", "mixed_scale"])
@pytest.mark.parametrize("fmt", ["nvfp4_46", "nvfp4_6"])
def test_rowwise_1x16_rne(shape, kind, fmt):
    dev = require_gpu()
    x = _rand(shape, kind, 1 + len(kind) * 31 + shape[2], dev)
    check_quantize(x, fmt=fmt)


@pytest.mark.parametrize("kind", ["tiny", "zeros"])
def test_rowwise_degenerate(kind):
    dev = require_gpu()
    x = _rand((2, 7, 64), kind, 5, dev)
    check_quantize(x)
    check_quantize(x, fmt="nvfp4_6")


def test_rowwise_ties_and_signed_zeros():
    dev = require_gpu()
    x = _ties(dev)
    check_quantize(x)
    check_quantize(x, rounding="sr", seed=4)
    check_quantize(x, fmt="nvfp4_6")


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("fmt", ["nvfp4_46", "nvfp4_6"])
def test_rowwise_sr(shape, fmt):
    dev = require_gpu()
    x = _rand(shape, "heavy", 77 + shape[1], dev)
    check_quantize(x, fmt=fmt, rounding="sr", seed=12345 + shape[2])
    check_quantize(x, fmt=fmt, rounding="sr", seed=(7 << 40) | 9, elem_offset=16 * 1000)


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("rounding", ["rne", "sr"])
def test_rowwise_rht(shape, rounding):
    dev = require_gpu()
    x = _rand(shape, "outliers", 3 + shape[0], dev)
    check_quantize(x, rht=True, seed=shape[2], rounding=rounding)


@pytest.mark.parametrize("shape", [(1, 128, 64), (2, 130, 48), (1, 257, 2880)])
@pytest.mark.parametrize("fmt", ["nvfp4_46", "nvfp4_6", "mxfp4"])
def test_swizzled_scales(shape, fmt):
    dev = require_gpu()
    if fmt == "mxfp4" and shape[2] % 32:
        pytest.skip("MXFP4 needs cols % 32 == 0")
    x = _rand(shape, "normal", 11, dev)
    check_quantize(x, fmt=fmt, swizzle=True)


def test_strided_rows():
    dev = require_gpu()
    big = _rand((1, 40, 160), "heavy", 21, dev)
    x = big[:, :, 32:128]  # ld = 160, cols = 96
    assert x.stride(1) == 160
    check_quantize(x, x_bits=np_bits(x))
    check_quantize(x, rounding="sr", seed=3, x_bits=np_bits(x))


def test_amax_supplied():
    dev = require_gpu()
    x = _rand((2, 16, 64), "normal", 8, dev)
    a = torch.tensor([7.5, 0.25], dtype=torch.float32, device=dev)  # not the true amax
    check_quantize(x, amax=a)


@pytest.mark.parametrize("shape", [(1, 1, 32), (2, 9, 96), (4, 64, 2880)])
@pytest.mark.parametrize("kind", ["normal", "mixed_scale", "tiny", "zeros"])
def test_mxfp4(shape, kind):
    dev = require_gpu()
    x = _rand(shape, kind, shape[1] + 100, dev)
    check_quantize(x, fmt="mxfp4")


@pytest.mark.parametrize("rht", [False, True])
def test_amax_entry_point(rht):
    dev = require_gpu()
    x = _rand((3, 33, 80), "outliers", 41, dev)
    a = F.amax(x, rht=rht, seed=6)
    torch.cuda.synchronize()
    ref = oracle.amax(np_bits(x), rht=rht, seed=6)
    assert np.array_equal(a.cpu().numpy().view(np.uint32), ref.view(np.uint32))


def test_nonfinite_sets_status():
    dev = require_gpu()
    x = _rand((1, 16, 64), "normal", 2, dev)
    x[0, 3, 5] = float("nan")
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    F.quantize(x, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & F.STATUS_NONFINITE
    st.zero_()
    x[0, 3, 5] = float("inf")
    F.amax(x, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & F.STATUS_NONFINITE


@pytest.mark.parametrize("fmt", ["nvfp4_46", "nvfp4_6", "mxfp4"])
@pytest.mark.parametrize("swizzle", [False, True])
def test_dequantize_oracle_codes(fmt, swizzle):
    """GPU dequantize of oracle-made codes equals the oracle's dequantize."""
    dev = require_gpu()
    batch, R, C = 3, 130, 192
    x = _rand((batch, R, C), "heavy", 9, dev)
    xb = np_bits(x)
    blk = oracle.BLK_1X32 if fmt == "mxfp4" else oracle.BLK_1X16
    fo = {"nvfp4_46": oracle.FMT_NVFP4_46, "nvfp4_6": oracle.FMT_NVFP4_6, "mxfp4": oracle.FMT_MXFP4}[fmt]
    q = oracle.quantize(xb, fmt=fo, blk=blk)
    ref = oracle.dequantize(q["r_codes"], q["r_scales"], q["tensor_scale"], fmt=fo)
    flags = F.FLAG_SCALE_SWIZZLED if swizzle else 0
    sc = oracle.swizzle_scales(q["r_scales"]).reshape(batch, -1) if swizzle else q["r_scales"]
    qt = F.QTensor(torch.from_numpy(q["r_codes"]).to(dev), torch.from_numpy(np.ascontiguousarray(sc)).to(dev),
                   torch.from_numpy(q["tensor_scale"]).to(dev) if fmt != "mxfp4" else None,
                   None, batch, R, C, fmt, "1x32" if fmt == "mxfp4" else "1x16", flags)
    y = F.dequantize(qt)
    torch.cuda.synchronize()
    assert_bytes_equal(np_bits(y), ref, "dequantized")


@pytest.mark.parametrize("fmt", ["nvfp4_46", "mxfp4"])
def test_dequantize_strided_output(fmt):
    """Output rows 8 elements longer than the tensor (16-byte but not
    32-byte aligned rows): the strided path, and nothing written past a row."""
    dev = require_gpu()
    batch, R, C = 2, 48, 320
    x = _rand((batch, R, C), "heavy", 13, dev)
    q = F.quantize(x, fmt=fmt)[0]
    want = F.dequantize(q)
    yf = torch.full((batch, R, C + 8), 3.0, dtype=torch.bfloat16, device=dev)
    F.dequantize(q, out=yf[:, :, :C])
    torch.cuda.synchronize()
    assert torch.equal(yf[:, :, :C].view(torch.int16), want.view(torch.int16))
    assert torch.all(yf[:, :, C:] == 3.0)


# A block whose two candidate errors are exactly equal in binary32 (found in a
# seeded Student-t tensor): the tie must keep 6.  Rows 0 and 1 carry the same
# block in both halves of a pair, row 2 sets the tensor amax.
TIE_BLOCK = [0.0002307891845703125, 0.00262451171875, 0.0006256103515625, -9.918212890625e-05,
             -0.0089111328125, 0.00011682510375976562, -0.00115966796875, -6.4849853515625e-05,
             -0.0004405975341796875, -0.00360107421875, 0.00201416015625, 0.00144195556640625,
             0.000324249267578125, 0.0010528564453125, 0.000339508056640625, 0.0008544921875]


def test_exact_tie_block_keeps_6():
    dev = require_gpu()
    rows = torch.zeros(16, 32)
    rows[0, :16] = torch.tensor(TIE_BLOCK)
    rows[0, 16:] = torch.tensor(TIE_BLOCK)
    rows[1, 16:] = torch.tensor(TIE_BLOCK)
    rows[2, 0] = 0.06787109375
    x = rows.to(torch.bfloat16).to(dev)
    r, _, ref = check_quantize(x)
    # the oracle sees an exact tie here and keeps the 6-candidate
    assert not (ref["r_choice"][0] & 0b1011)
    check_quantize(x.t().contiguous(), colwise=True)
    check_quantize(x, rounding="sr", seed=1)
