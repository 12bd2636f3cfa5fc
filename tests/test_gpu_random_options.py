"""Seeded random sweep over the quantizer's option space: for each seed a
shape (batch entries, ragged rows and columns) and a valid combination of
format, block mode, rounding, transform flags, swizzled scales, orientations,
a supplied or computed amax and an element offset, quantized on the GPU and
by the oracle and compared byte for byte (codes, scales, S_t, choice bits).
The per-feature tests cover each option; this one covers their mixtures."""
import random

import pytest
import torch

import mxfp4_block_scaled_fos_b200 as F

from helpers import check_quantize, require_gpu

pytestmark = pytest.mark.gpu


def _case(seed):
    rnd = random.Random(seed)
    fmt = rnd.choice(["nvfp4_46", "nvfp4_46", "nvfp4_6", "mxfp4"])
    if fmt == "mxfp4":
        block, rounding, rht, rht_col = "1x32", "rne", False, False
        colwise = False
    else:
        block = rnd.choice(["1x16", "1x16", "16x16"])
        rounding = rnd.choice(["rne", "sr"])
        colwise = rnd.random() < 0.5
        rht = block == "1x16" and not colwise and rnd.random() < 0.4
        rht_col = block == "1x16" and colwise and fmt != "mxfp4" and rnd.random() < 0.4
    rowwise = True if not colwise else rnd.random() < 0.7
    bs = 32 if fmt == "mxfp4" else 16
    rows = 16 * rnd.randint(1, 24)
    cols = bs * rnd.randint(1, 640 // bs)
    batch = rnd.randint(1, 3)
    swizzle = rnd.random() < 0.4
    supply_amax = rnd.random() < 0.3 and not rht_col
    offset = 16 * rnd.randint(0, 1000) if rounding == "sr" else 0
    scale = 2.0 ** rnd.randint(-12, 8)
    return dict(fmt=fmt, block=block, rounding=rounding, rht=rht, rht_col=rht_col, rowwise=rowwise,
                colwise=colwise, swizzle=swizzle, seed=rnd.randint(0, 2 ** 40), elem_offset=offset), \
        (batch, rows, cols), supply_amax, scale


@pytest.mark.parametrize("seed", range(200))
def test_random_option_mix(seed):
    dev = require_gpu()
    kw, shape, supply_amax, scale = _case(seed)
    g = torch.Generator().manual_seed(1000 + seed)
    z = torch.randn(shape, generator=g)
    heavy = z / torch.sqrt(sum(torch.randn(shape, generator=g) ** 2 for _ in range(3)) / 3 + 1e-3)
    x = (heavy * scale).to(torch.bfloat16).to(dev)
    amax = F.amax(x, rht=kw["rht"], seed=kw["seed"]) if supply_amax else None
    check_quantize(x, amax=amax, **kw)
