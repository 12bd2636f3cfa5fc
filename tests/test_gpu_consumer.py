"""The swizzled scale layout, checked by a real consumer: cuBLAS's block-scaled
FP4 GEMM (torch._scaled_mm with float4_e2m1fn_x2 operands) reads our codes
and swizzled scales, and its product must equal an fp64 GEMM of the same
operands decoded from the linear-layout codes and scales.  A wrong tile,
row-group or byte order in the swizzled layout would pair elements with the
wrong block scales and miss by far more than the tolerance.  The sizes are
ragged (rows not a multiple of 128, block columns not a multiple of 4) so
the padding of the layout is exercised too."""
import numpy as np
import pytest
import torch

import mxfp4_block_scaled_fos_b200 as F

from helpers import require_gpu

pytestmark = pytest.mark.gpu

E2M1 = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def _decode_codes(codes: np.ndarray, cols: int) -> np.ndarray:
    """uint8 [R, cols/2] packed E2M1 -> float64 [R, cols] (even element in the low nibble)."""
    lo = codes & 0xF
    hi = codes >> 4
    nib = np.stack([lo, hi], axis=-1).reshape(codes.shape[0], cols)
    v = E2M1[nib & 7]
    return np.where(nib & 8, -v, v)


def _e4m3(b: np.ndarray) -> np.ndarray:
    return torch.from_numpy(b.copy()).view(torch.float8_e4m3fn).float().double().numpy()


def _e8m0(b: np.ndarray) -> np.ndarray:
    return np.ldexp(1.0, b.astype(np.int64) - 127)


def _operand(x, fmt):
    """(swizzled quantization for cuBLAS, fp64 decode of the linear one)."""
    block = "1x32" if fmt == "mxfp4" else "1x16"
    bs = 32 if fmt == "mxfp4" else 16
    qs, _ = F.quantize(x, fmt=fmt, block=block, swizzle=True)
    ql, _ = F.quantize(x, fmt=fmt, block=block, swizzle=False)
    torch.cuda.synchronize()
    rows, cols = x.shape
    q = _decode_codes(ql.codes.view(rows, cols // 2).cpu().numpy(), cols)
    sc = ql.scales.view(rows, cols // bs).cpu().numpy()
    s = _e8m0(sc) if fmt == "mxfp4" else _e4m3(sc)
    deq = q * np.repeat(s, bs, axis=1)
    st = 1.0 if fmt == "mxfp4" else float(ql.tensor_scale.cpu().double()[0])
    return qs, deq, st


@pytest.mark.parametrize("fmt", ["nvfp4_46", "nvfp4_6", "mxfp4"])
def test_swizzled_scales_drive_cublas_block_scaled_gemm(fmt):
    dev = require_gpu()
    M, N, K = 200, 144, 544   # 2 row tiles (ragged), K/16 = 34 and K/32 = 17 blocks (padded)
    g = torch.Generator().manual_seed(13)
    a = (torch.randn(M, K, generator=g) * torch.exp2(torch.randint(-3, 4, (M, 1), generator=g).float()))
    b = (torch.randn(N, K, generator=g) * torch.exp2(torch.randint(-3, 4, (1, K), generator=g).float()))
    a = a.to(torch.bfloat16).to(dev)
    b = b.to(torch.bfloat16).to(dev)
    qa, da, sta = _operand(a, fmt)
    qb, db, stb = _operand(b, fmt)
    sdt = torch.float8_e8m0fnu if fmt == "mxfp4" else torch.float8_e4m3fn
    A = qa.codes.view(M, K // 2).view(torch.float4_e2m1fn_x2)
    B = qb.codes.view(N, K // 2).view(torch.float4_e2m1fn_x2)
    try:
        out = torch._scaled_mm(A, B.t(), qa.scales.view(-1).view(sdt), qb.scales.view(-1).view(sdt),
                               out_dtype=torch.float32)
    except (RuntimeError, NotImplementedError) as e:   # this torch has no block-scaled FP4 GEMM
        pytest.skip("cuBLAS block-scaled FP4 GEMM unavailable: %s" % str(e).splitlines()[0])
    torch.cuda.synchronize()
    got = out.double().cpu().numpy() * (sta * stb)
    want = (da @ db.T) * (sta * stb)
    # fp32 accumulation over K = 544 products: bounded by a small multiple of
    # K * 2^-24 times the sum of |products|; a misplaced scale is off by a
    # factor of the scale ratio on whole blocks
    bound = 1e-4 * (np.abs(da) @ np.abs(db).T) * (sta * stb) + 1e-30
    assert np.all(np.abs(got - want) <= bound), (fmt, float(np.abs(got - want).max()), float(bound.max()))
    assert np.abs(want).max() > 0
