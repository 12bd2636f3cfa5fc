"""The NVFP4 block-scaled GEMM on the tensor cores (fos_gemm_nvfp4), fed by
the quantizer's swizzled output: D = (S_tA * S_tB) * A @ B^T.

The reference is computed in fp64 from the oracle's own quantization of the
same bf16 inputs: every element is q * s with q the E2M1 value and s the
E4M3 block scale (both exact in fp64), so the reference product is exact up
to fp64 rounding.  Each product q_a s_a q_b s_b is exact in fp32 as well;
only the fp32 summation over K rounds, so the kernel is checked within the
worst-case bound of a K-term fp32 sum in any order, |D - D_ref| <=
K * 2^-24 * sum_k |A_mk * B_nk| * S_tA * S_tB, plus the final rounding of D
(2^-24 relative for f32, 2^-8 for bf16).  A wrong operand, scale or tile
layout gives errors of the order of D itself and fails it.
Sources: Ultralytics glossary "FP4", "Como funciona FP4" (NVFP4 blocks of 16
with an E4M3 scale and an FP32 tensor scale) and "Inferencia e Treinamento
FP4" (FP4 GEMMs on Blackwell tensor cores)."""
import numpy as np
import pytest
import torch

import oracle
import mxfp4_block_scaled_fos_b200 as F

from helpers import np_bits, require_gpu

pytestmark = pytest.mark.gpu

E2M1 = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6, -0.0, -0.5, -1, -1.5, -2, -3, -4, -6], np.float64)


def _oracle_values(xb, fmt):
    """q * s (no tensor scale) of the oracle's rowwise quantization, fp64."""
    q = oracle.quantize(xb, fmt=fmt)
    codes = q["r_codes"][0]
    lo, hi = codes & 0xF, codes >> 4
    nib = np.stack([lo, hi], axis=-1).reshape(codes.shape[0], -1)
    s = np.array([oracle.e4m3_decode(c) for c in range(256)], np.float64)[q["r_scales"][0]]
    return E2M1[nib] * np.repeat(s, 16, axis=1), float(q["tensor_scale"][0])


def _operand(rows, K, seed, dev, fmt):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(rows, K, generator=g) * torch.exp2(torch.randint(-3, 3, (rows, 1), generator=g).float())
    x.view(-1)[::97] *= 20
    x = x.to(torch.bfloat16).to(dev)
    q = F.quantize(x, fmt=fmt, swizzle=True, choice=False)[0]
    return x, q


@pytest.mark.parametrize("M,N,K", [(128, 128, 256), (256, 384, 512), (384, 256, 1024), (128, 512, 2304)])
@pytest.mark.parametrize("fmt", ["nvfp4_46", "nvfp4_6"])
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("wide", [True, False])
def test_gemm_matches_fp64_reference(M, N, K, fmt, out_dtype, wide):
    dev = require_gpu()
    xa, qa = _operand(M, K, M + 3 * K, dev, fmt)
    xb, qb = _operand(N, K, N + 7 * K + 1, dev, fmt)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    d = F.gemm_nvfp4(qa, qb, out_dtype=out_dtype, status=status, wide=wide)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    fo = oracle.FMT_NVFP4_46 if fmt == "nvfp4_46" else oracle.FMT_NVFP4_6
    va, sta = _oracle_values(np_bits(xa)[None], fo)
    vb, stb = _oracle_values(np_bits(xb)[None], fo)
    # the kernel's tensor scales are the oracle's (bit parity of the quantizer)
    assert qa.tensor_scale.item() == sta and qb.tensor_scale.item() == stb
    alpha = float(np.float32(sta) * np.float32(stb))
    ref = alpha * (va @ vb.T)
    bound = alpha * (np.abs(va) @ np.abs(vb).T) * K * 2.0 ** -24 + 1e-30
    got = d.double().cpu().numpy()
    bound = bound + np.abs(ref) * (2.0 ** -8 if out_dtype == torch.bfloat16 else 2.0 ** -23)
    err = np.abs(got - ref)
    bad = np.argwhere(err > bound)
    assert bad.size == 0, "GEMM differs at %s: got %r ref %r bound %r" % (
        bad[:3].tolist(), got[tuple(bad[0])], ref[tuple(bad[0])], bound[tuple(bad[0])])


@pytest.mark.parametrize("M,N,K", [(1024, 1024, 2048), (512, 896, 1280)])
def test_wide_scale_layout_gives_the_same_bits(M, N, K):
    """The workspace path (scales rewritten for the 128 x 256-bit tensor-memory
    copy) feeds the same scales to the same MMAs in the same order as the
    plain path: the outputs are equal bit for bit, on 128 x 256 tiles
    (N % 256 == 0) and on 128 x 128 tiles."""
    dev = require_gpu()
    _, qa = _operand(M, K, 5, dev, "nvfp4_46")
    _, qb = _operand(N, K, 6, dev, "nvfp4_46")
    d_wide = F.gemm_nvfp4(qa, qb, out_dtype=torch.float32, wide=True)
    d_plain = F.gemm_nvfp4(qa, qb, out_dtype=torch.float32, wide=False)
    torch.cuda.synchronize()
    assert torch.equal(d_wide.view(torch.int32), d_plain.view(torch.int32))
    ws = torch.empty(F.gemm_workspace_size(M, N, K) - 16, dtype=torch.uint8, device=dev)
    with pytest.raises(F.FosError):
        F.gemm_nvfp4(qa, qb, workspace=ws)   # one 16-byte chunk short


def test_gemm_rejects_bad_shapes():
    dev = require_gpu()
    _, qa = _operand(128, 256, 1, dev, "nvfp4_46")
    _, qb = _operand(100 + 28, 256, 2, dev, "nvfp4_46")
    F.gemm_nvfp4(qa, qb)
    _, qc = _operand(136, 256, 3, dev, "nvfp4_46")
    with pytest.raises(F.FosError):
        F.gemm_nvfp4(qa, qc)  # N = 136 is not a multiple of 128
