"""The quantized Linear layer (mxfp4_block_scaled_fos_b200/linear.py): the
forward GEMM and the dgrad and wgrad GEMMs, each on operands the library
quantizes (x 1x16, W 16x16 2D with its transposed copy, dy 1x16 with
stochastic rounding in both orientations, x^T 1x16 along M).

The reference quantizes the same bf16 inputs with the oracle, with the same
options, seed and orientation, decodes every operand to fp64 values q * s,
and multiplies in fp64.  Only the kernel's fp32 summation and the final
rounding separate the two, so the check uses the bound of
tests/test_gpu_gemm.py: |D - D_ref| <= alpha * K * 2^-24 * sum |a b| plus
2^-23 |D_ref| (f32 out).  One wrong code, scale, orientation or random byte
moves D by far more.
Sources: Hugging Face transformers doc "Four Over Six", usage section;
Ultralytics glossary "FP4", "Inferencia e Treinamento FP4"."""
import numpy as np
import pytest
import torch

import oracle
import mxfp4_block_scaled_fos_b200 as F

from helpers import np_bits, require_gpu

pytestmark = pytest.mark.gpu

E2M1 = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6, -0.0, -0.5, -1, -1.5, -2, -3, -4, -6], np.float64)
E4M3 = np.array([oracle.e4m3_decode(c) for c in range(256)], np.float64)


def _values(codes, scales):
    """q * s of one orientation [R, C] (no tensor scale), fp64."""
    lo, hi = codes & 0xF, codes >> 4
    nib = np.stack([lo, hi], axis=-1).reshape(codes.shape[0], -1)
    return E2M1[nib] * np.repeat(E4M3[scales], 16, axis=1)


def _ref(va, sta, vb, stb):
    alpha = float(np.float32(sta) * np.float32(stb))
    ref = alpha * (va @ vb.T)
    bound = alpha * (np.abs(va) @ np.abs(vb).T) * va.shape[1] * 2.0 ** -24 + np.abs(ref) * 2.0 ** -23 + 1e-30
    return ref, bound


def _check(got, ref, bound, what):
    err = np.abs(got.double().cpu().numpy() - ref)
    bad = np.argwhere(err > bound)
    assert bad.size == 0, "%s differs at %s: got %r ref %r" % (
        what, bad[:3].tolist(), float(got[tuple(bad[0])]), ref[tuple(bad[0])])


def _inputs(M, N, K, dev, seed):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(M, K, generator=g) * torch.exp2(torch.randint(-2, 3, (1, K), generator=g).float())
    x[:, ::53] *= 30                                   # outlier channels
    w = torch.randn(N, K, generator=g) * 0.02
    dy = torch.distributions.StudentT(3.0).sample((M, N)) * 1e-3
    return (x.to(torch.bfloat16).to(dev), w.to(torch.bfloat16).to(dev), dy.to(torch.bfloat16).to(dev))


@pytest.mark.parametrize("M,N,K,rht", [(256, 256, 256, False), (512, 256, 768, False), (256, 768, 512, False),
                                       (512, 256, 256, True), (256, 512, 768, True)])
def test_linear_forward_and_backward_match_oracle_operands(M, N, K, rht):
    dev = require_gpu()
    torch.manual_seed(M + N + K)
    x, w, dy = _inputs(M, N, K, dev, M * 7 + N * 3 + K)
    seed = 1234 + M
    qw = F.quantize_weight(w)
    y = F.linear_forward(x, qw, out_dtype=torch.float32)
    dx, dw = F.linear_backward(dy, x, qw, seed=seed, rht=rht)
    torch.cuda.synchronize()

    xb, wb, gb = np_bits(x)[None], np_bits(w)[None], np_bits(dy)[None]
    ox = oracle.quantize(xb)
    ow = oracle.quantize(wb, blk=oracle.BLK_16X16, colwise=True)
    og = oracle.quantize(gb, rnd=oracle.RND_SR, seed=seed, colwise=True, rht_col=rht)
    oxt = oracle.quantize(xb, rowwise=False, colwise=True, rht_col=rht, seed=seed)
    st_x, st_w, st_g = (float(o["tensor_scale"][0]) for o in (ox, ow, og))
    # the wgrad operands' own S_t (transformed columns with rht)
    st_gt, st_xt = float(og["c_tensor_scale"][0]), float(oxt["c_tensor_scale"][0])
    assert qw.row.tensor_scale.item() == st_w and qw.col.tensor_scale.item() == st_w

    x_v = _values(ox["r_codes"][0], ox["r_scales"][0])            # [M, K]
    w_v = _values(ow["r_codes"][0], ow["r_scales"][0])            # [N, K]
    wt_v = _values(ow["c_codes"][0], ow["c_scales"][0])           # [K, N]
    g_v = _values(og["r_codes"][0], og["r_scales"][0])            # [M, N]
    gt_v = _values(og["c_codes"][0], og["c_scales"][0])           # [N, M]
    xt_v = _values(oxt["c_codes"][0], oxt["c_scales"][0])         # [K, M]
    # 2D blocks: the transposed copy holds the same values as the weight
    assert np.array_equal(wt_v, w_v.T)

    _check(y, *_ref(x_v, st_x, w_v, st_w), "forward y")
    _check(dx, *_ref(g_v, st_g, wt_v, st_w), "dgrad dx")
    _check(dw, *_ref(gt_v, st_gt, xt_v, st_xt), "wgrad dW")


@pytest.mark.parametrize("rht", [False, True])
def test_saved_colwise_copy_gives_the_same_layer(rht):
    """linear_forward(save_colwise=True) makes x^T's copy from the forward's
    read of x (the two-orientation kernel); the forward output and the
    backward's dx and dW equal those of the path that quantizes x again in
    the backward, bit for bit."""
    dev = require_gpu()
    M, N, K, seed = 512, 256, 768, 77
    x, w, dy = _inputs(M, N, K, dev, 9)
    qw = F.quantize_weight(w)
    y0 = F.linear_forward(x, qw, out_dtype=torch.float32)
    dx0, dw0 = F.linear_backward(dy, x, qw, seed=seed, rht=rht)
    y1, qx_t = F.linear_forward(x, qw, out_dtype=torch.float32, save_colwise=True, rht=rht, seed=seed)
    dx1, dw1 = F.linear_backward(dy, None, qw, seed=seed, rht=rht, qx_t=qx_t)
    torch.cuda.synchronize()
    for a, b in ((y0, y1), (dx0, dx1), (dw0, dw1)):
        assert torch.equal(a.view(torch.int32), b.view(torch.int32))
    with pytest.raises(ValueError):
        F.linear_backward(dy[:256].contiguous(), None, qw, seed=seed, qx_t=qx_t)   # M differs


def test_linear_shape_errors():
    dev = require_gpu()
    x, w, dy = _inputs(256, 256, 256, dev, 5)
    with pytest.raises(ValueError):
        F.quantize_weight(w[:, :128].contiguous())
    qw = F.quantize_weight(w)
    with pytest.raises(ValueError):
        F.linear_forward(x[:128].contiguous(), qw)
    with pytest.raises(ValueError):
        F.linear_backward(dy[:, :128].contiguous(), x, qw)
