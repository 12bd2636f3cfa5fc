"""A quantized Linear layer y = x @ W^T in NVFP4 with Four Over Six scaling:
the forward GEMM and the two backward GEMMs, each operand quantized by
fos_quantize into the swizzled tensor-core layout and multiplied by
fos_gemm_nvfp4 on the tcgen05 tensor cores.  This module only allocates
buffers and orders the library calls; every step runs in the library's
kernels.

Sources: Hugging Face transformers doc "Four Over Six", usage section (the
options 2D block scaling, transposed inputs and stochastic rounding, offered
for training); Ultralytics glossary "FP4", "Inferencia e Treinamento FP4"
(FP4 training on Blackwell: stochastic rounding for the gradients, the
block-scaled FP4 GEMM on the tensor cores).

Operands (x [M, K] activations, W [N, K] weights, dy [M, N] output
gradients; every tensor quantized with its own per-tensor scale):

  forward  y  = x @ W^T   A = x, 1x16 blocks along K;
                          B = W, 16x16 2D blocks (its rowwise copy)
  dgrad    dx = dy @ W    A = dy, 1x16 blocks along N, stochastic rounding;
                          B = the transposed copy of the same 2D W
  wgrad    dW = dy^T @ x  A = dy^T, 1x16 blocks along M, the same random
                          bytes as dgrad's copy (one draw per source element);
                          B = x^T, 1x16 blocks along M

The 2D weight blocks make W and W^T quantize to the same values, so the
forward and dgrad GEMMs see one weight.  With rht=True the two wgrad
operands are quantized with the 16-wide random Hadamard transform along M
(FOS_FLAG_RHT16_COL, the same seeded signs for both): the transform is
orthogonal and applied to both sides of the reduction, so dW is unchanged
in exact arithmetic while the outliers of dy and x are spread before
quantization.  Shapes: M and N multiples of 256, K a multiple of 256 (the
GEMM's 128-row tiles and 256-wide K steps, in each of the three products).
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Optional, Tuple

import torch

from . import fos


@dataclass
class QuantizedWeight:
    """The 16x16-scaled weight W [N, K] and its transposed copy [K, N]."""
    row: fos.QTensor
    col: fos.QTensor

    @property
    def shape(self) -> Tuple[int, int]:
        return self.row.rows, self.row.cols


def _check(name: str, n: int, mult: int) -> None:
    if n <= 0 or n % mult:
        raise ValueError("%s = %d must be a positive multiple of %d" % (name, n, mult))


def quantize_weight(w: torch.Tensor, fmt: str = "nvfp4_46", stream=None) -> QuantizedWeight:
    """W [N, K] bf16 -> 16x16 2D NVFP4 with its exact transposed copy, both
    with swizzled scales."""
    if w.dim() != 2:
        raise ValueError("w must be [N, K]")
    _check("N", w.shape[0], 256)
    _check("K", w.shape[1], 256)
    r, c = fos.quantize(w, fmt=fmt, block="16x16", swizzle=True, colwise=True, choice=False, stream=stream)
    return QuantizedWeight(r, c)


def linear_forward(x: torch.Tensor, qw: QuantizedWeight, fmt: str = "nvfp4_46",
                   out: Optional[torch.Tensor] = None, out_dtype=torch.bfloat16, save_colwise: bool = False,
                   rht: bool = False, seed: int = 0, stream=None):
    """y [M, N] = x [M, K] @ W^T with x quantized 1x16 along K (RNE).

    save_colwise: also quantize x^T along M (the wgrad operand) from the same
    read of x, and return (y, qx_t) for linear_backward(..., qx_t=qx_t); with
    rht the colwise copy is transformed along M with the signs of `seed` (pass
    the backward's seed).  The rowwise copy is the same either way."""
    if x.dim() != 2 or x.shape[1] != qw.shape[1]:
        raise ValueError("x must be [M, K] with the weight's K")
    _check("M", x.shape[0], 256)
    if save_colwise:
        qx, qx_t = fos.quantize(x, fmt=fmt, swizzle=True, colwise=True, choice=False, rht_col=rht, seed=seed,
                                stream=stream)
        return fos.gemm_nvfp4(qx, qw.row, out=out, out_dtype=out_dtype, stream=stream), qx_t
    qx = fos.quantize(x, fmt=fmt, swizzle=True, choice=False, stream=stream)[0]
    return fos.gemm_nvfp4(qx, qw.row, out=out, out_dtype=out_dtype, stream=stream)


def linear_backward(dy: torch.Tensor, x: Optional[torch.Tensor], qw: QuantizedWeight, seed: int = 0,
                    elem_offset: int = 0, fmt: str = "nvfp4_46", out_dtype=torch.float32,
                    rht: bool = False, qx_t: Optional[fos.QTensor] = None,
                    stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """(dx [M, K], dW [N, K]) from dy [M, N], the forward input x [M, K] and
    the quantized weight.  dy is quantized once, in both orientations, with
    stochastic rounding keyed on (seed, elem_offset + element index).  rht:
    the wgrad operands (dy^T, x^T) are transformed along M with the signs of
    the same key (seed), each with its own S_t.  qx_t: x^T as saved by
    linear_forward(save_colwise=True) with the same rht and seed; x is then
    not read (and may be None)."""
    N, K = qw.shape
    M = dy.shape[0] if dy.dim() == 2 else -1
    if dy.dim() != 2 or dy.shape[1] != N:
        raise ValueError("dy must be [M, N] for a weight [N, K]")
    if qx_t is None:
        if x is None or x.dim() != 2 or x.shape[1] != K or x.shape[0] != M:
            raise ValueError("x must be [M, K] for dy [M, N] and a weight [N, K]")
    elif qx_t.rows != K or qx_t.cols != M or qx_t.batch != 1:
        raise ValueError("qx_t must be the colwise copy of an [M, K] input")
    _check("M", M, 256)
    qdy, qdy_t = fos.quantize(dy, fmt=fmt, rounding="sr", seed=seed, elem_offset=elem_offset, swizzle=True,
                              colwise=True, choice=False, rht_col=rht, stream=stream)
    if qx_t is None:
        qx_t = fos.quantize(x, fmt=fmt, swizzle=True, rowwise=False, colwise=True, choice=False, rht_col=rht,
                            seed=seed, stream=stream)[1]
    dx = fos.gemm_nvfp4(qdy, qw.col, out_dtype=out_dtype, stream=stream)
    dw = fos.gemm_nvfp4(qdy_t, qx_t, out_dtype=out_dtype, stream=stream)
    return dx, dw
