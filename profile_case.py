"""Small, self-contained launches of one kernel for profiler captures.

    python profile_case.py --case moe46 --experts 8 --iters 3

Each case builds its synthetic input (the same recipes as the benchmark, at
a reduced batch so a capture stays small), runs one untimed call, then
`iters` calls of the kernel of interest on the current stream.  Cases:

  moe46     4/6 NVFP4 1x16 rowwise on expert weights, amax supplied (k_q1x16)
  moe46_full  the same with the per-expert amax computed in the call (k_q1x16_fused)
  moe6      6-only NVFP4 1x16 rowwise, amax supplied
  moe_amax  the per-expert amax pass (k_amax)
  moe_mx    MXFP4 1x32 (k_mxfp4)
  moe_deq   NVFP4 dequantize (k_dequant)
  act_rht   4/6 with the 16-wide RHT on activation rows (8192 x cols), amax supplied
  grad_dual 4/6 SR rowwise + colwise on Student-t gradients (rows x 8192)
  weight_2d 4/6 16x16 2D with the transposed copy on 0.02-normal weights (rows x 4096)
  moe_fake  4/6 fake quantization (quantize + dequantize, bf16 out), amax in the call
  gemm      NVFP4 block-scaled GEMM, rows x rows x rows (rows a multiple of 256)
  linear    one step of the quantized Linear layer, 8192 x 4096 -> 4096: forward,
            dgrad and wgrad with x and dy quantized in the step (several kernels)
"""
from __future__ import annotations

import argparse

import torch

import os
import sys

sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))

import mxfp4_block_scaled_fos_b200 as F  # noqa: E402
from mxfp4_block_scaled_fos_b200 import workloads  # noqa: E402


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--case", default="moe46")
    ap.add_argument("--experts", type=int, default=8)
    ap.add_argument("--rows", type=int, default=4096)
    ap.add_argument("--iters", type=int, default=3)
    args = ap.parse_args()
    dev = torch.device("cuda:0")
    c = args.case
    if c.startswith("moe"):
        x = workloads.moe_experts(args.experts, 2880, 2880, device=dev)
        amax = F.amax(x)
        if c == "moe46_full":
            ws = torch.empty(F.workspace_size(args.experts, 2880, 2880), dtype=torch.uint8, device=dev)
            out = F.quantize(x, workspace=ws)[0]
            fn = lambda: F.quantize(x, out_row=out, workspace=ws)
        elif c == "moe46":
            out = F.quantize(x, amax=amax)[0]
            fn = lambda: F.quantize(x, amax=amax, out_row=out)
        elif c == "moe6":
            out = F.quantize(x, fmt="nvfp4_6", amax=amax)[0]
            fn = lambda: F.quantize(x, fmt="nvfp4_6", amax=amax, out_row=out)
        elif c == "moe_amax":
            fn = lambda: F.amax(x, out=amax)
        elif c == "moe_mx":
            out = F.quantize(x, fmt="mxfp4")[0]
            fn = lambda: F.quantize(x, fmt="mxfp4", out_row=out)
        elif c == "moe_deq":
            q = F.quantize(x, amax=amax)[0]
            y = torch.empty_like(x)
            fn = lambda: F.dequantize(q, out=y)
        elif c == "moe_fake":
            ws = torch.empty(F.workspace_size(args.experts, 2880, 2880), dtype=torch.uint8, device=dev)
            y = torch.empty_like(x)
            fn = lambda: F.fake_quantize(x, out=y, workspace=ws)
        else:
            raise SystemExit("unknown case " + c)
    elif c == "act_rht":
        x = workloads.activation_outliers(args.rows, 4096, device=dev)
        amax = F.amax(x, rht=True)
        out = F.quantize(x, rht=True, amax=amax)[0]
        fn = lambda: F.quantize(x, rht=True, amax=amax, out_row=out)
    elif c == "grad_dual":
        x = workloads.gradient_student_t(args.rows, 8192, device=dev)
        amax = F.amax(x)
        r, cc = F.quantize(x, rounding="sr", colwise=True, amax=amax)
        fn = lambda: F.quantize(x, rounding="sr", colwise=True, amax=amax, out_row=r, out_col=cc)
    elif c == "weight_2d":
        x = workloads.weight_normal(args.rows, 4096, device=dev)
        amax = F.amax(x)
        r, cc = F.quantize(x, block="16x16", colwise=True, amax=amax)
        fn = lambda: F.quantize(x, block="16x16", colwise=True, amax=amax, out_row=r, out_col=cc)
    elif c == "gemm":
        n = args.rows
        g = torch.Generator(device=dev).manual_seed(0)
        xa = torch.randn(n, n, generator=g, device=dev).to(torch.bfloat16)
        xb = torch.randn(n, n, generator=g, device=dev).to(torch.bfloat16)
        qa = F.quantize(xa, swizzle=True, choice=False)[0]
        qb = F.quantize(xb, swizzle=True, choice=False)[0]
        d = torch.empty(n, n, dtype=torch.bfloat16, device=dev)
        ws = torch.empty(F.gemm_workspace_size(n, n, n), dtype=torch.uint8, device=dev)
        fn = lambda: F.gemm_nvfp4(qa, qb, out=d, workspace=ws)
    elif c == "linear":
        # the bench's Linear step: 8192 tokens x 4096 -> 4096, forward, dgrad
        # and wgrad with x and dy quantized inside the step
        xl = workloads.activation_outliers(8192, 4096, device=dev)[0]
        wl = workloads.weight_normal(4096, 4096, device=dev)[0]
        dyl = workloads.gradient_student_t(8192, 4096, device=dev)[0]
        qw = F.quantize_weight(wl)

        def fn():
            _, qx_t = F.linear_forward(xl, qw, save_colwise=True, seed=7)
            F.linear_backward(dyl, None, qw, seed=7, qx_t=qx_t)
    else:
        raise SystemExit("unknown case " + c)
    fn()
    torch.cuda.synchronize()
    for _ in range(args.iters):
        fn()
    torch.cuda.synchronize()
    print("profile case %s done (%d iters)" % (c, args.iters))


if __name__ == "__main__":
    main()
