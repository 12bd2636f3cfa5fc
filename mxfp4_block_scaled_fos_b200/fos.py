"""ctypes binding of libfos.so (include/fos.h) with torch tensors as buffers.

This module only marshals arguments: it checks dtypes and devices, allocates
output tensors with torch when the caller does not pass them, and hands raw
device pointers and the current CUDA stream to the C ABI.  Every step of the
quantizer runs in the library's sm_100a kernels; there is no CPU fallback.
If libfos.so is missing the first call raises.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
# FOS_LIBRARY may point at another build of the same library (e.g. one
# compiled with different tuning constants); default: the in-tree build.
LIB_PATH = os.environ.get("FOS_LIBRARY") or os.path.join(_PKG, "libfos.so")

FMT = {"nvfp4_46": 0, "nvfp4_6": 1, "mxfp4": 2}
BLK = {"1x16": 0, "16x16": 1, "1x32": 2}
RND = {"rne": 0, "sr": 1}
FLAG_RHT16 = 0x1
FLAG_SCALE_SWIZZLED = 0x2
FLAG_RHT16_COL = 0x4
STATUS_NONFINITE = 0x1
STATUS_TIMEOUT = 0x2

ERRORS = {
    1: "FOS_ERR_NULL", 2: "FOS_ERR_ALIGN", 3: "FOS_ERR_SHAPE", 4: "FOS_ERR_UNSUPPORTED",
    5: "FOS_ERR_WORKSPACE", 6: "FOS_ERR_CUDA", 7: "FOS_ERR_ARG",
}

# every symbol include/fos.h declares
EXPORTS = ("fos_quantize", "fos_quantize_host", "fos_amax", "fos_dequantize", "fos_workspace_size",
           "fos_scales_size", "fos_status_string", "fos_version", "fos_quantize_static",
           "fos_testing_quantize_stalled", "fos_testing_quantize_2d_strip", "fos_fake_quantize",
           "fos_gemm_nvfp4", "fos_gemm_nvfp4_ws", "fos_gemm_workspace_size")


class Options(ctypes.Structure):
    _fields_ = [("fmt", ctypes.c_int32), ("blk", ctypes.c_int32), ("rnd", ctypes.c_int32),
                ("flags", ctypes.c_uint32), ("seed", ctypes.c_uint64),
                ("elem_offset", ctypes.c_int64)]


class QTensorC(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p),
                ("tensor_scale", ctypes.c_void_p), ("choice_bits", ctypes.c_void_p),
                ("codes_ld", ctypes.c_int64), ("scales_ld", ctypes.c_int64)]


class FosError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__("%s failed: %s (%d)" % (what, ERRORS.get(code, "?"), code))
        self.code = code


_lib = None


def lib(path: str = LIB_PATH):
    """Load libfos.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError("libfos.so is missing at %s; build it with "
                           "`python -m mxfp4_block_scaled_fos_b200.build`" % path)
    L = ctypes.CDLL(path)
    P, i64, i32, u32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_uint32
    L.fos_quantize.restype = i32
    L.fos_quantize.argtypes = [P, i64, i64, i64, i64, ctypes.POINTER(Options), P,
                               ctypes.POINTER(QTensorC), ctypes.POINTER(QTensorC), P,
                               ctypes.c_size_t, P, P]
    L.fos_quantize_host.restype = i32
    L.fos_quantize_host.argtypes = [P, i64, i64, i64, ctypes.POINTER(Options), P, ctypes.POINTER(QTensorC), P,
                                    ctypes.POINTER(QTensorC), P, ctypes.c_size_t, P, i64, P, P, P,
                                    ctypes.POINTER(ctypes.c_void_p)]
    L.fos_quantize_static.restype = i32
    L.fos_quantize_static.argtypes = [P, i64, i64, i64, i64, ctypes.POINTER(Options), P,
                                      ctypes.POINTER(QTensorC), ctypes.POINTER(QTensorC), P, P]
    L.fos_testing_quantize_stalled.restype = i32
    L.fos_testing_quantize_stalled.argtypes = [P, i64, i64, i64, i64, ctypes.POINTER(Options),
                                               ctypes.POINTER(QTensorC), P, ctypes.c_size_t, P,
                                               i32, u32, P]
    L.fos_testing_quantize_2d_strip.restype = i32
    L.fos_testing_quantize_2d_strip.argtypes = [P, i64, i64, i64, i64, ctypes.POINTER(Options), P,
                                                ctypes.POINTER(QTensorC), ctypes.POINTER(QTensorC), P,
                                                ctypes.c_size_t, P, i32, P]
    L.fos_fake_quantize.restype = i32
    L.fos_fake_quantize.argtypes = [P, i64, i64, i64, i64, ctypes.POINTER(Options), P, P, i64, P,
                                    ctypes.c_size_t, P, P]
    L.fos_gemm_nvfp4_ws.restype = i32
    L.fos_gemm_nvfp4_ws.argtypes = [ctypes.POINTER(QTensorC), ctypes.POINTER(QTensorC), i64, i64, i64, P, i64,
                                    i32, P, ctypes.c_size_t, P, P]
    L.fos_gemm_workspace_size.restype = ctypes.c_size_t
    L.fos_gemm_workspace_size.argtypes = [i64, i64, i64]
    L.fos_gemm_nvfp4.restype = i32
    L.fos_gemm_nvfp4.argtypes = [ctypes.POINTER(QTensorC), ctypes.POINTER(QTensorC), i64, i64, i64, P, i64,
                                 i32, P, P]
    L.fos_amax.restype = i32
    L.fos_amax.argtypes = [P, i64, i64, i64, i64, ctypes.POINTER(Options), P, P, P]
    L.fos_dequantize.restype = i32
    L.fos_dequantize.argtypes = [ctypes.POINTER(QTensorC), i32, i64, i64, i64, u32, P, i64, P]
    L.fos_workspace_size.restype = ctypes.c_size_t
    L.fos_workspace_size.argtypes = [i64, i64, i64, ctypes.POINTER(Options)]
    L.fos_scales_size.restype = ctypes.c_size_t
    L.fos_scales_size.argtypes = [i64, i64, u32]
    L.fos_status_string.restype = ctypes.c_char_p
    L.fos_status_string.argtypes = [i32]
    L.fos_version.restype = i32
    L.fos_version.argtypes = []
    _lib = L
    return L


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


@dataclass
class QTensor:
    """One quantized orientation of a [batch, R, C] tensor (device tensors)."""
    codes: torch.Tensor              # uint8 [batch, R, C/2]
    scales: torch.Tensor             # uint8 [batch, R, C/bs] or flat swizzled
    tensor_scale: Optional[torch.Tensor]  # float32 [batch] (NVFP4)
    choice: Optional[torch.Tensor]   # uint8 bitmap, 8 * ceil(nblocks/64) bytes
    batch: int
    rows: int
    cols: int
    fmt: str
    block: str
    flags: int

    def c_struct(self) -> QTensorC:
        sld = 0 if self.flags & FLAG_SCALE_SWIZZLED else self.scales.shape[-1]
        return QTensorC(self.codes.data_ptr(), self.scales.data_ptr(),
                        self.tensor_scale.data_ptr() if self.tensor_scale is not None else None,
                        self.choice.data_ptr() if self.choice is not None else None,
                        self.codes.shape[-1], sld)


def scales_size(R: int, sf_cols: int, flags: int = 0) -> int:
    return int(lib().fos_scales_size(R, sf_cols, flags))


def workspace_size(batch: int, rows: int, cols: int, opts: Optional[Options] = None) -> int:
    return int(lib().fos_workspace_size(batch, rows, cols, ctypes.byref(opts or Options())))


def _alloc_qtensor(batch, R, C, fmt, block, flags, device, with_choice, nblocks) -> QTensor:
    bs = 32 if fmt == "mxfp4" else 16
    codes = torch.empty(batch, R, C // 2, dtype=torch.uint8, device=device)
    if flags & FLAG_SCALE_SWIZZLED:
        # zeroed where the layout has padding (rows not a multiple of 128 or
        # scale columns not a multiple of 4): the library leaves the padding
        # unwritten, and a tensor-core GEMM reads the padded scales of
        # partial tiles; without padding the quantizer writes every byte
        padded = R % 128 != 0 or (C // bs) % 4 != 0
        alloc = torch.zeros if padded else torch.empty
        scales = alloc(batch, scales_size(R, C // bs, flags), dtype=torch.uint8, device=device)
    else:
        scales = torch.empty(batch, R, C // bs, dtype=torch.uint8, device=device)
    ts = torch.empty(batch, dtype=torch.float32, device=device) if fmt != "mxfp4" else None
    ch = None
    if with_choice and fmt == "nvfp4_46":
        ch = torch.empty(8 * ((nblocks + 63) // 64), dtype=torch.uint8, device=device)
    return QTensor(codes, scales, ts, ch, batch, R, C, fmt, block, flags)


def _as3d(x: torch.Tensor) -> torch.Tensor:
    if x.dim() == 2:
        x = x.unsqueeze(0)
    if x.dim() != 3:
        raise ValueError("expected [rows, cols] or [batch, rows, cols]")
    return x


def quantize(x: torch.Tensor, fmt: str = "nvfp4_46", block: Optional[str] = None,
             rounding: str = "rne", rht: bool = False, swizzle: bool = False, seed: int = 0,
             elem_offset: int = 0, rowwise: bool = True, colwise: bool = False,
             choice: bool = True, amax: Optional[torch.Tensor] = None, rht_col: bool = False,
             status: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
             out_row: Optional[QTensor] = None, out_col: Optional[QTensor] = None,
             stream=None):
    """Quantize a CUDA bf16 tensor [batch, rows, cols] (or [rows, cols]).

    Returns (rowwise QTensor or None, colwise QTensor or None).
    """
    x = _as3d(x)
    if x.dtype != torch.bfloat16 or not x.is_cuda:
        raise TypeError("x must be a CUDA bfloat16 tensor")
    if x.stride(-1) != 1 or x.stride(0) != x.shape[1] * x.stride(1):
        raise ValueError("x rows must be contiguous with batch stride rows * ld")
    batch, rows, cols = x.shape
    ld = x.stride(1)
    block = block or ("1x32" if fmt == "mxfp4" else "1x16")
    flags = (FLAG_RHT16 if rht else 0) | (FLAG_SCALE_SWIZZLED if swizzle else 0) | \
        (FLAG_RHT16_COL if rht_col else 0)
    opts = Options(FMT[fmt], BLK[block], RND[rounding], flags, seed, elem_offset)
    bs = 32 if fmt == "mxfp4" else 16
    if block == "16x16":
        nb_row = nb_col = batch * (rows // 16) * (cols // 16)
    else:
        nb_row = batch * rows * (cols // bs)
        nb_col = batch * cols * (rows // 16)
    if rowwise and out_row is None:
        out_row = _alloc_qtensor(batch, rows, cols, fmt, block, flags, x.device, choice, nb_row)
    if colwise and out_col is None:
        out_col = _alloc_qtensor(batch, cols, rows, fmt, block, flags, x.device, choice, nb_col)
    if not rowwise:
        out_row = None
    if not colwise:
        out_col = None
    wsz = workspace_size(batch, rows, cols, opts)
    if workspace is None and (amax is None or rht_col) and fmt != "mxfp4":
        workspace = torch.empty(wsz, dtype=torch.uint8, device=x.device)
    r = out_row.c_struct() if out_row is not None else None
    c = out_col.c_struct() if out_col is not None else None
    st = lib().fos_quantize(
        ctypes.c_void_p(x.data_ptr()), batch, rows, cols, ld, ctypes.byref(opts), _ptr(amax),
        ctypes.byref(r) if r is not None else None, ctypes.byref(c) if c is not None else None,
        _ptr(workspace), workspace.numel() if workspace is not None else 0, _ptr(status),
        _stream(stream))
    if st != 0:
        raise FosError(st, "fos_quantize")
    return out_row, out_col


def fake_quantize(x: torch.Tensor, fmt: str = "nvfp4_46", rounding: str = "rne", rht: bool = False,
                  seed: int = 0, elem_offset: int = 0, amax: Optional[torch.Tensor] = None,
                  out: Optional[torch.Tensor] = None, status: Optional[torch.Tensor] = None,
                  workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Quantize and dequantize a CUDA bf16 tensor in one pass (bf16 out, same
    shape): the simulated-FP4 forward, equal to dequantize(quantize(x))."""
    x3 = _as3d(x)
    if x3.dtype != torch.bfloat16 or not x3.is_cuda:
        raise TypeError("x must be a CUDA bfloat16 tensor")
    if x3.stride(-1) != 1 or x3.stride(0) != x3.shape[1] * x3.stride(1):
        raise ValueError("x rows must be contiguous with batch stride rows * ld")
    batch, rows, cols = x3.shape
    block = "1x32" if fmt == "mxfp4" else "1x16"
    opts = Options(FMT[fmt], BLK[block], RND[rounding], FLAG_RHT16 if rht else 0, seed, elem_offset)
    if out is None:
        out = torch.empty(batch, rows, cols, dtype=torch.bfloat16, device=x3.device)
    out3 = _as3d(out)
    if workspace is None and amax is None and fmt != "mxfp4":
        workspace = torch.empty(workspace_size(batch, rows, cols, opts), dtype=torch.uint8, device=x3.device)
    st = lib().fos_fake_quantize(
        ctypes.c_void_p(x3.data_ptr()), batch, rows, cols, x3.stride(1), ctypes.byref(opts), _ptr(amax),
        ctypes.c_void_p(out3.data_ptr()), out3.stride(1), _ptr(workspace),
        workspace.numel() if workspace is not None else 0, _ptr(status), _stream(stream))
    if st != 0:
        raise FosError(st, "fos_fake_quantize")
    return out


def amax(x: torch.Tensor, rht: bool = False, seed: int = 0, out: Optional[torch.Tensor] = None,
         status: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Per-batch-entry amax of |x| (of the 16-wide RHT of x when rht)."""
    x = _as3d(x)
    batch, rows, cols = x.shape
    if out is None:
        out = torch.empty(batch, dtype=torch.float32, device=x.device)
    opts = Options(0, 0, 0, FLAG_RHT16 if rht else 0, seed, 0)
    st = lib().fos_amax(ctypes.c_void_p(x.data_ptr()), batch, rows, cols, x.stride(1),
                        ctypes.byref(opts), _ptr(out), _ptr(status), _stream(stream))
    if st != 0:
        raise FosError(st, "fos_amax")
    return out


def dequantize(q: QTensor, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Codes + scales (+ S_t) of one orientation back to bf16 [batch, R, C]."""
    if out is None:
        out = torch.empty(q.batch, q.rows, q.cols, dtype=torch.bfloat16, device=q.codes.device)
    qc = q.c_struct()
    st = lib().fos_dequantize(ctypes.byref(qc), FMT[q.fmt], q.batch, q.rows, q.cols,
                              q.flags & FLAG_SCALE_SWIZZLED, ctypes.c_void_p(out.data_ptr()),
                              out.stride(-2), _stream(stream))
    if st != 0:
        raise FosError(st, "fos_dequantize")
    return out


def gemm_nvfp4(a: QTensor, b: QTensor, out: Optional[torch.Tensor] = None, out_dtype=torch.bfloat16,
               status: Optional[torch.Tensor] = None, stream=None, wide: bool = True,
               workspace: Optional[torch.Tensor] = None) -> torch.Tensor:
    """D = (S_tA * S_tB) * A @ B^T on the tensor cores, for rowwise NVFP4
    quantizations A [M, K] and B [N, K] with swizzled scales (batch 1).
    wide: the scales are first rewritten into `workspace` (allocated here when
    None) for the wider tensor-memory scale copy (fos_gemm_nvfp4_ws); False
    runs fos_gemm_nvfp4 without a workspace.  Same result either way."""
    if not (a.flags & FLAG_SCALE_SWIZZLED and b.flags & FLAG_SCALE_SWIZZLED):
        raise ValueError("gemm_nvfp4 needs scales in the swizzled tensor-core layout")
    if a.fmt == "mxfp4" or b.fmt == "mxfp4" or a.batch != 1 or b.batch != 1 or a.cols != b.cols:
        raise ValueError("gemm_nvfp4 takes two NVFP4 [rows, K] operands with the same K")
    M, N, K = a.rows, b.rows, a.cols
    if out is None:
        out = torch.empty(M, N, dtype=out_dtype, device=a.codes.device)
    if out.dtype not in (torch.bfloat16, torch.float32) or out.stride(-1) != 1:
        raise ValueError("out must be a row-contiguous bf16 or f32 tensor")
    ac, bc = a.c_struct(), b.c_struct()
    if wide and workspace is None:
        workspace = torch.empty(gemm_workspace_size(M, N, K), dtype=torch.uint8, device=a.codes.device)
    if not wide:
        workspace = None
    st = lib().fos_gemm_nvfp4_ws(ctypes.byref(ac), ctypes.byref(bc), M, N, K, ctypes.c_void_p(out.data_ptr()),
                                 out.stride(0), 1 if out.dtype == torch.float32 else 0, _ptr(workspace),
                                 workspace.numel() if workspace is not None else 0, _ptr(status),
                                 _stream(stream))
    if st != 0:
        raise FosError(st, "fos_gemm_nvfp4_ws" if wide else "fos_gemm_nvfp4")
    return out


def gemm_workspace_size(M: int, N: int, K: int) -> int:
    """Bytes of workspace gemm_nvfp4(wide=True) needs."""
    return int(lib().fos_gemm_workspace_size(M, N, K))


def status_string(code: int) -> str:
    return lib().fos_status_string(code).decode()


def version() -> int:
    return int(lib().fos_version())
