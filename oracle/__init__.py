"""CPU oracle for Four Over Six NVFP4 quantization (test infrastructure).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library
and its Python binding) never imports, links or calls it, and the two share
no code.  The arithmetic lives in ``fos_oracle.c`` (plain C, binary32,
``-ffp-contract=off``); this module builds it with gcc on first use and
wraps it with numpy.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "fos_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

FMT_NVFP4_46, FMT_NVFP4_6, FMT_MXFP4 = 0, 1, 2
BLK_1X16, BLK_16X16, BLK_1X32 = 0, 1, 2
RND_RNE, RND_SR = 0, 1
OK, NONFINITE, UNSUPPORTED, SHAPE = 0, 1, 2, 3

CFLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math"]


class Opts(ctypes.Structure):
    _fields_ = [
        ("fmt", ctypes.c_int32),
        ("blk", ctypes.c_int32),
        ("rnd", ctypes.c_int32),
        ("rht", ctypes.c_int32),
        ("seed", ctypes.c_uint64),
        ("elem_offset", ctypes.c_int64),
        ("rht_col", ctypes.c_int32),
        ("pad", ctypes.c_int32),
    ]


def build(force: bool = False, mutant: int | None = None) -> str:
    """Compile fos_oracle.c into liboracle.so (gcc, binary32, no contraction).

    mutant k > 0 (default: the FOS_ORACLE_MUTANT environment variable, only
    set by tests/test_oracle_mutants.py) builds liboracle_m<k>.so with one
    planted mistake instead, to show that the pins catch it.
    """
    if mutant is None:
        mutant = int(os.environ.get("FOS_ORACLE_MUTANT", "0") or 0)
    path = _LIB if not mutant else os.path.join(_HERE, "liboracle_m%d.so" % mutant)
    stale = (not os.path.exists(path)) or os.path.getmtime(path) < os.path.getmtime(_SRC)
    if force or stale:
        tmp = path + ".tmp%d" % os.getpid()
        extra = ["-DOR_MUTANT=%d" % mutant] if mutant else []
        subprocess.check_call(["gcc", *CFLAGS, *extra, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, path)
    return path


def lib():
    global _lib
    with _lock:
        if _lib is None:
            L = ctypes.CDLL(build())
            P = ctypes.c_void_p
            i64, u64, i32 = ctypes.c_int64, ctypes.c_uint64, ctypes.c_int
            L.or_version.restype = i32
            L.or_e2m1_encode.restype = ctypes.c_uint8
            L.or_e2m1_encode.argtypes = [ctypes.c_float]
            L.or_e2m1_decode.restype = ctypes.c_float
            L.or_e2m1_decode.argtypes = [ctypes.c_uint8]
            L.or_e4m3_encode.restype = ctypes.c_uint8
            L.or_e4m3_encode.argtypes = [ctypes.c_float]
            L.or_e4m3_decode.restype = ctypes.c_float
            L.or_e4m3_decode.argtypes = [ctypes.c_uint8]
            L.or_e8m0_exponent.restype = i32
            L.or_e8m0_exponent.argtypes = [ctypes.c_float]
            L.or_e8m0_decode.restype = ctypes.c_float
            L.or_e8m0_decode.argtypes = [ctypes.c_uint8]
            L.or_rht16_signs.restype = ctypes.c_uint32
            L.or_rht16_signs.argtypes = [u64]
            L.or_tensor_scale.restype = ctypes.c_float
            L.or_tensor_scale.argtypes = [ctypes.c_float, i32]
            L.or_amax.restype = i32
            L.or_amax.argtypes = [P, i64, i64, i64, i32, u64, P]
            L.or_quantize.restype = i32
            L.or_quantize.argtypes = [P, i64, i64, i64, ctypes.POINTER(Opts), P,
                                      P, P, P, P, P, P, P, P]
            L.or_dequantize.restype = i32
            L.or_dequantize.argtypes = [P, P, P, i64, i64, i64, i32, P]
            L.or_swizzle_offset.restype = i64
            L.or_swizzle_offset.argtypes = [i64, i64, i64]
            L.or_swizzled_size.restype = i64
            L.or_swizzled_size.argtypes = [i64, i64]
            L.or_swizzle_scales.restype = None
            L.or_swizzle_scales.argtypes = [P, i64, i64, i64, P]
            L.or_page_example_mae.restype = ctypes.c_double
            L.or_page_example_mae.argtypes = [P, i64, i64]
            for name in ("or_e2m1_encode_array", "or_e4m3_encode_array",
                         "or_e8m0_exponent_array", "or_f32_to_bf16_array"):
                getattr(L, name).restype = None
                getattr(L, name).argtypes = [P, i64, P]
            L.or_philox_array.restype = None
            L.or_philox_array.argtypes = [P, P, i64, P]
            L.or_e2m1_sr_array.restype = None
            L.or_e2m1_sr_array.argtypes = [P, P, i64, P]
            L.or_sr_bytes.restype = None
            L.or_sr_bytes.argtypes = [u64, P, i64, P]
            L.or_rht16_rows.restype = None
            L.or_rht16_rows.argtypes = [P, i64, u64]
            _lib = L
    return _lib


def _p(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


# ---------------------------------------------------------------- codecs
def e2m1_encode(v: np.ndarray) -> np.ndarray:
    v = np.ascontiguousarray(v, dtype=np.float32)
    out = np.empty(v.shape, np.uint8)
    lib().or_e2m1_encode_array(_p(v), v.size, _p(out))
    return out


def e2m1_decode(code: int) -> float:
    return lib().or_e2m1_decode(code)


def e4m3_encode(v: np.ndarray) -> np.ndarray:
    v = np.ascontiguousarray(v, dtype=np.float32)
    out = np.empty(v.shape, np.uint8)
    lib().or_e4m3_encode_array(_p(v), v.size, _p(out))
    return out


def e4m3_decode(code: int) -> float:
    return lib().or_e4m3_decode(code)


def e8m0_exponent(v: np.ndarray) -> np.ndarray:
    v = np.ascontiguousarray(v, dtype=np.float32)
    out = np.empty(v.shape, np.int32)
    lib().or_e8m0_exponent_array(_p(v), v.size, _p(out))
    return out


def f32_to_bf16(v: np.ndarray) -> np.ndarray:
    v = np.ascontiguousarray(v, dtype=np.float32)
    out = np.empty(v.shape, np.uint16)
    lib().or_f32_to_bf16_array(_p(v), v.size, _p(out))
    return out


def philox(ctr: np.ndarray, key: np.ndarray) -> np.ndarray:
    """ctr [n,4] uint32, key [n,2] uint32 -> [n,4] uint32."""
    ctr = np.ascontiguousarray(ctr, dtype=np.uint32).reshape(-1, 4)
    key = np.ascontiguousarray(key, dtype=np.uint32).reshape(-1, 2)
    out = np.empty_like(ctr)
    lib().or_philox_array(_p(ctr), _p(key), ctr.shape[0], _p(out))
    return out


def e2m1_sr(v: np.ndarray, byte: np.ndarray) -> np.ndarray:
    v = np.ascontiguousarray(v, dtype=np.float32)
    byte = np.ascontiguousarray(byte, dtype=np.uint8)
    out = np.empty(v.shape, np.uint8)
    lib().or_e2m1_sr_array(_p(v), _p(byte), v.size, _p(out))
    return out


def sr_bytes(seed: int, g: np.ndarray) -> np.ndarray:
    g = np.ascontiguousarray(g, dtype=np.int64)
    out = np.empty(g.shape, np.uint8)
    lib().or_sr_bytes(seed, _p(g), g.size, _p(out))
    return out


def rht16_signs(seed: int) -> int:
    return lib().or_rht16_signs(seed)


def rht16(x: np.ndarray, seed: int) -> np.ndarray:
    """Apply the 16-wide RHT to consecutive groups of 16 (fp32)."""
    y = np.array(x, dtype=np.float32, copy=True, order="C")
    assert y.size % 16 == 0
    lib().or_rht16_rows(_p(y), y.size // 16, seed)
    return y


def tensor_scale(amax: float, fmt: int) -> float:
    return lib().or_tensor_scale(amax, fmt)


def swizzle_offset(r: int, c: int, sf_cols: int) -> int:
    return lib().or_swizzle_offset(r, c, sf_cols)


def swizzled_size(rows: int, sf_cols: int) -> int:
    return lib().or_swizzled_size(rows, sf_cols)


def swizzle_scales(lin: np.ndarray) -> np.ndarray:
    """lin [batch, rows, sf_cols] uint8 -> flat swizzled [batch * padded]."""
    lin = np.ascontiguousarray(lin, dtype=np.uint8)
    if lin.ndim == 2:
        lin = lin[None]
    b, r, c = lin.shape
    out = np.empty(b * swizzled_size(r, c), np.uint8)
    lib().or_swizzle_scales(_p(lin), b, r, c, _p(out))
    return out


def page_example_mae(x: np.ndarray, block: int) -> float:
    x = np.ascontiguousarray(x, dtype=np.float32)
    return lib().or_page_example_mae(_p(x), x.size, block)


# ---------------------------------------------------------------- tensors
def amax(x_bits: np.ndarray, rht: bool = False, seed: int = 0) -> np.ndarray:
    """x_bits: uint16 bf16 bits [batch, rows, cols] (or 2-D)."""
    x = np.ascontiguousarray(x_bits, dtype=np.uint16)
    if x.ndim == 2:
        x = x[None]
    b, r, c = x.shape
    out = np.zeros(b, np.float32)
    st = lib().or_amax(_p(x), b, r, c, int(rht), seed, _p(out))
    if st:
        raise ValueError("oracle: non-finite input")
    return out


def quantize(x_bits: np.ndarray, fmt: int = FMT_NVFP4_46, blk: int = BLK_1X16,
             rnd: int = RND_RNE, rht: bool = False, seed: int = 0,
             elem_offset: int = 0, rowwise: bool = True, colwise: bool = False,
             amax_in: np.ndarray | None = None, rht_col: bool = False) -> dict:
    """Quantize bf16 bits [batch, rows, cols] -> dict of numpy outputs.

    Keys: r_codes [b,rows,cols/2], r_scales [b,rows,cols/bs], r_choice (bitmap),
    c_codes [b,cols,rows/2], c_scales [b,cols,rows/16], c_choice, tensor_scale [b],
    c_tensor_scale [b] (the colwise copy's S_t; differs from tensor_scale only
    with rht_col, the 16-wide transform of the colwise blocks along rows).
    """
    x = np.ascontiguousarray(x_bits, dtype=np.uint16)
    if x.ndim == 2:
        x = x[None]
    b, r, c = x.shape
    bs = 32 if fmt == FMT_MXFP4 else 16
    out = {}
    if rowwise:
        out["r_codes"] = np.zeros((b, r, c // 2), np.uint8)
        out["r_scales"] = np.zeros((b, r, c // bs), np.uint8)
        nblk = b * r * c // bs if blk != BLK_16X16 else b * (r // 16) * (c // 16)
        out["r_choice"] = np.zeros((nblk + 7) // 8, np.uint8)
    if colwise:
        out["c_codes"] = np.zeros((b, c, r // 2), np.uint8)
        out["c_scales"] = np.zeros((b, c, r // 16), np.uint8)
        nblk_c = b * c * r // 16 if blk != BLK_16X16 else b * (r // 16) * (c // 16)
        out["c_choice"] = np.zeros((nblk_c + 7) // 8, np.uint8)
    out["tensor_scale"] = np.zeros(b, np.float32)
    out["c_tensor_scale"] = np.zeros(b, np.float32)
    o = Opts(fmt, blk, rnd, int(rht), seed, elem_offset, int(rht_col), 0)
    ain = None
    if amax_in is not None:
        ain = np.ascontiguousarray(amax_in, dtype=np.float32)
    st = lib().or_quantize(
        _p(x), b, r, c, ctypes.byref(o), _p(ain),
        _p(out.get("r_codes")), _p(out.get("r_scales")), _p(out.get("r_choice")),
        _p(out.get("c_codes")), _p(out.get("c_scales")), _p(out.get("c_choice")),
        _p(out["tensor_scale"]), _p(out["c_tensor_scale"]))
    if st == NONFINITE:
        raise ValueError("oracle: non-finite input")
    if st == UNSUPPORTED:
        raise NotImplementedError("oracle: unsupported option combination")
    if st == SHAPE:
        raise ValueError("oracle: shape not divisible by the block")
    return out


def quantize_parallel(entries, threads: int, chunk_rows: int = 64, **kw) -> list:
    """Quantize a list of [rows, cols] bf16-bit arrays (one batch entry each)
    with the oracle on `threads` host threads, for timing on many cores.

    The C calls release the GIL, so threads run in parallel.  Each entry is
    cut into row chunks: the per-entry amax is the max over the chunks'
    amaxes, then every chunk is quantized with that amax supplied (the same
    result as one call on the whole entry, since each block depends only on
    its values and S_t).  Returns the per-entry lists of chunk outputs."""
    from concurrent.futures import ThreadPoolExecutor

    tasks = []
    for e, x in enumerate(entries):
        rows = x.shape[-2]
        for r0 in range(0, rows, chunk_rows):
            tasks.append((e, r0, min(rows, r0 + chunk_rows)))

    def _amax(t):
        e, r0, r1 = t
        return amax(np.ascontiguousarray(entries[e][..., r0:r1, :]).reshape(1, r1 - r0, -1),
                    rht=kw.get("rht", False), seed=kw.get("seed", 0))[0]

    with ThreadPoolExecutor(max_workers=threads) as ex:
        part = list(ex.map(_amax, tasks))
        A = np.zeros(len(entries), np.float32)
        for (e, _, _), a in zip(tasks, part):
            A[e] = max(A[e], a)

        def _quant(t):
            e, r0, r1 = t
            xs = np.ascontiguousarray(entries[e][..., r0:r1, :]).reshape(1, r1 - r0, -1)
            rows, cols = entries[e].shape[-2], entries[e].shape[-1]
            return quantize(xs, amax_in=A[e:e + 1], elem_offset=(e * rows + r0) * cols, **kw)

        outs = list(ex.map(_quant, tasks))
    per = [[] for _ in entries]
    for (e, _, _), o in zip(tasks, outs):
        per[e].append(o)
    return per


def dequantize(codes: np.ndarray, scales: np.ndarray, tensor_scale: np.ndarray | None,
               fmt: int = FMT_NVFP4_46) -> np.ndarray:
    """codes [b,rows,cols/2], scales [b,rows,cols/bs] -> bf16 bits [b,rows,cols]."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    if codes.ndim == 2:
        codes, scales = codes[None], scales[None]
    b, r, c2 = codes.shape
    ts = np.ascontiguousarray(tensor_scale if tensor_scale is not None else np.zeros(b),
                              dtype=np.float32)
    y = np.empty((b, r, 2 * c2), np.uint16)
    st = lib().or_dequantize(_p(codes), _p(scales), _p(ts), b, r, 2 * c2, fmt, _p(y))
    if st:
        raise ValueError("oracle: bad dequantize shape")
    return y
