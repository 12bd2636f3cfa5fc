"""Host-side checks of libfos.so (no GPU needed): the library loads, exports
every symbol include/fos.h declares, and rejects bad arguments with the
documented status codes before touching the device."""
import ctypes
import os
import re

import pytest

import mxfp4_block_scaled_fos_b200 as F
from mxfp4_block_scaled_fos_b200 import build as fbuild
from mxfp4_block_scaled_fos_b200.fos import EXPORTS, Options, QTensorC

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    fbuild.build()
    return F.lib()


def _declared_functions():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            txt = open(os.path.join(ROOT, "include", fn)).read()
            names |= set(re.findall(r"^\s*(?:fos_status|size_t|int32_t|const char\*)\s+(fos_\w+)\s*\(",
                                    txt, re.M))
    return names


def test_exports_every_declared_symbol(L):
    declared = _declared_functions()
    assert declared, "no declarations found"
    assert declared <= set(EXPORTS)
    for name in declared:
        assert hasattr(L, name), name


def test_check_library_exports_every_declared_symbol():
    """libfos_check.so (the tests' exhaustive device checks) exports what
    include/fos_check.h declares."""
    txt = open(os.path.join(ROOT, "include", "fos_check.h")).read()
    declared = set(re.findall(r"^int\s+(fosck_\w+)\s*\(", txt, re.M))
    assert len(declared) >= 10
    C = ctypes.CDLL(fbuild.build_check())
    for name in declared:
        assert hasattr(C, name), name


def test_version_and_strings(L):
    assert F.version() == 1
    assert F.status_string(0) == "ok"
    for code in range(1, 8):
        assert F.status_string(code) != "unknown status"


def test_sizes(L):
    assert F.scales_size(2880, 180, 0) == 2880 * 180
    assert F.scales_size(2880, 180, F.FLAG_SCALE_SWIZZLED) == 2944 * 180
    assert F.scales_size(1, 1, F.FLAG_SCALE_SWIZZLED) == 512
    assert F.workspace_size(128, 2880, 2880) >= 4 * 128


def _call(L, x=16, batch=1, rows=16, cols=32, ld=32, opts=None, row=True, col=False,
          ws=16, wsb=1 << 16, amax=None):
    o = opts or Options(0, 0, 0, 0, 0, 0)
    q = QTensorC(64, 128, 256, None, cols // 2, cols // 16)
    qc = QTensorC(64, 128, 256, None, rows // 2, rows // 16)
    return L.fos_quantize(ctypes.c_void_p(x), batch, rows, cols, ld, ctypes.byref(o),
                          ctypes.c_void_p(amax) if amax else None,
                          ctypes.byref(q) if row else None, ctypes.byref(qc) if col else None,
                          ctypes.c_void_p(ws) if ws else None, wsb, None, None)


def test_argument_errors(L):
    assert _call(L, x=0) == 1                                   # NULL input
    assert _call(L, row=False, col=False) == 1                  # no output
    assert _call(L, opts=Options(3, 0, 0, 0, 0, 0)) == 7        # bad format
    assert _call(L, opts=Options(0, 0, 0, 0x80, 0, 0)) == 7     # unknown flag
    assert _call(L, x=8) == 2                                   # misaligned x
    assert _call(L, ld=36) == 2                                 # ld % 8
    assert _call(L, cols=24, ld=24) == 3                        # cols % 16
    assert _call(L, rows=15, col=True) == 3                     # colwise needs rows % 16
    assert _call(L, opts=Options(2, 0, 0, 0, 0, 0)) == 4        # MXFP4 with 1x16
    assert _call(L, opts=Options(0, 2, 0, 0, 0, 0)) == 4        # NVFP4 with 1x32
    assert _call(L, opts=Options(2, 2, 1, 0, 0, 0)) == 4        # MXFP4 + SR
    assert _call(L, opts=Options(0, 0, 0, 1, 0, 0), col=True) == 4  # RHT + colwise
    assert _call(L, opts=Options(0, 1, 0, 1, 0, 0)) == 4        # RHT + 16x16
    assert _call(L, opts=Options(0, 0, 1, 0, 0, 8)) == 7        # SR offset % 16
    assert _call(L, ws=0) == 5                                  # no workspace
    assert _call(L, wsb=16) == 5                                # workspace too small
    assert _call(L, ld=16) == 3                                 # ld < cols
    assert _call(L, rows=-1) == 3


def test_strip_hook_argument_errors(L):
    """fos_testing_quantize_2d_strip checks its own arguments before any
    device work: 16x16 blocks only, 1..8 sub-tiles per strip."""
    q = QTensorC(64, 128, 256, None, 16, 2)

    def call(blk, nsub):
        o = Options(0, blk, 0, 0, 0, 0)
        return L.fos_testing_quantize_2d_strip(ctypes.c_void_p(16), 1, 32, 32, 32, ctypes.byref(o), None,
                                               ctypes.byref(q), None, ctypes.c_void_p(16), 1 << 16, None,
                                               nsub, None)
    assert call(0, 4) == 4      # 1x16
    assert call(1, 0) == 7
    assert call(1, 9) == 7
    assert L.fos_testing_quantize_2d_strip(ctypes.c_void_p(16), 1, 32, 32, 32, None, None, ctypes.byref(q),
                                           None, None, 0, None, 4, None) == 1


def test_host_pipeline_argument_errors(L):
    """fos_quantize_host checks its arguments before enqueueing anything."""
    q = QTensorC(64, 128, 256, None, 16, 2)
    ev = (ctypes.c_void_p * 2)(16, 32)

    def call(x=16, opts=None, out_host=True, x_dev=32, chunk=1, events=True, qh=None):
        o = opts or Options(0, 0, 0, 0, 0, 0)
        return L.fos_quantize_host(ctypes.c_void_p(x) if x else None, 1, 16, 32, ctypes.byref(o), None,
                                   ctypes.byref(qh or q) if out_host else None,
                                   ctypes.c_void_p(x_dev) if x_dev else None, ctypes.byref(q),
                                   ctypes.c_void_p(16), 1 << 16, None, chunk, None, None, None,
                                   ev if events else None)
    assert call(x=0) == 1
    assert call(out_host=False) == 1
    assert call(events=False) == 1
    assert call(chunk=0) == 7
    assert call(opts=Options(0, 1, 0, 0, 0, 0)) == 4                        # 16x16
    assert call(opts=Options(0, 0, 0, 2, 0, 0)) == 4                        # swizzled scales
    assert call(qh=QTensorC(64, 128, 256, 512, 16, 2)) == 4                 # choice bits
    assert call(qh=QTensorC(64, 128, 256, None, 32, 2)) == 7                # host and device strides differ
    assert call(x_dev=48) == 2                                              # staging not 32-byte aligned
    assert call(opts=Options(3, 0, 0, 0, 0, 0)) == 7                        # bad format (fos_quantize's check)
    # 3 rows of 8 code bytes per entry: the second chunk's codes would be 8-byte aligned
    qo = QTensorC(64, 128, 256, None, 8, 1)
    o = Options(0, 0, 0, 0, 0, 0)
    assert L.fos_quantize_host(ctypes.c_void_p(16), 2, 3, 16, ctypes.byref(o), None, ctypes.byref(qo),
                               ctypes.c_void_p(32), ctypes.byref(qo), ctypes.c_void_p(16), 1 << 16, None, 1,
                               None, None, None, (ctypes.c_void_p * 4)(16, 32, 48, 64)) == 2


def test_library_has_no_oracle_dependency():
    """The product library must not link or name the CPU oracle."""
    src_dir = os.path.join(ROOT, "mxfp4_block_scaled_fos_b200")
    for dirpath, _, files in os.walk(src_dir):
        for fn in files:
            if fn.endswith((".py", ".cu", ".cuh", ".h")):
                txt = open(os.path.join(dirpath, fn)).read()
                assert "oracle" not in txt.lower(), fn


def test_missing_library_fails_loudly(tmp_path):
    """Without libfos.so the binding raises: there is no CPU fallback."""
    import subprocess
    import sys
    code = ("import torch, mxfp4_block_scaled_fos_b200 as F\n"
            "try:\n"
            "    F.quantize(torch.zeros(1, 16, 16, dtype=torch.bfloat16))\n"
            "except (RuntimeError, TypeError) as e:\n"
            "    print('raised', type(e).__name__)\n"
            "try:\n"
            "    F.lib()\n"
            "except RuntimeError as e:\n"
            "    print('raised', 'missing' in str(e))\n")
    env = dict(os.environ, FOS_LIBRARY=str(tmp_path / "no_such_libfos.so"))
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, env=env, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stderr
    assert r.stdout.split("\n")[:2] == ["raised TypeError", "raised True"], r.stdout
