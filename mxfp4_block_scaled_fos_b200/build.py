"""Build libfos.so (sm_100a) in-tree with nvcc.

    python -m mxfp4_block_scaled_fos_b200.build [--force] [--verbose-ptxas]

Every .cu under csrc/ is compiled for sm_100a only (no PTX for other
architectures), without fast-math, with contraction off and IEEE division,
so that the binary32 steps the quantizer defines are rounded as written.
Objects go to _build/ at the repository root; the library lands next to
this file, where the Python binding loads it.

The same flags build libfos_check.so from csrc/check/ (the exhaustive
device-side checks of the kernels' arithmetic helpers, used by the tests
only; include/fos_check.h).
"""
from __future__ import annotations

import argparse
import glob
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libfos.so")
CHECK_SRC = os.path.join(CSRC, "check", "fos_check.cu")
CHECK_LIB = os.path.join(PKG, "libfos_check.so")

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC,-O2", "-ftz=false",
         "-prec-div=true", "-prec-sqrt=true", "-fmad=false", "--expt-relaxed-constexpr",
         "-I", INCLUDE, "-I", CSRC]


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return _sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + \
        glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(INCLUDE, "*.h")) + [__file__]


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(d) <= t for d in _deps())


def build(force: bool = False, verbose_ptxas: bool = False, quiet: bool = True,
          defines=(), out: str | None = None) -> str:
    """Compile every csrc/*.cu and link libfos.so (or `out`, with extra -D
    `defines`, e.g. tuning constants; objects then go to a separate folder)."""
    lib = out or LIB
    if not force and not defines and out is None and up_to_date():
        return LIB
    bdir = BUILD if not defines else os.path.join(BUILD, "variant_%d" % abs(hash(tuple(defines))))
    os.makedirs(bdir, exist_ok=True)
    extra = ["-Xptxas", "-v"] if verbose_ptxas else []
    extra += ["-D" + d for d in defines]

    def compile_one(src):
        obj = os.path.join(bdir, os.path.basename(src) + ".o")
        cmd = [NVCC, *ARCH, *FLAGS, *extra, "-c", src, "-o", obj]
        p = subprocess.run(cmd, capture_output=True, text=True)
        if p.returncode != 0:
            raise RuntimeError("nvcc failed for %s:\n%s" % (src, p.stderr[-8000:]))
        return obj, p.stderr

    with ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        results = list(ex.map(compile_one, _sources()))
    if verbose_ptxas or not quiet:
        for _, err in results:
            sys.stderr.write(err)
    objs = [o for o, _ in results]
    tmp = lib + ".tmp%d" % os.getpid()
    cmd = [NVCC, *ARCH, "-shared", "-cudart", "static", "-o", tmp, *objs]
    p = subprocess.run(cmd, capture_output=True, text=True)
    if p.returncode != 0:
        raise RuntimeError("nvcc link failed:\n" + p.stderr[-8000:])
    os.replace(tmp, lib)
    return lib


def build_check(force: bool = False) -> str:
    """Compile csrc/check/fos_check.cu into libfos_check.so (test checks)."""
    deps = [CHECK_SRC] + glob.glob(os.path.join(CSRC, "*.cuh")) + \
        glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(INCLUDE, "*.h")) + [__file__]
    if not force and os.path.exists(CHECK_LIB) and \
            all(os.path.getmtime(d) <= os.path.getmtime(CHECK_LIB) for d in deps):
        return CHECK_LIB
    tmp = CHECK_LIB + ".tmp%d" % os.getpid()
    cmd = [NVCC, *ARCH, *FLAGS, "-shared", "-cudart", "static", "-o", tmp, CHECK_SRC]
    p = subprocess.run(cmd, capture_output=True, text=True)
    if p.returncode != 0:
        raise RuntimeError("nvcc failed for %s:\n%s" % (CHECK_SRC, p.stderr[-8000:]))
    os.replace(tmp, CHECK_LIB)
    return CHECK_LIB


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose-ptxas", action="store_true")
    args = ap.parse_args()
    print(build(force=args.force, verbose_ptxas=args.verbose_ptxas, quiet=False))
    print(build_check(force=args.force))


if __name__ == "__main__":
    main()
