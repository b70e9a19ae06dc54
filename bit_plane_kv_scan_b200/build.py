"""Build libfathom.so (sm_100a) in-tree with nvcc.

    python -m bit_plane_kv_scan_b200.build [--force]

Each .cu under csrc/ is compiled to an object under _build/ (in parallel),
then linked into bit_plane_kv_scan_b200/libfathom.so; the same sources with
-DFATHOM_DEVICE_CHECKS give libfathom_checked.so (objects under
_build/checked/).  Rebuilds only when a source or header is newer than the
library.
"""

from __future__ import annotations

import concurrent.futures as cf
import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libfathom.so")
# The checked build: every plane-row, sample and candidate index the kernels
# use is bounds-checked on the device; a failure counts a device fault in the
# workspace status and the access is skipped (FATHOM_LIB=checked selects it).
LIB_CHECKED = os.path.join(PKG, "libfathom_checked.so")

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
         "--expt-relaxed-constexpr", "-I", INCLUDE, "-I", CSRC]


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return _sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(INCLUDE, "*.h"))


def needs_build(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(f) > t for f in _deps())


def _compile(src: str, verbose_ptxas: bool, checked: bool = False) -> str:
    sub = os.path.join(BUILD, "checked") if checked else BUILD
    obj = os.path.join(sub, os.path.basename(src) + ".o")
    cmd = [NVCC, *ARCH, *FLAGS, "-c", src, "-o", obj]
    if checked:
        cmd.append("-DFATHOM_DEVICE_CHECKS")
    if verbose_ptxas:
        cmd += ["-Xptxas", "-v"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("nvcc failed for %s:\n%s%s" % (src, r.stdout, r.stderr))
    if verbose_ptxas:
        sys.stderr.write(r.stderr)
    return obj


def _build_one(lib: str, checked: bool, force: bool, verbose_ptxas: bool) -> str:
    if not force and not needs_build(lib):
        return lib
    os.makedirs(os.path.join(BUILD, "checked") if checked else BUILD, exist_ok=True)
    srcs = _sources()
    with cf.ThreadPoolExecutor(max_workers=min(8, len(srcs))) as ex:
        objs = list(ex.map(lambda s: _compile(s, verbose_ptxas, checked), srcs))
    tmp = lib + ".tmp%d" % os.getpid()
    cmd = [NVCC, *ARCH, "-shared", "-Xcompiler", "-fPIC", "-o", tmp, *objs]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("link failed:\n%s%s" % (r.stdout, r.stderr))
    os.replace(tmp, lib)
    return lib


def build(force: bool = False, verbose_ptxas: bool = False, checked: bool = True) -> str:
    """Builds libfathom.so and (unless checked=False) libfathom_checked.so."""
    _build_one(LIB, False, force, verbose_ptxas)
    if checked:
        _build_one(LIB_CHECKED, True, force, False)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose_ptxas="-v" in sys.argv)
    print(LIB)
