"""Build libonetrans.so in-tree with nvcc for sm_100a.

    python -m unified_transformer_recommender_onetrans_b200.build [--force] [--checked]

Every .cu under csrc/ is compiled with
``-gencode arch=compute_100a,code=sm_100a -lineinfo -O3`` (in parallel) and
linked into one shared library next to this file (``_lib/libonetrans.so``),
which the ctypes binding loads.  ``--checked`` builds the debug variant
``_lib/libonetrans_checked.so`` with ``-DOT_DEVICE_CHECKS``: the kernels'
plain row-mapped loads and stores are checked against the extents of the
caller's buffers and a violation is reported as OT_ERR_DEVICE_BOUNDS instead
of being made (the binding loads it when OT_CHECKED=1).  No GPU is needed to
build.
"""

from __future__ import annotations

import glob
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(os.path.dirname(HERE), "include")
OUT_DIR = os.path.join(HERE, "_lib")
LIB = os.path.join(OUT_DIR, "libonetrans.so")
LIB_CHECKED = os.path.join(OUT_DIR, "libonetrans_checked.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _nvcc() -> str:
    for p in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if p and (os.path.isabs(p) and os.path.exists(p) or not os.path.isabs(p)):
            return p
    return "nvcc"


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _stale(lib: str) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.cuh"))
    deps += glob.glob(os.path.join(INCLUDE, "*.h"))
    return any(os.path.getmtime(p) > t for p in deps)


def build(force: bool = False, verbose: bool = False, checked: bool = False) -> str:
    lib = LIB_CHECKED if checked else LIB
    if not force and not _stale(lib):
        return lib
    os.makedirs(OUT_DIR, exist_ok=True)
    nvcc = _nvcc()
    common = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC",
                     "-I", INCLUDE, "-I", CSRC]
    if checked:
        common += ["-DOT_DEVICE_CHECKS"]
    if verbose:
        common += ["-Xptxas", "-v"]
    tag = ".checked" if checked else ""
    objs = [os.path.join(OUT_DIR, os.path.basename(src) + f"{tag}.{os.getpid()}.o") for src in sources()]

    def compile_one(pair):
        src, obj = pair
        subprocess.run([nvcc, *common, "-c", src, "-o", obj], check=True)

    with ThreadPoolExecutor(max_workers=max(1, min(8, os.cpu_count() or 1))) as ex:
        list(ex.map(compile_one, zip(sources(), objs)))
    tmp = lib + f".tmp{os.getpid()}"
    subprocess.run([nvcc, *ARCH, "-shared", "-o", tmp, *objs], check=True)
    os.replace(tmp, lib)
    for o in objs:
        os.remove(o)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv, checked="--checked" in sys.argv))
