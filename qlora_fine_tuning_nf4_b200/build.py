"""Build libqlora.so in-tree for sm_100a with nvcc.

    python -m qlora_fine_tuning_nf4_b200.build [--verbose-ptxas] [--check]

Compiles every ``csrc/*.cu`` into ``qlora_fine_tuning_nf4_b200/lib/libqlora.so``
(C ABI declared in ``include/qlora.h``; CUDA runtime linked statically).
``--check`` builds the debug variant ``lib/libqlora_check.so`` instead: the
same sources with -DQLORA_CHECK, whose kernels check their indices and
arguments, record QL_DEV_BAD_CONFIG in the status word and skip the access on
a failed check.  Rebuilds only when a source or header is newer than the
library.
"""

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIBDIR = os.path.join(PKG, "lib")
LIB = os.path.join(LIBDIR, "libqlora.so")
LIB_CHECK = os.path.join(LIBDIR, "libqlora_check.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "--expt-relaxed-constexpr",
]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _inputs():
    return sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + [os.path.join(ROOT, "include", "qlora.h")]


def up_to_date(lib=LIB):
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(p) <= t for p in _inputs())


def build(force=False, verbose_ptxas=False, check=False):
    """Compile the shared library, or with check=True its bounds-checked debug
    variant (no-op when it is newer than its sources)."""
    lib = LIB_CHECK if check else LIB
    if not force and not verbose_ptxas and up_to_date(lib):
        return lib
    os.makedirs(LIBDIR, exist_ok=True)
    objs = []
    extra = (["-Xptxas", "-v"] if verbose_ptxas else []) + (["-DQLORA_CHECK"] if check else [])
    suffix = "_check.o" if check else ".o"
    for src in sources():
        obj = os.path.join(LIBDIR, os.path.basename(src)[:-3] + suffix)
        cmd = [NVCC, *FLAGS, *extra, "-I", os.path.join(ROOT, "include"), "-c", src, "-o", obj]
        subprocess.run(cmd, check=True)
        objs.append(obj)
    tmp = lib + ".tmp"
    subprocess.run([NVCC, "-shared", "-gencode", "arch=compute_100a,code=sm_100a", "-o", tmp, *objs], check=True)
    os.replace(tmp, lib)
    for o in objs:
        os.remove(o)
    return lib


if __name__ == "__main__":
    print(build(force=True, verbose_ptxas="--verbose-ptxas" in sys.argv, check="--check" in sys.argv))
