"""Build the sm_100a shared library ``libstief.so`` in-tree with nvcc.

Usage: ``python -m decode_attention_stief_b200.build`` (or ``build_library()``).
nvcc cross-compiles for sm_100a without a GPU.  The CUDA runtime is linked
statically so the library loads beside any torch build.

``build_library(variant="testhooks")`` builds ``libstief_testhooks.so`` from the
same sources with ``-DSTIEF_TEST_HOOKS``: bounded waits that give up after 50 ms
and two test-only exports (a setup-barrier stall that makes the waits run out,
the address of the no-allocation scratch).  Only the timeout tests load it.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libstief.so")
VARIANTS = {  # name -> (library file, object folder, extra nvcc flags)
    None: ("libstief.so", "_build", []),
    "testhooks": ("libstief_testhooks.so", "_build_testhooks", ["-DSTIEF_TEST_HOOKS"]),
}
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "--expt-relaxed-constexpr",
    "-I", os.path.join(ROOT, "include"),
]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _stale(out: str) -> bool:
    if not os.path.exists(out):
        return True
    t = os.path.getmtime(out)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h"))
    deps += glob.glob(os.path.join(ROOT, "include", "*.h"))
    return any(os.path.getmtime(p) > t for p in deps)


def library_file(variant=None) -> str:
    return os.path.join(PKG, VARIANTS[variant][0])


def build_library(force: bool = False, verbose: bool = False, extra_flags=(),
                  variant=None) -> str:
    """Compile every csrc/*.cu for sm_100a and link the library next to this file."""
    lib_name, obj_name, variant_flags = VARIANTS[variant]
    lib = os.path.join(PKG, lib_name)
    if not force and not _stale(lib):
        return lib
    extra_flags = [*variant_flags, *extra_flags]
    objdir = os.path.join(PKG, obj_name)
    os.makedirs(objdir, exist_ok=True)
    objs, procs = [], []
    for src in sources():  # the translation units compile side by side
        obj = os.path.join(objdir, os.path.basename(src)[:-3] + ".o")
        cmd = [NVCC, *NVCC_FLAGS, *extra_flags, "-c", src, "-o", obj]
        if verbose:
            print(" ".join(cmd), flush=True)
        procs.append((cmd, subprocess.Popen(cmd)))
        objs.append(obj)
    failed = [cmd for cmd, proc in procs if proc.wait() != 0]
    if failed:
        raise subprocess.CalledProcessError(1, failed[0])
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-cudart", "static",
           *objs, "-o", tmp]
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build_library(force="--force" in sys.argv, verbose=True,
                        variant="testhooks" if "--testhooks" in sys.argv else None))
