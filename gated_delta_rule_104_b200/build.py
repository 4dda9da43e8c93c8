"""Build step of the CUDA library: nvcc -> gated_delta_rule_104_b200/libdeltalog.so.

Compiles every ``csrc/*.cu`` for sm_100a only (``-gencode
arch=compute_100a,code=sm_100a``), with line info, into one shared library
that exports the C ABI declared in ``include/deltalog.h``. The CUDA runtime
is linked statically, so the library depends only on the driver.

``--guard`` builds the index-guard debug library instead,
``libdeltalog_guard.so`` (the same sources with ``-DDL_INDEX_GUARD``: every
shared-memory write of the kernels checks its bounds and alignment, skips
and records a write that fails; see ``csrc/guard.cuh``).

Usage: ``python -m gated_delta_rule_104_b200.build [--force] [--guard] [-v]``
"""
from __future__ import annotations

import argparse
import glob
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libdeltalog.so")
GUARD_LIB = os.path.join(HERE, "libdeltalog_guard.so")
OBJDIR = os.path.join(HERE, "_build")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC,-O2", "--expt-relaxed-constexpr",
              "-Xptxas", "-warn-spills", f"-I{INCLUDE}"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libdeltalog.so")


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + \
        [os.path.join(INCLUDE, "deltalog.h"), __file__]


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(p) <= t for p in _deps())


def build(force: bool = False, verbose: bool = False, jobs: int = 0, guard: bool = False) -> str:
    lib = GUARD_LIB if guard else LIB
    if not force and up_to_date(lib):
        return lib
    objdir = OBJDIR + ("_guard" if guard else "")
    os.makedirs(objdir, exist_ok=True)
    cc = nvcc()
    objs, procs = [], []
    extra = ["-Xptxas", "-v"] if verbose else []
    if guard:
        extra.append("-DDL_INDEX_GUARD")
    for src in sources():
        obj = os.path.join(objdir, os.path.basename(src)[:-3] + ".o")
        objs.append(obj)
        cmd = [cc, *ARCH, *NVCC_FLAGS, *extra, "-c", src, "-o", obj]
        procs.append((cmd, subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.STDOUT, text=True)))
    failed = []
    for cmd, p in procs:
        out, _ = p.communicate()
        if verbose or p.returncode:
            sys.stdout.write(out)
        if p.returncode:
            failed.append(" ".join(cmd))
    if failed:
        raise RuntimeError("nvcc failed:\n" + "\n".join(failed))
    tmp = lib + f".tmp{os.getpid()}"
    subprocess.run([cc, *ARCH, "-shared", "-o", tmp, *objs], check=True)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("-v", "--verbose", action="store_true")
    ap.add_argument("--guard", action="store_true", help="the index-guard debug library")
    a = ap.parse_args()
    print(build(force=a.force, verbose=a.verbose, guard=a.guard))
