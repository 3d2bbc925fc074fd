"""Build the C-ABI shared library ``libfa_sm100.so`` in-tree with nvcc (sm_100a only).

Usage: ``python -m exact_io_aware_94_b200.build [--force] [--verbose-ptxas] [--test-hooks]``.

``--test-hooks`` builds ``libfa_sm100_testhooks.so`` instead: the same sources
compiled with ``FA_TEST_HOOKS``, which shortens every bounded wait to 20 ms and
exports ``fa_test_inject_fault``, so the tests can make a wait run out.  The
product library never contains the hooks.
"""
from __future__ import annotations

import argparse
import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB_NAME = "libfa_sm100.so"
LIB_PATH = os.path.join(PKG, LIB_NAME)
TEST_LIB_PATH = os.path.join(PKG, "libfa_sm100_testhooks.so")

ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _inputs():
    return sources() + glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.cuh")) + \
        glob.glob(os.path.join(INCLUDE, "*.h"))


def up_to_date(path: str = LIB_PATH) -> bool:
    if not os.path.exists(path):
        return False
    t = os.path.getmtime(path)
    return all(os.path.getmtime(f) <= t for f in _inputs())


def build(force: bool = False, verbose_ptxas: bool = False, jobs: int | None = None, test_hooks: bool = False) -> str:
    out_path = TEST_LIB_PATH if test_hooks else LIB_PATH
    if not force and up_to_date(out_path):
        return out_path
    nvcc = nvcc_path()
    objdir = os.path.join(PKG, "_build_testhooks" if test_hooks else "_build")
    os.makedirs(objdir, exist_ok=True)
    common = ARCH_FLAGS + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-I" + INCLUDE, "-I" + CSRC,
                           "--expt-relaxed-constexpr"]
    if test_hooks:
        common += ["-DFA_TEST_HOOKS"]
    if verbose_ptxas:
        common += ["-Xptxas", "-v"]
    objs = []
    procs = []
    for src in sources():
        obj = os.path.join(objdir, os.path.basename(src) + ".o")
        objs.append(obj)
        procs.append((src, subprocess.Popen([nvcc, "-c", src, "-o", obj] + common, stdout=subprocess.PIPE,
                                            stderr=subprocess.STDOUT, text=True)))
    failed = False
    for src, pr in procs:
        out, _ = pr.communicate()
        if out.strip():
            sys.stderr.write(out)
        if pr.returncode != 0:
            failed = True
            sys.stderr.write("nvcc failed on %s\n" % src)
    if failed:
        raise RuntimeError("CUDA build failed")
    tmp = out_path + ".tmp%d" % os.getpid()
    subprocess.check_call([nvcc, "-shared", "-o", tmp] + objs + ARCH_FLAGS + ["-Xcompiler", "-fPIC"])
    os.replace(tmp, out_path)
    return out_path


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose-ptxas", action="store_true")
    ap.add_argument("--test-hooks", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force, verbose_ptxas=a.verbose_ptxas, test_hooks=a.test_hooks))
