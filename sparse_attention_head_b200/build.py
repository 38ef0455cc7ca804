"""Build libea.so in-tree with nvcc for sm_100a.

    python -m sparse_attention_head_b200.build [--verbose]

The CUDA runtime is linked statically, so the library only needs the NVIDIA
driver at run time.  Rebuilds when any source under csrc/ or include/ is
newer than the library.

The same sources are also built, with -DEA_TEST_HOOKS, into
libea_testhooks.so: that copy alone carries the failure-injection hooks
(environment variables that make a device wait run out on purpose) which the
failure-detection tests load in a child process.  libea.so has none.
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libea.so")
TESTHOOKS_LIB = os.path.join(PKG, "libea_testhooks.so")

ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc_path() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libea.so")


def sources() -> list:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _stale(lib: str) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.h")) + \
        glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(INCLUDE, "*.h"))
    return any(os.path.getmtime(p) > t for p in deps)


def _nvcc_cmd(lib: str, verbose: bool, extra) -> list:
    cmd = [nvcc_path(), "-O3", "-std=c++17", *ARCH_FLAGS, "-lineinfo",
           "-Xcompiler", "-fPIC", "-shared", "--expt-relaxed-constexpr",
           "-I", INCLUDE, "-I", CSRC, "-o", lib + ".tmp", *sources()]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    if extra:
        cmd[1:1] = list(extra)
    return cmd


def build(force: bool = False, verbose: bool = False, extra=None, testhooks: bool = True) -> str:
    """Build libea.so (and libea_testhooks.so) if stale; both nvcc runs go in
    parallel.  Returns the release library's path."""
    jobs = []
    if force or _stale(LIB):
        jobs.append((LIB, _nvcc_cmd(LIB, verbose, extra)))
    if testhooks and (force or _stale(TESTHOOKS_LIB)):
        jobs.append((TESTHOOKS_LIB, _nvcc_cmd(TESTHOOKS_LIB, False,
                                              list(extra or []) + ["-DEA_TEST_HOOKS"])))
    procs = [(lib, cmd, subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.PIPE,
                                         text=True)) for lib, cmd in jobs]
    errors = []
    for lib, cmd, proc in procs:
        out, err = proc.communicate()
        if proc.returncode != 0:
            errors.append("nvcc failed:\n" + " ".join(cmd) + "\n" + out + err)
            continue
        if verbose and lib == LIB:
            sys.stderr.write(out + err)
        os.replace(lib + ".tmp", lib)
    if errors:
        raise RuntimeError("\n".join(errors))
    return LIB


if __name__ == "__main__":
    build(force=True, verbose="--verbose" in sys.argv)
    print(LIB)
