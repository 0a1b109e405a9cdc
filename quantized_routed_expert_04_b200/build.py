"""Build libstrata_moe.so in-tree with nvcc for sm_100a.

    python -m quantized_routed_expert_04_b200.build [--verbose]

Compiles every .cu under csrc/ to an object (in parallel) and links them into
quantized_routed_expert_04_b200/libstrata_moe.so.  No GPU is needed.  The
ptxas register / shared-memory report of each object goes to
_build/ptxas_<name>.log.
"""
from __future__ import annotations

import concurrent.futures
import fcntl
import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libstrata_moe.so")

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-Wall",
         "--expt-relaxed-constexpr", "-Xptxas", "-v", "-I", INCLUDE, "-I", CSRC]


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return _sources() + glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(
        os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(INCLUDE, "*.h"))


def _compile(src):
    name = os.path.splitext(os.path.basename(src))[0]
    obj = os.path.join(BUILD, name + ".o")
    log = os.path.join(BUILD, "ptxas_%s.log" % name)
    cmd = [NVCC, *ARCH, *FLAGS, "-c", src, "-o", obj]
    r = subprocess.run(cmd, capture_output=True, text=True)
    with open(log, "w") as f:
        f.write(r.stdout + r.stderr)
    if r.returncode != 0:
        raise RuntimeError("nvcc failed on %s:\n%s" % (src, r.stderr[-6000:]))
    return obj


def up_to_date() -> bool:
    """The library exists, is newer than every source, and the ptxas report
    of each source (which the tests read) is there."""
    if not os.path.exists(LIB):
        return False
    for src in _sources():
        name = os.path.splitext(os.path.basename(src))[0]
        if not os.path.exists(os.path.join(BUILD, "ptxas_%s.log" % name)):
            return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(d) <= t for d in _deps())


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile and link if a source is newer than the library.  Several
    processes may call this at once (one per GPU): a file lock lets one build
    while the others wait, then find the library up to date."""
    if not force and up_to_date():
        return LIB
    os.makedirs(BUILD, exist_ok=True)
    with open(os.path.join(BUILD, ".lock"), "w") as lock:
        fcntl.flock(lock, fcntl.LOCK_EX)
        try:
            if not force and up_to_date():
                return LIB
            return _build_locked(verbose)
        finally:
            fcntl.flock(lock, fcntl.LOCK_UN)


def _build_locked(verbose: bool) -> str:
    srcs = _sources()
    with concurrent.futures.ThreadPoolExecutor(max_workers=min(8, len(srcs))) as ex:
        objs = list(ex.map(_compile, srcs))
    tmp = LIB + ".tmp%d" % os.getpid()
    cmd = [NVCC, *ARCH, "-shared", "-Xcompiler", "-fPIC", *objs, "-o", tmp, "-lcudart"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("link failed:\n" + r.stderr[-4000:])
    os.replace(tmp, LIB)
    if verbose:
        for src in srcs:
            name = os.path.splitext(os.path.basename(src))[0]
            with open(os.path.join(BUILD, "ptxas_%s.log" % name)) as f:
                for line in f:
                    if "registers" in line or "spill" in line or "Compiling entry" in line:
                        print(line.rstrip())
    return LIB


if __name__ == "__main__":
    print(build(force=True, verbose="--verbose" in sys.argv))
