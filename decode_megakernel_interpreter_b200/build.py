"""Build libmk.so (the C-ABI engine) in-tree with nvcc for sm_100a."""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libmk.so")
SOURCES = ["api.cu", "interp.cu", "interp_spec_llama1b.cu", "interp_spec_llama1b_batched.cu",
           "interp_spec_llama1b_batched_tqo.cu", "interp_spec_llama8b.cu",
           "noalloc.cu", "planner.cpp"]
HEADERS = ["mk_internal.h", "planner.h", "interp_body.cuh", "interp_launch.h"]
PUBLIC = [os.path.join(ROOT, "include", h) for h in ("mk.h", "mk_host.h")]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O2,-pthread", "--expt-relaxed-constexpr",
         "-Xcudafe", "--diag_suppress=177"]


def _inputs():
    return [os.path.join(CSRC, f) for f in SOURCES + HEADERS] + PUBLIC + [__file__]


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(f) <= t for f in _inputs())


def build(force: bool = False, verbose: bool = False, ptxas_info: bool = False) -> str:
    if not force and up_to_date():
        return LIB
    objdir = os.path.join(HERE, "_build")
    os.makedirs(objdir, exist_ok=True)
    objs, procs = [], []
    # every translation unit compiles in its own nvcc process, in parallel
    for src in SOURCES:
        obj = os.path.join(objdir, src + ".o")
        cmd = [NVCC, *ARCH, *FLAGS, "-c", os.path.join(CSRC, src), "-o", obj]
        if ptxas_info and src.endswith(".cu"):
            cmd.insert(1, "-Xptxas=-v")
        if verbose:
            print(" ".join(cmd), file=sys.stderr)
        log = open(obj + ".log", "w")
        procs.append((src, subprocess.Popen(cmd, stdout=log, stderr=subprocess.STDOUT), log, obj + ".log"))
        objs.append(obj)
    failed = []
    for src, proc, log, log_path in procs:
        rc = proc.wait()
        log.close()
        if verbose or rc != 0:
            with open(log_path) as f:
                sys.stderr.write(f.read())
        if rc != 0:
            failed.append(src)
    if failed:
        raise subprocess.CalledProcessError(1, "nvcc " + " ".join(failed))
    tmp = LIB + ".tmp"
    subprocess.check_call([NVCC, *ARCH, "-shared", "-o", tmp, *objs, "-Xcompiler", "-pthread"])
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True, ptxas_info="--ptxas" in sys.argv)
    print(LIB)
