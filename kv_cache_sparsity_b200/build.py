"""Build the HyLRA C-ABI library (libhylra.so) for sm_100a, in-tree.

    python -m kv_cache_sparsity_b200.build [--force] [--ptxas-info]

nvcc compiles the CUDA translation unit for sm_100a only
(-gencode arch=compute_100a,code=sm_100a) and the host policy code with the
host compiler; the result sits next to this file so that it travels with
the repository.  No GPU is needed to build.
"""

from __future__ import annotations

import argparse
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libhylra.so")

SOURCES = [os.path.join(CSRC, "hylra_api.cu"), os.path.join(CSRC, "hylra_policy.cpp")]
DEPS = SOURCES + [os.path.join(CSRC, "hylra_kernels.cuh"), os.path.join(CSRC, "hylra_device.cuh"),
                  os.path.join(INCLUDE, "hylra.h")]
GENCODE = "arch=compute_100a,code=sm_100a"


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found; set NVCC or add CUDA's bin directory to PATH")


def needs_build() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(p) > t for p in DEPS)


def build(force: bool = False, ptxas_info: bool = False, verbose: bool = False) -> str:
    """Compile libhylra.so if a source changed (or ``force``); return its path."""
    if not force and not ptxas_info and not needs_build():
        return LIB
    # one temporary file per process: several ranks may build at once, and
    # each then installs a complete library with one atomic rename
    tmp = f"{LIB}.{os.getpid()}.tmp"
    cmd = [nvcc_path(), "-gencode", GENCODE, "-lineinfo", "-O3", "-std=c++17",
           "-Xcompiler", "-fPIC,-O3", "-shared", "-I", INCLUDE, "-I", CSRC,
           "-o", tmp] + SOURCES
    if ptxas_info:
        cmd.insert(1, "-Xptxas=-v")
    if verbose:
        print(" ".join(cmd), flush=True)
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        if os.path.exists(tmp):
            os.remove(tmp)
        raise RuntimeError("nvcc failed:\n" + res.stdout + res.stderr)
    if ptxas_info or verbose:
        sys.stdout.write(res.stdout + res.stderr)
    os.replace(tmp, LIB)
    return LIB


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--ptxas-info", action="store_true", help="print registers/spills/smem")
    args = ap.parse_args(argv)
    print(build(force=args.force, ptxas_info=args.ptxas_info, verbose=True))
    return 0


if __name__ == "__main__":
    raise SystemExit(main())
