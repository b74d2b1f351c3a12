"""Build libsbp.so in-tree with nvcc for sm_100a (B200).

    python -m memory_efficient_exact_chunk_b200.build [--ptxas-v] [--timing]

Each .cu under csrc/ is compiled to an object in _build/ (in parallel) and linked into
memory_efficient_exact_chunk_b200/libsbp.so with the CUDA runtime linked statically, so the
library loads on a machine without a GPU (symbols can be listed, nothing is launched).
`--timing` builds a separate instrumented library, libsbp_timing.so (objects in
_build_timing/), whose pair GEMM prints per-launch cycle accounts (SBP_GEMM_TIMING); the
product library is not touched.
"""
from __future__ import annotations

import concurrent.futures as cf
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libsbp.so")
BUILD_TIMING = os.path.join(ROOT, "_build_timing")
LIB_TIMING = os.path.join(PKG, "libsbp_timing.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
CFLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-Wall",
          "--expt-relaxed-constexpr", f"-I{INCLUDE}", f"-I{CSRC}"]


def nvcc() -> str:
    for c in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if c and os.path.exists(c):
            return c
    raise RuntimeError("nvcc not found")


def _sources():
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cu"))


def _deps_mtime():
    return max(os.path.getmtime(os.path.join(d, f)) for d in (CSRC, INCLUDE)
               for f in os.listdir(d))


def build(force: bool = False, verbose: bool = False, extra: list[str] | None = None,
          timing: bool = False) -> str:
    srcs = _sources()
    lib_path, build_dir = (LIB_TIMING, BUILD_TIMING) if timing else (LIB, BUILD)
    if timing:
        extra = (extra or []) + ["-DSBP_GEMM_TIMING"]
    if not force and os.path.exists(lib_path) and os.path.getmtime(lib_path) >= _deps_mtime():
        return lib_path
    os.makedirs(build_dir, exist_ok=True)
    cc = nvcc()
    flags = CFLAGS + (extra or [])

    def compile_one(src):
        obj = os.path.join(build_dir, os.path.basename(src)[:-3] + ".o")
        cmd = [cc, *ARCH, *flags, "-c", src, "-o", obj]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
        if verbose and (r.stdout or r.stderr):
            print(r.stdout, r.stderr, file=sys.stderr)
        return obj

    with cf.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        objs = list(ex.map(compile_one, srcs))
    tmp = lib_path + ".tmp"
    cmd = [cc, *ARCH, "-shared", "-cudart", "static", "-o", tmp, *objs]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, lib_path)
    return lib_path


if __name__ == "__main__":
    extra = []
    if "--ptxas-v" in sys.argv:
        extra += ["-Xptxas", "-v"]
    print(build(force=True, verbose="--ptxas-v" in sys.argv, extra=extra,
                timing="--timing" in sys.argv))
