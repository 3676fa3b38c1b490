"""Builds libgqa_attn.so in-tree from csrc/*.cu for sm_100a (nvcc, static cudart).

Usage: ``python -m long_context_causal_flash_b200.build [--verbose] [--debug-bounds]``.
Objects and the ``-Xptxas -v`` report (registers, spills, shared memory per kernel) go
to ``_build/`` at the repository root; the shared library goes next to this file.

``--debug-bounds`` builds the checked variant, libgqa_attn_debug_bounds.so, with
``-DGQA_DEBUG_BOUNDS``: the fp32 FFMA kernels (forward, dQ, dK/dV) verify every
shared-memory access against the region it belongs to and every output row index
against its buffer, skip a failing access and report GQA_ERR_DEVICE_BOUNDS through
the status word.  The package loads it instead of the normal library when the
environment sets GQA_ATTN_DEBUG_BOUNDS=1.
"""

from __future__ import annotations

import concurrent.futures as cf
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(HERE, "libgqa_attn.so")
LIB_DEBUG_BOUNDS = os.path.join(HERE, "libgqa_attn_debug_bounds.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O2", "--expt-relaxed-constexpr",
         "-Xptxas", "-v", "-I", INCLUDE, "-I", CSRC]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is needed to build libgqa_attn.so")


def sources():
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cu"))


def _stale(lib, deps):
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(d) > t for d in deps)


def build(verbose: bool = False, force: bool = False, debug_bounds: bool = False) -> str:
    lib_path = LIB_DEBUG_BOUNDS if debug_bounds else LIB
    build_dir = os.path.join(BUILD, "debug_bounds") if debug_bounds else BUILD
    defines = ["-DGQA_DEBUG_BOUNDS"] if debug_bounds else []
    os.makedirs(build_dir, exist_ok=True)
    srcs = sources()
    deps = srcs + [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".h", ".cuh"))]
    deps.append(os.path.join(INCLUDE, "gqa_attn.h"))
    if not force and not _stale(lib_path, deps + [os.path.abspath(__file__)]):
        return lib_path
    cc = nvcc()

    def compile_one(src):
        obj = os.path.join(build_dir, os.path.basename(src) + ".o")
        cmd = [cc, *ARCH, *FLAGS, *defines, "-c", src, "-o", obj]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed on {src}:\n{r.stdout}\n{r.stderr}")
        return obj, r.stderr

    with cf.ThreadPoolExecutor(max_workers=min(8, len(srcs))) as ex:
        results = list(ex.map(compile_one, srcs))
    with open(os.path.join(build_dir, "ptxas_report.txt"), "w") as f:
        for (obj, log), src in zip(results, srcs):
            f.write(f"== {os.path.basename(src)}\n{log}\n")
    tmp = lib_path + ".tmp"
    cmd = [cc, *ARCH, "-shared", "-o", tmp, *[o for o, _ in results], "-cudart", "static"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, lib_path)
    if verbose:
        with open(os.path.join(build_dir, "ptxas_report.txt")) as f:
            sys.stdout.write(f.read())
    return lib_path


if __name__ == "__main__":
    print(build(verbose="--verbose" in sys.argv, force="--force" in sys.argv,
                debug_bounds="--debug-bounds" in sys.argv))
