"""Build ``libh3b.so`` in-tree with nvcc for sm_100a.

    python -m audio_diffusion_transformer_dit_b200.build [--verbose]

Each CUDA source compiles to an object under ``_build/`` (in parallel), then
nvcc links the shared library next to this file.  The CUDA runtime is linked
statically and the driver is reached through ``cudaGetDriverEntryPoint``, so
the library loads on a machine without a GPU driver (the symbol-export tests
rely on that).

The same sources also build ``libh3b_check.so`` (``-DH3B_CHECK=1``, objects
under ``_build/check/``): every hand-indexed global access checks its index
range against its buffer's extent and records a violation in the device error
word instead of performing it.  Point ``H3B_LIBRARY`` at it to run any caller
under those checks.
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
LIB = os.path.join(PKG, "libh3b.so")
LIB_CHECK = os.path.join(PKG, "libh3b_check.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O2", "-I", INCLUDE, "-I", CSRC,
         "--expt-relaxed-constexpr"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources():
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cu"))


def _newest_input() -> float:
    paths = sources() + [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cuh", ".h"))]
    paths.append(os.path.join(INCLUDE, "h3b.h"))
    return max(os.path.getmtime(p) for p in paths)


def up_to_date() -> bool:
    newest = _newest_input()
    return all(os.path.exists(p) and os.path.getmtime(p) >= newest for p in (LIB, LIB_CHECK))


def build(verbose: bool = False, force: bool = False, ptxas_verbose: bool = False) -> str:
    """Builds libh3b.so and libh3b_check.so; returns the path of the former."""
    if not force and up_to_date():
        return LIB
    cc = nvcc()
    extra = ["-Xptxas", "-v"] if ptxas_verbose else []
    variants = [(LIB, BUILD, []), (LIB_CHECK, os.path.join(BUILD, "check"), ["-DH3B_CHECK=1"])]
    for _, objdir, _ in variants:
        os.makedirs(objdir, exist_ok=True)

    def compile_one(job):
        src, objdir, defs = job
        obj = os.path.join(objdir, os.path.basename(src) + ".o")
        cmd = [cc, *ARCH, *FLAGS, *defs, *extra, "-c", src, "-o", obj]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed for {src} {' '.join(defs)}:\n{r.stdout}\n{r.stderr}")
        return obj, r.stdout + r.stderr

    jobs = [(src, objdir, defs) for _, objdir, defs in variants for src in sources()]
    with cf.ThreadPoolExecutor(max_workers=min(10, os.cpu_count() or 1)) as ex:
        results = list(ex.map(compile_one, jobs))
    if verbose or ptxas_verbose:
        for _, log in results[:len(sources())]:
            if log.strip():
                print(log)
    n = len(sources())
    for k, (lib, _, _) in enumerate(variants):
        objs = [o for o, _ in results[k * n:(k + 1) * n]]
        tmp = lib + ".tmp"
        cmd = [cc, *ARCH, "-shared", "-cudart", "static", "-o", tmp, *objs]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed for {lib}:\n{r.stdout}\n{r.stderr}")
        os.replace(tmp, lib)
    return LIB


if __name__ == "__main__":
    print(build(verbose="--verbose" in sys.argv, force=True, ptxas_verbose="--ptxas" in sys.argv))
