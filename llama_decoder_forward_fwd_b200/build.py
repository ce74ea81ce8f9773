"""Build the CUDA library liblfwd.so in-tree with nvcc for sm_100a.

Usage: ``python -m llama_decoder_forward_fwd_b200.build [--force] [-v]``.
Objects go to ``_build/`` at the repository root; the shared library lands next
to this file so that it travels with the source tree. The same sources are also
built with -DLLM_BOUNDS_CHECK into liblfwd_checked.so (objects in
``_build/checked``): the bounds-checking build, whose kernels check the indices
that come from run-time data and report a failed check instead of accessing.
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
LIB = os.path.join(PKG, "liblfwd.so")
LIB_CHECKED = os.path.join(PKG, "liblfwd_checked.so")
VARIANTS = {"plain": (LIB, BUILD, []), "checked": (LIB_CHECKED, os.path.join(BUILD, "checked"), ["-DLLM_BOUNDS_CHECK"])}

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-O3",
                     "--expt-relaxed-constexpr", "-I", INCLUDE, "-I", CSRC]


def nvcc() -> str:
    for c in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if c and os.path.exists(c):
            return c
    raise RuntimeError("nvcc not found")


def sources():
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cu"))


def headers():
    hs = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cuh", ".h"))]
    hs += [os.path.join(INCLUDE, f) for f in os.listdir(INCLUDE) if f.endswith(".h")]
    return hs


def _mtime(p):
    return os.path.getmtime(p) if os.path.exists(p) else -1.0


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = _mtime(lib)
    return all(_mtime(f) <= t for f in sources() + headers() + [os.path.abspath(__file__)])


def _compile(src: str, verbose: bool, extra=(), build_dir: str = BUILD):
    obj = os.path.join(build_dir, os.path.basename(src)[:-3] + ".o")
    cmd = [nvcc()] + NVCC_FLAGS + list(extra) + ["-c", src, "-o", obj]
    if verbose:
        print(" ".join(cmd), flush=True)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
    if verbose and (r.stdout or r.stderr):
        print(r.stdout, r.stderr, flush=True)
    return obj


def build(force: bool = False, verbose: bool = False, ptxas_info: bool = False, variant: str = "all") -> str:
    """Compile every .cu under csrc/ and link liblfwd.so and (variant "all")
    liblfwd_checked.so; returns the path of liblfwd.so (or of the one variant asked for)."""
    if variant == "all":
        build(force, verbose, ptxas_info, "checked")
        return build(force, verbose, ptxas_info, "plain")
    lib, build_dir, defs = VARIANTS[variant]
    if not force and not ptxas_info and up_to_date(lib):
        return lib
    os.makedirs(build_dir, exist_ok=True)
    extra = defs + (["-Xptxas", "-v"] if ptxas_info else [])
    with cf.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        objs = list(ex.map(lambda s: _compile(s, verbose or ptxas_info, extra, build_dir), sources()))
    tmp = lib + ".tmp"
    cmd = [nvcc()] + ARCH + ["-shared", "-o", tmp] + objs + ["-lcuda"] * 0
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="-v" in sys.argv, ptxas_info="--ptxas" in sys.argv)
    print(LIB)
