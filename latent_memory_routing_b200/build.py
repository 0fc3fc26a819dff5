"""Builds libmsa.so in-tree for sm_100a with nvcc.

    python -m latent_memory_routing_b200.build [--verbose] [--debug]

Each csrc/*.cu is compiled to an object in parallel (nvcc -c), then linked
into latent_memory_routing_b200/libmsa.so with the static CUDA runtime (no
-lcuda: the driver's tensor-map encoder is resolved at run time).  Objects
are rebuilt only when a source or header is newer.

``--debug`` builds libmsa_debug.so instead, from the same sources with
-DMSA_DEBUG: every entry point validates the device-side index arrays it is
given (CSR offsets, memory lengths) before its kernels read through them and
waits for its own work, returning device-detected errors from the call
itself.  Its kernels are otherwise those of the release library: sources
that do not call the debug checks are linked from the release objects.
"""

from __future__ import annotations

import concurrent.futures as cf
import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(PKG, "csrc")
BUILD = os.path.join(os.path.dirname(PKG), "_build")
LIB = os.path.join(PKG, "libmsa.so")
LIB_DEBUG = os.path.join(PKG, "libmsa_debug.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC,-O2",
         "--expt-relaxed-constexpr", "-DNDEBUG"]


def nvcc() -> str:
    p = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(p):
        raise RuntimeError("nvcc not found")
    return p


def _newest_header() -> float:
    hs = glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(
        os.path.join(os.path.dirname(PKG), "include", "*.h"))
    return max((os.path.getmtime(h) for h in hs), default=0.0)


def _compile(src: str, verbose: bool, out_dir: str, extra: list[str]) -> str:
    obj = os.path.join(out_dir, os.path.basename(src)[:-3] + ".o")
    if (os.path.exists(obj) and os.path.getmtime(obj) >= os.path.getmtime(src)
            and os.path.getmtime(obj) >= _newest_header()):
        return obj
    cmd = [nvcc(), *ARCH, *FLAGS, *extra, "-c", src, "-o", obj]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed on {src}:\n{r.stdout}\n{r.stderr}")
    if verbose and r.stderr:
        sys.stderr.write(r.stderr)
    return obj


def _uses_debug_hooks(src: str) -> bool:
    """True if the source calls the debug build's checks (or tests for it);
    every other source compiles to the same object in both builds."""
    with open(src, encoding="utf-8") as f:
        text = f.read()
    return "debug_check_" in text or "debug_finish" in text or "MSA_DEBUG" in text


def build(verbose: bool = False, debug: bool = False) -> str:
    lib = LIB_DEBUG if debug else LIB
    debug_dir = os.path.join(BUILD, "debug")
    os.makedirs(BUILD, exist_ok=True)
    if debug:
        os.makedirs(debug_dir, exist_ok=True)
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))

    def obj(src: str) -> str:
        if debug and _uses_debug_hooks(src):
            return _compile(src, verbose, debug_dir, ["-DMSA_DEBUG"])
        return _compile(src, verbose, BUILD, [])

    with cf.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 4)) as ex:
        objs = list(ex.map(obj, srcs))
    if (not os.path.exists(lib)
            or max(os.path.getmtime(o) for o in objs) > os.path.getmtime(lib)):
        tmp = lib + ".tmp"
        cmd = [nvcc(), *ARCH, "-shared", "-o", tmp, *objs]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
        os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(verbose="--verbose" in sys.argv, debug="--debug" in sys.argv))
