"""Builds libsamba.so in-tree for sm_100a with nvcc (no JIT cache, no pip install).

    python -m sliding_window_attention_samba_b200.build [--verbose] [--debug-checks]

Each csrc/*.cu is compiled separately (in parallel) into _build/, then linked
with the static CUDA runtime into sliding_window_attention_samba_b200/libsamba.so.
Objects are rebuilt when their source or any csrc header is newer.
--debug-checks builds the debug-check variant instead (-DSAMBA_DEBUG_CHECKS=1:
device index checks and workspace guard bands) into _build/debug/ and
libsamba_debug.so; the binding loads it when SAMBA_DEBUG_CHECKS=1 is set.
"""
from __future__ import annotations

import concurrent.futures as cf
import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libsamba.so")
LIB_DEBUG = os.path.join(PKG, "libsamba_debug.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC,-O3", "-I" + os.path.join(ROOT, "include"),
         "--expt-relaxed-constexpr", "-Xptxas", "-warn-spills"]


def _newest_header() -> float:
    hs = glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + \
        glob.glob(os.path.join(ROOT, "include", "*.h"))
    return max((os.path.getmtime(h) for h in hs), default=0.0)


def _compile(src: str, verbose: bool, hdr_t: float, flags, outdir: str, force: bool) -> str:
    obj = os.path.join(outdir, os.path.basename(src)[:-3] + ".o")
    if not force and os.path.exists(obj) and os.path.getmtime(obj) >= max(os.path.getmtime(src), hdr_t):
        return obj
    cmd = [NVCC, *ARCH, *FLAGS, *flags, "-c", src, "-o", obj]
    if verbose:
        print(" ".join(cmd), flush=True)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
    if verbose and (r.stdout or r.stderr):
        print(r.stdout + r.stderr, flush=True)
    return obj


def build(verbose: bool = False, extra=(), debug_checks: bool = False) -> str:
    """Builds libsamba.so (or, with debug_checks, libsamba_debug.so); `extra`
    nvcc flags force a rebuild of every object."""
    outdir = os.path.join(BUILD, "debug") if debug_checks else BUILD
    lib = LIB_DEBUG if debug_checks else LIB
    flags = list(extra) + (["-DSAMBA_DEBUG_CHECKS=1"] if debug_checks else [])
    os.makedirs(outdir, exist_ok=True)
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    hdr_t = _newest_header()
    with cf.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        objs = list(ex.map(lambda s: _compile(s, verbose, hdr_t, flags, outdir, bool(extra)), srcs))
    if not os.path.exists(lib) or os.path.getmtime(lib) < max(os.path.getmtime(o) for o in objs):
        cmd = [NVCC, *ARCH, "-shared", "-o", lib, *objs, "-cudart", "static"]
        if verbose:
            print(" ".join(cmd), flush=True)
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    return lib


if __name__ == "__main__":
    extra = [a for a in sys.argv[1:] if a not in ("--verbose", "--debug-checks")]
    print(build(verbose="--verbose" in sys.argv, extra=extra, debug_checks="--debug-checks" in sys.argv))
