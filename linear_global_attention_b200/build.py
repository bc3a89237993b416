"""Build libzebra.so (sm_100a) in-tree with nvcc.

Usage: python -m linear_global_attention_b200.build [-v]
Objects go to linear_global_attention_b200/_build/; the shared library lands
next to this file. Sources are recompiled only when they (or a header) are
newer than their object.
"""
from __future__ import annotations

import concurrent.futures as cf
import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "libzebra.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
              "--expt-relaxed-constexpr", "-Xptxas", "-warn-spills"]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _cuda_lib_dir(nvcc: str) -> str:
    return os.path.join(os.path.dirname(os.path.dirname(os.path.realpath(nvcc))), "lib64")


def _newest_header() -> float:
    hs = glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(INCLUDE, "*.h"))
    return max((os.path.getmtime(h) for h in hs), default=0.0)


def build(verbose: bool = False, force: bool = False, extra_flags=None, out: str = None) -> str:
    """Compile every csrc/*.cu and link the shared library (default: next to this file).

    `extra_flags` (e.g. ["-DZEBRA_TC_STAGES=6"]) and `out` build a variant into
    its own object directory and library path.
    """
    nvcc = _nvcc()
    lib = out or LIB
    build_dir = BUILD if not out else os.path.join(BUILD, "variant_" + os.path.basename(out).replace(".", "_"))
    os.makedirs(build_dir, exist_ok=True)
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    hdr_t = _newest_header()
    flags = NVCC_FLAGS + list(extra_flags or [])

    def compile_one(src):
        obj = os.path.join(build_dir, os.path.basename(src) + ".o")
        if not force and os.path.exists(obj) and os.path.getmtime(obj) >= max(os.path.getmtime(src), hdr_t):
            return obj, ""
        cmd = [nvcc, *ARCH, *flags, "-I", INCLUDE, "-I", CSRC, "-c", src, "-o", obj]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed on {os.path.basename(src)}:\n{r.stderr}")
        return obj, r.stderr

    with cf.ThreadPoolExecutor(max(1, min(len(srcs), os.cpu_count() or 1))) as ex:
        results = list(ex.map(compile_one, srcs))
    objs = [o for o, _ in results]
    if verbose:
        for o, log in results:
            if log.strip():
                print(f"--- {os.path.basename(o)}\n{log}", file=sys.stderr)
    libdir = _cuda_lib_dir(nvcc)
    newest_obj = max(os.path.getmtime(o) for o in objs)
    if force or not os.path.exists(lib) or os.path.getmtime(lib) < newest_obj:
        cmd = [nvcc, *ARCH, "-shared", "-o", lib + ".tmp", *objs, "-L", libdir, "-lcublasLt",
               "-Xlinker", f"-rpath,{libdir}"]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stderr}")
        os.replace(lib + ".tmp", lib)
    return lib


if __name__ == "__main__":
    import argparse
    ap = argparse.ArgumentParser()
    ap.add_argument("-v", action="store_true")
    ap.add_argument("-f", action="store_true")
    ap.add_argument("--define", action="append", default=[], help="extra -D definitions, e.g. ZEBRA_TC_STAGES=6")
    ap.add_argument("--out", default=None, help="library path of a variant build")
    a = ap.parse_args()
    print(build(verbose=a.v, force=a.f, extra_flags=["-D" + d for d in a.define], out=a.out))
