"""Build libflashsvd.so in-tree from csrc/*.cu for sm_100a.

    python -m rank_transformer_b200.build [--force] [-j N] [--trace]

Each translation unit is compiled with nvcc to an object under _build/ and
linked into rank_transformer_b200/libflashsvd.so.  Objects are rebuilt when
their source, any csrc header or include/flashsvd.h is newer.

--trace builds a separate library, libflashsvd_trace.so (objects under
_build_trace/), with FLASHSVD_TRACE defined: the fused decode kernel then
records its stage timeline (flashsvd_trace_read / flashsvd_trace_clear,
exported by that build only).  Point FLASHSVD_LIBRARY at it to load it
through the binding.  The product library never contains the trace code.
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libflashsvd.so")
BUILD_TRACE = os.path.join(ROOT, "_build_trace")
LIB_TRACE = os.path.join(PKG, "libflashsvd_trace.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-lineinfo", "-std=c++17", "--expt-relaxed-constexpr",
              "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
              "-Xptxas", "-warn-spills"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _deps_mtime() -> float:
    files = glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h"))
    files.append(os.path.join(ROOT, "include", "flashsvd.h"))
    return max(os.path.getmtime(f) for f in files if os.path.exists(f))


def _compile(src: str, force: bool, verbose_ptxas: bool, trace: bool = False) -> str:
    obj = os.path.join(BUILD_TRACE if trace else BUILD, os.path.basename(src) + ".o")
    if (not force and os.path.exists(obj)
            and os.path.getmtime(obj) >= max(os.path.getmtime(src), _deps_mtime())):
        return obj
    cmd = [nvcc(), *ARCH, *NVCC_FLAGS, "-I", os.path.join(ROOT, "include"),
           "-c", src, "-o", obj]
    if trace:
        cmd.append("-DFLASHSVD_TRACE")
    if verbose_ptxas:
        cmd += ["-Xptxas", "-v"]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed on {src}:\n{res.stdout}\n{res.stderr}")
    if verbose_ptxas and res.stderr:
        sys.stderr.write(res.stderr)
    return obj


def build(force: bool = False, jobs: int = 8, verbose_ptxas: bool = False,
          trace: bool = False) -> str:
    bdir, lib = (BUILD_TRACE, LIB_TRACE) if trace else (BUILD, LIB)
    os.makedirs(bdir, exist_ok=True)
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    with cf.ThreadPoolExecutor(max_workers=jobs) as ex:
        objs = list(ex.map(lambda s: _compile(s, force, verbose_ptxas, trace), srcs))
    if (force or not os.path.exists(lib)
            or os.path.getmtime(lib) < max(os.path.getmtime(o) for o in objs)):
        tmp = lib + ".tmp"
        cmd = [nvcc(), *ARCH, "-shared", "--cudart", "static", "-o", tmp, *objs]
        res = subprocess.run(cmd, capture_output=True, text=True)
        if res.returncode != 0:
            raise RuntimeError(f"link failed:\n{res.stdout}\n{res.stderr}")
        os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("-j", type=int, default=8)
    ap.add_argument("--ptxas-v", action="store_true")
    ap.add_argument("--trace", action="store_true",
                    help="build libflashsvd_trace.so (fused decode stage timeline)")
    a = ap.parse_args()
    print(build(a.force, a.j, a.ptxas_v, a.trace))
