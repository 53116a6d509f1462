"""Build the CUDA library in-tree: masked_block_diffusion_denoise_b200/libdlm.so.

    python -m masked_block_diffusion_denoise_b200.build [--jobs N] [--trace]

Compiles every .cu file under csrc/ for sm_100a (nvcc -gencode
arch=compute_100a,code=sm_100a -lineinfo) and links one shared library
against the shared CUDA runtime.  Sources are recompiled only when they, or a
header, are newer than their object file.  --trace builds the device-timeline
variant instead (-DDLM_TRACE, libdlm_trace.so; see dlm_trace_read in
include/dlm.h); --bounds the index-checking variant (-DDLM_DEBUG_BOUNDS,
libdlm_bounds.so: accesses whose index comes from device data are checked
and a violation is reported as DLM_EBOUNDS instead of being made).
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
BUILD = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "libdlm.so")
BUILD_TRACE = os.path.join(HERE, "_build_trace")
LIB_TRACE = os.path.join(HERE, "libdlm_trace.so")
BUILD_BOUNDS = os.path.join(HERE, "_build_bounds")
LIB_BOUNDS = os.path.join(HERE, "libdlm_bounds.so")
INCLUDE = os.path.join(os.path.dirname(HERE), "include")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-std=c++17", "-O3", "-lineinfo", "-Xcompiler", "-fPIC", "-I" + INCLUDE,
         "--expt-relaxed-constexpr"]


def _headers():
    return glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + \
        glob.glob(os.path.join(INCLUDE, "*.h"))


def _stale(src, obj, newest_header):
    if not os.path.exists(obj):
        return True
    t = os.path.getmtime(obj)
    return os.path.getmtime(src) > t or newest_header > t


def _compile(src, obj, verbose, extra=()):
    cmd = [NVCC] + ARCH + FLAGS + list(extra) + ["-c", src, "-o", obj]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("nvcc failed for %s:\n%s" % (src, r.stderr))
    return r.stderr


def build(jobs: int = 0, verbose: bool = False, trace: bool = False,
          bounds: bool = False) -> str:
    if trace and bounds:
        raise ValueError("one variant at a time: trace or bounds")
    build_dir, lib, extra = BUILD, LIB, []
    if trace:
        build_dir, lib, extra = BUILD_TRACE, LIB_TRACE, ["-DDLM_TRACE"]
    if bounds:
        build_dir, lib, extra = BUILD_BOUNDS, LIB_BOUNDS, ["-DDLM_DEBUG_BOUNDS"]
    os.makedirs(build_dir, exist_ok=True)
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    newest = max(os.path.getmtime(h) for h in _headers())
    objs, todo = [], []
    for s in srcs:
        o = os.path.join(build_dir, os.path.basename(s)[:-3] + ".o")
        objs.append(o)
        if _stale(s, o, newest) or verbose:
            todo.append((s, o))
    jobs = jobs or min(8, os.cpu_count() or 1)
    with cf.ThreadPoolExecutor(max_workers=jobs) as ex:
        for (s, o), log in zip(todo, ex.map(lambda so: _compile(so[0], so[1], verbose, extra),
                                            todo)):
            if verbose and log:
                sys.stderr.write(log)
    if todo or not os.path.exists(lib):
        cmd = [NVCC] + ARCH + ["-shared", "-cudart", "shared", "-o", lib] + objs + \
            ["-Xlinker", "-rpath,/usr/local/cuda/lib64"]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError("link failed:\n" + r.stderr)
    return lib


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--jobs", type=int, default=0)
    ap.add_argument("-v", "--verbose", action="store_true")
    ap.add_argument("--trace", action="store_true",
                    help="the device-timeline variant (libdlm_trace.so)")
    ap.add_argument("--bounds", action="store_true",
                    help="the index-checking variant (libdlm_bounds.so)")
    a = ap.parse_args()
    print(build(a.jobs, a.verbose, a.trace, a.bounds))
