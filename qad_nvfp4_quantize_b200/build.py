"""Build libnvfp4.so (the C-ABI library) in-tree for sm_100a with nvcc, and its
bounds-checking variant libnvfp4_debug.so (-DNVFP4_DEBUG_BOUNDS: every
kernel checks its computed global indices and reports NVFP4_ERR_BOUNDS).

Objects go to ``_build/`` (``_build_debug/``) beside this file; a source is
recompiled when it or any header is newer than its object. Usage: ``python
-m qad_nvfp4_quantize_b200.build [-v] [-f] [--debug]`` or ``build()`` from
Python.
"""
from __future__ import annotations

import concurrent.futures as cf
import glob
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
OBJDIR = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "libnvfp4.so")
OBJDIR_DEBUG = os.path.join(HERE, "_build_debug")
LIB_DEBUG = os.path.join(HERE, "libnvfp4_debug.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
# -fmad=false: no multiply is fused into a following add or subtract, packed
# f32x2 operations included, so every FP32 product and sum of the method is
# rounded on its own (the four_over_six error sum depends on it bit for bit).
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-fmad=false", "-Xcompiler", "-fPIC", "-DNDEBUG", f"-I{INCLUDE}"]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _headers() -> list[str]:
    return glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + \
        glob.glob(os.path.join(INCLUDE, "*.h"))


def build(verbose: bool = False, force: bool = False, debug: bool = False) -> str:
    """Compile every csrc/*.cu for sm_100a and link libnvfp4.so (debug:
    libnvfp4_debug.so with the index checks); returns its path."""
    nvcc = _nvcc()
    objdir, lib = (OBJDIR_DEBUG, LIB_DEBUG) if debug else (OBJDIR, LIB)
    flags = [*FLAGS, "-DNVFP4_DEBUG_BOUNDS"] if debug else FLAGS
    os.makedirs(objdir, exist_ok=True)
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    stamp = os.path.join(objdir, "flags.txt")
    flags_line = " ".join([*ARCH, *flags])
    if not os.path.exists(stamp) or open(stamp).read() != flags_line:
        force = True  # compiler flags changed since the objects were built
    newest_header = max((os.path.getmtime(h) for h in _headers()), default=0.0)
    jobs = []
    objs = []
    for src in srcs:
        obj = os.path.join(objdir, os.path.basename(src) + ".o")
        objs.append(obj)
        if force or not os.path.exists(obj) or os.path.getmtime(obj) < max(os.path.getmtime(src), newest_header):
            jobs.append([nvcc, *ARCH, *flags, "-c", src, "-o", obj])

    def run(cmd):
        if verbose:
            print(" ".join(cmd), flush=True)
        res = subprocess.run(cmd, capture_output=True, text=True)
        if res.returncode != 0:
            raise RuntimeError(f"nvcc failed for {cmd[-3]}:\n{res.stdout}\n{res.stderr}")
        return res

    with cf.ThreadPoolExecutor(max_workers=max(1, min(len(jobs), os.cpu_count() or 1))) as ex:
        list(ex.map(run, jobs))
    if jobs or force or not os.path.exists(lib):
        run([nvcc, *ARCH, "-shared", "-o", lib, *objs])
    with open(stamp, "w") as f:
        f.write(flags_line)
    return lib


if __name__ == "__main__":
    print(build(verbose="-v" in sys.argv, force="-f" in sys.argv, debug="--debug" in sys.argv))
