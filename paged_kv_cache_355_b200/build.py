"""Build libpa.so (the CUDA kernels and their C ABI) in-tree for sm_100a.

    python -m paged_kv_cache_355_b200.build [--force] [--verbose]

Each csrc/*.cu (and host-only csrc/*.cpp) is compiled separately (in parallel) with
``-gencode arch=compute_100a,code=sm_100a -O3 -lineinfo`` into _build/, then
linked into paged_kv_cache_355_b200/libpa.so with the CUDA runtime linked
statically, so the library does not depend on which libcudart the host
process has loaded.  The same objects, with pa_decode.cu and pa_prefill.cu
compiled once more with -DPA_TIMELINE, make libpa_timeline.so (per-CTA
timelines of the decode and prefill kernels, include/pa_timeline.h; read by
``python -m paged_kv_cache_355_b200.timeline``).
"""
from __future__ import annotations

import argparse
import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD_DIR = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libpa.so")
TIMELINE_LIB = os.path.join(PKG, "libpa_timeline.so")

ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]
CFLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O2", "--expt-relaxed-constexpr",
          "-I", INCLUDE, "-I", CSRC]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libpa.so")


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cpp")))


def _headers():
    return sorted(glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h"))
                  + glob.glob(os.path.join(INCLUDE, "*.h")))


def _mtime(path: str) -> float:
    return os.path.getmtime(path) if os.path.exists(path) else -1.0


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile what changed and (re)link libpa.so; returns its path."""
    nvcc = _nvcc()
    os.makedirs(BUILD_DIR, exist_ok=True)
    newest_header = max((_mtime(h) for h in _headers()), default=0.0)
    jobs, objs = [], []
    # the timeline build's objects, replacing these of libpa.so
    timeline_objs_of = {name: os.path.join(BUILD_DIR, name.replace(".cu", "_timeline.cu") + ".o")
                        for name in ("pa_decode.cu", "pa_prefill.cu")}
    units = [(src, os.path.join(BUILD_DIR, os.path.basename(src) + ".o"), []) for src in _sources()]
    units += [(os.path.join(CSRC, name), obj, ["-DPA_TIMELINE"]) for name, obj in timeline_objs_of.items()]
    for src, obj, extra in units:
        if not extra:
            objs.append(obj)
        if force or _mtime(obj) < max(_mtime(src), newest_header):
            cmd = [nvcc, *ARCH_FLAGS, *CFLAGS, *extra, "-c", src, "-o", obj]
            if verbose:
                cmd.insert(1, "-Xptxas=-v")
            jobs.append((src, subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.STDOUT, text=True)))
    failed = []
    for src, proc in jobs:
        out, _ = proc.communicate()
        if verbose or proc.returncode:
            sys.stderr.write(out)
        if proc.returncode:
            failed.append(os.path.basename(src))
    if failed:
        raise RuntimeError(f"nvcc failed for {', '.join(failed)}")
    timeline_objs = [timeline_objs_of.get(os.path.basename(o)[:-2], o) for o in objs]
    for lib, lib_objs in ((LIB, objs), (TIMELINE_LIB, timeline_objs)):
        if force or jobs or _mtime(lib) < max(_mtime(o) for o in lib_objs):
            tmp = lib + f".tmp{os.getpid()}"
            subprocess.run([nvcc, *ARCH_FLAGS, "-shared", "-cudart", "static", "-o", tmp, *lib_objs], check=True)
            os.replace(tmp, lib)
    return LIB


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true", help="print ptxas register/spill reports")
    a = ap.parse_args()
    print(build(force=a.force, verbose=a.verbose))
