"""In-tree build of libmedusa_b200.so (and the synthetic-input generator).

Every CUDA source is compiled for sm_100a only
(``-gencode arch=compute_100a,code=sm_100a``); the shared objects land next
to their sources so they travel with the repository checkout.
"""

from __future__ import annotations

import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
REPO = os.path.dirname(PKG_DIR)
CSRC = os.path.join(PKG_DIR, "csrc")
INCLUDE = os.path.join(REPO, "include")
LIB = os.path.join(PKG_DIR, "libmedusa_b200.so")
SYNTH_SRC = os.path.join(REPO, "synth", "csrc", "synth.cu")
SYNTH_LIB = os.path.join(REPO, "synth", "libmedusa_synth.so")
BUILD_DIR = os.path.join(REPO, "_build")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMMON = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O3", "--expt-relaxed-constexpr"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _run(cmd):
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("build failed:\n" + " ".join(cmd) + "\n" + r.stdout + r.stderr)
    return r.stdout + r.stderr


def _newer(target: str, sources) -> bool:
    if not os.path.exists(target):
        return False
    t = os.path.getmtime(target)
    return all(os.path.getmtime(s) <= t for s in sources)


def library_sources():
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cu", ".cpp")))


def library_headers():
    hs = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".h", ".cuh"))]
    return hs + [os.path.join(INCLUDE, "medusa_b200.h")]


def build_library(force: bool = False, verbose: bool = False, extra=()) -> str:
    srcs = library_sources()
    if not force and _newer(LIB, srcs + library_headers() + [__file__]):
        return LIB
    os.makedirs(BUILD_DIR, exist_ok=True)
    nv = nvcc()
    objs = []
    cmds = []
    for s in srcs:
        o = os.path.join(BUILD_DIR, os.path.basename(s) + ".o")
        objs.append(o)
        cmds.append([nv, *ARCH, *COMMON, *extra, "-I", INCLUDE, "-I", CSRC, "-c", s, "-o", o])
    with ThreadPoolExecutor(max(1, min(8, os.cpu_count() or 1))) as ex:
        logs = list(ex.map(_run, cmds))
    tmp = LIB + ".tmp"
    _run([nv, *ARCH, "-shared", "-o", tmp, *objs, "-Xcompiler", "-fPIC"])
    os.replace(tmp, LIB)
    if verbose:
        sys.stdout.write("".join(logs))
    return LIB


def build_synth(force: bool = False) -> str:
    if not force and _newer(SYNTH_LIB, [SYNTH_SRC, __file__]):
        return SYNTH_LIB
    tmp = SYNTH_LIB + ".tmp"
    _run([nvcc(), *ARCH, *COMMON, "-shared", SYNTH_SRC, "-o", tmp])
    os.replace(tmp, SYNTH_LIB)
    return SYNTH_LIB


def build_all(force: bool = False, verbose: bool = False):
    return build_library(force, verbose), build_synth(force)


if __name__ == "__main__":
    force = "--force" in sys.argv
    verbose = "-v" in sys.argv
    extra = ["-Xptxas", "-v"] if "--ptxas" in sys.argv else []
    print(build_library(force or bool(extra), verbose or bool(extra), extra))
    print(build_synth(force))
