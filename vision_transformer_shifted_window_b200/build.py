"""Builds libswinattn.so (sm_100a) in-tree with nvcc.

    python -m vision_transformer_shifted_window_b200.build [--force] [-v] [--debug]

``--debug`` builds libswinattn_debug.so instead: the same sources with
SWIN_DEBUG defined, whose kernels range-check their global-memory indices,
TMA coordinates and bias-slot reads and report a failed check through the
device status word (swin_stream_status) instead of faulting.  The binding
loads it when the environment variable SWIN_ATTN_DEBUG is 1.

Each .cu file under csrc/ is compiled separately (in parallel) and linked into
one shared library next to this file.  Rebuilds only when a source or header
is newer than the library.
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
BUILD = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "libswinattn.so")
LIB_DEBUG = os.path.join(PKG, "libswinattn_debug.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ARCH + ["-O3", "-lineinfo", "-std=c++17", "--expt-relaxed-constexpr",
                     "-Xcompiler", "-fPIC,-O2", "-I" + os.path.join(ROOT, "include")]


def _nvcc() -> str:
    cand = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(cand):
        raise RuntimeError("nvcc not found")
    return cand


def _inputs():
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    deps = srcs + sorted(glob.glob(os.path.join(CSRC, "*.cuh"))) + [
        os.path.join(ROOT, "include", "swin_attn.h")]
    return srcs, deps


def needs_build(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    _, deps = _inputs()
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(p) > t for p in deps)


def build(force: bool = False, verbose: bool = False, extra_flags=(), debug: bool = False) -> str:
    lib = LIB_DEBUG if debug else LIB
    build_dir = BUILD + ("_debug" if debug else "")
    if debug:
        extra_flags = tuple(extra_flags) + ("-DSWIN_DEBUG",)
    if not force and not needs_build(lib):
        return lib
    os.makedirs(build_dir, exist_ok=True)
    nvcc = _nvcc()
    srcs, _ = _inputs()

    def compile_one(src):
        obj = os.path.join(build_dir, os.path.basename(src)[:-3] + ".o")
        cmd = [nvcc, "-c", src, "-o", obj] + NVCC_FLAGS + list(extra_flags)
        if verbose:
            cmd.append("-Xptxas=-v")
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError("nvcc failed for %s:\n%s%s" % (src, r.stdout, r.stderr))
        if verbose:
            sys.stderr.write(r.stdout + r.stderr)
        return obj

    with cf.ThreadPoolExecutor(max_workers=max(1, min(len(srcs), os.cpu_count() or 1))) as ex:
        objs = list(ex.map(compile_one, srcs))
    tmp = lib + ".tmp.%d" % os.getpid()
    cmd = [nvcc, "-shared", "-o", tmp] + objs + ARCH + ["-lcublasLt"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("link failed:\n%s%s" % (r.stdout, r.stderr))
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("-v", "--verbose", action="store_true")
    ap.add_argument("--debug", action="store_true")
    args = ap.parse_args()
    print(build(force=args.force, verbose=args.verbose, debug=args.debug))
