"""Builds libmla_b200.so (the C-ABI library) for sm_100a with nvcc, in-tree.

    python -m mla_latent_kv_attn_b200.build [--verbose-ptxas] [--force]

Objects go to ``_build/`` at the repository root (git-ignored); the shared library lands next to
this file so that it travels with the package.  cudart is linked statically and libcuda is
reached through the runtime's driver entry points, so the library loads on machines without a
GPU driver (symbol checks) and needs none of torch's CUDA libraries.
"""
from __future__ import annotations

import argparse
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
LIB = os.path.join(PKG, "libmla_b200.so")
DEBUG_LIB = os.path.join(PKG, "libmla_b200_debug.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC,-O2", "--expt-relaxed-constexpr",
         "-I", INCLUDE, "-I", CSRC]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources():
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cu"))


def headers():
    hs = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cuh", ".h", ".map"))]
    return hs + [os.path.join(INCLUDE, f) for f in os.listdir(INCLUDE) if f.endswith(".h")]


def extra_flags(debug: bool = False):
    """MLA_NVTX=1 in the environment builds NVTX ranges around every C-ABI call (for profilers;
    off by default); debug builds add the device-side contract checks (MLA_DEBUG)."""
    f = ["-DMLA_NVTX"] if os.environ.get("MLA_NVTX") == "1" else []
    return f + (["-DMLA_DEBUG"] if debug else [])


def _compile(src: str, obj: str, ptxas_verbose: bool, debug: bool = False) -> str:
    cmd = [nvcc(), *ARCH, *FLAGS, *extra_flags(debug), "-c", src, "-o", obj]
    if ptxas_verbose:
        cmd += ["-Xptxas", "-v"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed on {os.path.basename(src)}:\n{r.stdout}\n{r.stderr}")
    return r.stdout + r.stderr


def build(force: bool = False, ptxas_verbose: bool = False, quiet: bool = True,
          debug: bool = False) -> str:
    """Builds libmla_b200.so (or, with debug, libmla_b200_debug.so from objects of its own)."""
    build_dir = os.path.join(BUILD, "debug") if debug else BUILD
    lib_path = DEBUG_LIB if debug else LIB
    os.makedirs(build_dir, exist_ok=True)
    # objects built with other flags (e.g. NVTX on/off) are rebuilt
    stamp = os.path.join(build_dir, "flags.txt")
    flags = " ".join(ARCH + FLAGS + extra_flags(debug))
    if not os.path.exists(stamp) or open(stamp).read() != flags:
        force = True
        with open(stamp, "w") as f:
            f.write(flags)
    hdr_time = max(os.path.getmtime(h) for h in headers())
    jobs = []
    objs = []
    for src in sources():
        obj = os.path.join(build_dir, os.path.basename(src)[:-3] + ".o")
        objs.append(obj)
        stale = (force or ptxas_verbose or not os.path.exists(obj)
                 or os.path.getmtime(obj) < max(os.path.getmtime(src), hdr_time))
        if stale:
            jobs.append((src, obj))
    logs = []
    if jobs:
        with cf.ThreadPoolExecutor(max_workers=min(8, len(jobs))) as ex:
            futs = [ex.submit(_compile, s, o, ptxas_verbose, debug) for s, o in jobs]
            for f in futs:
                logs.append(f.result())
    if jobs or force or not os.path.exists(lib_path) or os.path.getmtime(lib_path) < max(
            os.path.getmtime(o) for o in objs):
        cmd = [nvcc(), *ARCH, "-shared", "-Xcompiler", "-fPIC", "-o", lib_path, *objs, "-cudart",
               "static", "-Xlinker", "--version-script=" + os.path.join(CSRC, "exports.map")]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    log = "".join(logs)
    if not quiet and log:
        print(log)
    return lib_path


def main(argv=None) -> int:
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose-ptxas", action="store_true")
    ap.add_argument("--debug", action="store_true",
                    help="also build libmla_b200_debug.so (device-side contract checks)")
    a = ap.parse_args(argv)
    path = build(force=a.force, ptxas_verbose=a.verbose_ptxas, quiet=False)
    print(path)
    if a.debug:
        print(build(force=a.force, ptxas_verbose=a.verbose_ptxas, quiet=False, debug=True))
    return 0


if __name__ == "__main__":
    sys.exit(main())
