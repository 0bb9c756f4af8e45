"""Build libbat.so in-tree for sm_100a.

    python -m prefix_shared_attention_b200.build [--force] [--verbose] [--debug | --phase]

Every CUDA source is compiled with nvcc for ``sm_100a`` only (tcgen05, TMA) and linked
with the static CUDA runtime into ``prefix_shared_attention_b200/libbat.so``.  Objects go
to ``prefix_shared_attention_b200/_build/``.  Sources newer than the library trigger a
rebuild of their object.

``--debug`` builds ``libbat_debug.so`` instead (objects in ``_build_debug/``), compiled with
``-DBAT_DEBUG``: its kernels check every tensor-map coordinate and store index against the
tensors' bounds and report a failed check through the device status word (no check traps).
Select it at run time with ``BAT_LIBRARY=<path to libbat_debug.so>``.

``--phase`` builds ``libbat_phase.so`` (objects in ``_build_phase/``), compiled with
``-DBAT_PHASE``: every warp of the attention kernel adds up the clocks it spends in each phase
of its loop and writes the totals once at its end (``phase_profile.py`` runs and reports it).
"""

from __future__ import annotations

import argparse
import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "libbat.so")
BUILD_DEBUG = os.path.join(PKG, "_build_debug")
LIB_DEBUG = os.path.join(PKG, "libbat_debug.so")
BUILD_PHASE = os.path.join(PKG, "_build_phase")
LIB_PHASE = os.path.join(PKG, "libbat_phase.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O3", "-I", INCLUDE, "-I", CSRC,
         "-diag-suppress", "177"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libbat.so")


def sources():
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cu", ".cpp")))


def headers():
    hs = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".h")]
    return hs + [os.path.join(INCLUDE, f) for f in os.listdir(INCLUDE) if f.endswith(".h")]


def _mtime(p):
    return os.path.getmtime(p) if os.path.exists(p) else -1.0


def build(force: bool = False, verbose: bool = False, ptxas_verbose: bool = False, debug: bool = False,
          phase: bool = False) -> str:
    assert not (debug and phase), "one variant at a time"
    build_dir, lib = (BUILD_DEBUG, LIB_DEBUG) if debug else (BUILD_PHASE, LIB_PHASE) if phase else (BUILD, LIB)
    flags = FLAGS + (["-DBAT_DEBUG"] if debug else []) + (["-DBAT_PHASE"] if phase else [])
    os.makedirs(build_dir, exist_ok=True)
    cc = nvcc()
    newest_header = max(_mtime(h) for h in headers())
    jobs = []
    objs = []
    for src in sources():
        obj = os.path.join(build_dir, os.path.basename(src) + ".o")
        objs.append(obj)
        if force or _mtime(obj) < max(_mtime(src), newest_header):
            cmd = [cc] + ARCH + flags + (["-Xptxas", "-v"] if ptxas_verbose else []) + ["-c", src, "-o", obj]
            if src.endswith(".cpp"):
                cmd = [cc] + flags + ["-x", "c++", "-c", src, "-o", obj]
            jobs.append(cmd)

    def run(cmd):
        if verbose:
            print(" ".join(cmd), flush=True)
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"compile failed: {' '.join(cmd)}\n{r.stdout}\n{r.stderr}")
        if verbose or ptxas_verbose:
            sys.stdout.write(r.stdout + r.stderr)

    with ThreadPoolExecutor(max_workers=min(8, max(1, len(jobs)))) as ex:
        list(ex.map(run, jobs))
    if force or jobs or _mtime(lib) < max(_mtime(o) for o in objs):
        tmp = lib + ".tmp"
        cmd = [cc] + ARCH + ["-shared", "-cudart", "static", "-o", tmp] + objs + ["-lpthread", "-ldl", "-lrt"]
        run(cmd)
        os.replace(tmp, lib)
    return lib


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--ptxas-verbose", action="store_true")
    ap.add_argument("--debug", action="store_true", help="build libbat_debug.so (device-side bounds checks)")
    ap.add_argument("--phase", action="store_true", help="build libbat_phase.so (per-warp phase clocks)")
    a = ap.parse_args()
    print(build(a.force, a.verbose, a.ptxas_verbose, a.debug, a.phase))


if __name__ == "__main__":
    main()
