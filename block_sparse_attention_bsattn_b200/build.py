"""Build the CUDA library ``libbsattn.so`` for sm_100a with nvcc.

    python -m block_sparse_attention_bsattn_b200.build [--force] [--verbose]
    python -m block_sparse_attention_bsattn_b200.build --probes

Each ``csrc/*.cu`` is compiled to an object in ``_build/`` and the objects are
linked into ``block_sparse_attention_bsattn_b200/lib/libbsattn.so`` (CUDA
runtime linked statically, so the library does not depend on which libcudart
the host process has loaded).  Rebuilds only what changed.

``--probes`` builds the hardware microbenchmarks of ``probes/*.cu`` (MMA issue
rate, TMEM read cost, L2 -> SM stream rate, exponential rates) into
``_build/probes/``; they are measurement programs, not part of the library.
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
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(PKG, "_build")
LIBDIR = os.path.join(PKG, "lib")
LIB = os.path.join(LIBDIR, "libbsattn.so")
PROBES = os.path.join(PKG, "probes")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr",
         "-I", INCLUDE, "-I", CSRC]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _deps_mtime() -> float:
    hdrs = glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + \
        glob.glob(os.path.join(INCLUDE, "*.h"))
    return max(os.path.getmtime(h) for h in hdrs)


def build(force: bool = False, verbose: bool = False, ptxas_info: bool = False) -> str:
    os.makedirs(BUILD, exist_ok=True)
    os.makedirs(LIBDIR, exist_ok=True)
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    hdr_t = _deps_mtime()
    cc = nvcc()
    jobs = []
    for src in srcs:
        obj = os.path.join(BUILD, os.path.basename(src)[:-3] + ".o")
        stale = force or ptxas_info or not os.path.exists(obj) or \
            os.path.getmtime(obj) < max(os.path.getmtime(src), hdr_t)
        extra = ["-Xptxas", "-v"] if ptxas_info else []
        jobs.append((obj, [cc, *ARCH, *FLAGS, *extra, "-c", src, "-o", obj] if stale else None))

    def run(cmd):
        if verbose:
            print(" ".join(cmd), flush=True)
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed:\n{' '.join(cmd)}\n{r.stdout}\n{r.stderr}")
        if ptxas_info or verbose:
            sys.stderr.write(r.stderr)

    todo = [cmd for _, cmd in jobs if cmd]
    with cf.ThreadPoolExecutor(max_workers=max(1, min(len(todo), os.cpu_count() or 4))) as ex:
        list(ex.map(run, todo))
    objs = [o for o, _ in jobs]
    if todo or not os.path.exists(LIB) or os.path.getmtime(LIB) < max(os.path.getmtime(o) for o in objs):
        tmp = LIB + f".tmp{os.getpid()}"
        run([cc, *ARCH, "-shared", "-cudart", "static", "-Xcompiler", "-fPIC", *objs, "-o", tmp])
        os.replace(tmp, LIB)
    return LIB


def build_probes(verbose: bool = False) -> list:
    out_dir = os.path.join(BUILD, "probes")
    os.makedirs(out_dir, exist_ok=True)
    cc = nvcc()
    outs = []
    for src in sorted(glob.glob(os.path.join(PROBES, "*.cu"))):
        exe = os.path.join(out_dir, os.path.basename(src)[:-3])
        cmd = [cc, *ARCH, "-O3", "-std=c++17", "-I", CSRC, src, "-o", exe, "-lcuda"]
        if verbose:
            print(" ".join(cmd), flush=True)
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed:\n{' '.join(cmd)}\n{r.stdout}\n{r.stderr}")
        outs.append(exe)
    return outs


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--ptxas-info", action="store_true")
    ap.add_argument("--probes", action="store_true", help="build probes/*.cu instead of the library")
    a = ap.parse_args()
    if a.probes:
        print("\n".join(build_probes(a.verbose)))
    else:
        print(build(a.force, a.verbose, a.ptxas_info))
