"""Build libqsa.so (this package) and libqsa_synth.so (the input generator) for sm_100a.

Each .cu file is compiled to an object under _build/ in parallel, then linked with nvcc into a
shared library placed next to its Python package.  Run ``python learned_block_sparse_qsa_b200/build.py``
(or ``__graft_entry__.build()``); it does not import the package, which needs the library.
"""
from __future__ import annotations

import concurrent.futures as cf
import glob
import os
import shutil
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "learned_block_sparse_qsa_b200")
SYNTH = os.path.join(ROOT, "qsa_synth")
BUILD = os.path.join(ROOT, "_build")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-O3",
         "--expt-relaxed-constexpr"]


def nvcc() -> str:
    path = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(path):
        raise RuntimeError("nvcc not found; the CUDA toolkit is required to build libqsa")
    return path


def _compile(src: str, obj: str, extra: list[str]) -> str:
    cmd = [nvcc(), *ARCH, *FLAGS, *extra, "-c", src, "-o", obj]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed on {src}:\n{r.stdout}\n{r.stderr}")
    return r.stderr


def _stale(target: str, deps: list[str]) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def build_lib(name: str, srcdir: str, outdir: str, headers: list[str], extra: list[str] | None = None,
              verbose_ptxas: bool = False) -> str:
    extra = list(extra or [])
    if verbose_ptxas:
        extra += ["-Xptxas", "-v"]
    os.makedirs(os.path.join(BUILD, name), exist_ok=True)
    srcs = sorted(glob.glob(os.path.join(srcdir, "*.cu")))
    out = os.path.join(outdir, f"lib{name}.so")
    objs = []
    jobs = []
    with cf.ThreadPoolExecutor(max_workers=os.cpu_count() or 4) as ex:
        for s in srcs:
            o = os.path.join(BUILD, name, os.path.basename(s) + ".o")
            objs.append(o)
            if verbose_ptxas or _stale(o, [s, *headers]):
                jobs.append((s, ex.submit(_compile, s, o, extra)))
        for s, j in jobs:
            log = j.result()
            if verbose_ptxas and log:
                sys.stderr.write(f"== {os.path.basename(s)}\n{log}")
    if _stale(out, objs):
        cmd = [nvcc(), *ARCH, "-shared", "--cudart", "static", "-o", out, *objs]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link of {out} failed:\n{r.stdout}\n{r.stderr}")
    return out


def build(verbose_ptxas: bool = False) -> list[str]:
    qsa_headers = glob.glob(os.path.join(PKG, "csrc", "*.cuh")) + glob.glob(os.path.join(PKG, "csrc", "*.h"))
    qsa_headers += [os.path.join(ROOT, "include", "qsa.h")]
    lib = build_lib("qsa", os.path.join(PKG, "csrc"), PKG, qsa_headers, verbose_ptxas=verbose_ptxas)
    syn = build_lib("qsa_synth", SYNTH, SYNTH,
                    [os.path.join(SYNTH, "gen_core.h"), os.path.join(ROOT, "include", "qsa_synth.h")])
    return [lib, syn]


if __name__ == "__main__":
    for p in build(verbose_ptxas="-v" in sys.argv):
        print(p)
