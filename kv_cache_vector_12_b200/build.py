"""Build ``libtq.so`` (the C-ABI library) in-tree with nvcc for sm_100a.

Usage: ``python -m kv_cache_vector_12_b200.build [--verbose]``.  Objects go to
``_build/`` inside the package; the shared library is written next to this
file, where the binding loads it from.  nvcc cross-compiles, so no GPU is
needed to build.
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
BUILD = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "libtq.so")

# (source, object name, extra flags): tq_decode_variants.cu is compiled once
# per (head dimension, K width) slice of the attention kernel's instantiations
SOURCES = [(s, os.path.splitext(s)[0], []) for s in
           ["tq_host.cpp", "tq_fragments.cpp", "tq_api.cu", "tq_kernels.cu", "tq_quantize_tc.cu",
            "tq_quantize_qjl_tc.cu", "tq_quantize_tc256.cu", "tq_decode.cu", "tq_prefill.cu", "tq_weight.cu",
            "tq_noalloc.cu"]]
SOURCES += [("tq_decode_variants.cu", f"tq_decode_variants_d{d}_k{bk}", [f"-DTQ_DECODE_DH={d}", f"-DTQ_DECODE_BK={bk}"])
            for d in (64, 128, 256) for bk in (2, 3, 4)]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMMON = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-Wall",
          "-I" + os.path.join(ROOT, "include"), "--expt-relaxed-constexpr"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _compile(entry, verbose: bool, ptxas_v: bool) -> str:
    src, name, flags = entry
    obj = os.path.join(BUILD, name + ".o")
    path = os.path.join(CSRC, src)
    deps = [path] + [os.path.join(CSRC, h) for h in os.listdir(CSRC) if h.endswith((".h", ".cuh"))]
    deps.append(os.path.join(ROOT, "include", "tq.h"))
    if os.path.exists(obj) and all(os.path.getmtime(obj) >= os.path.getmtime(d) for d in deps) and not ptxas_v:
        return obj
    cmd = [nvcc(), *ARCH, *COMMON, *flags, "-c", path, "-o", obj]
    if ptxas_v and src.endswith(".cu"):
        cmd += ["-Xptxas", "-v"]
    if verbose:
        print(" ".join(cmd), flush=True)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
    if (verbose or ptxas_v) and (r.stdout or r.stderr):
        print(r.stdout + r.stderr, flush=True)
    return obj


def build(verbose: bool = False, ptxas_v: bool = False) -> str:
    os.makedirs(BUILD, exist_ok=True)
    with cf.ThreadPoolExecutor(max_workers=min(len(SOURCES), os.cpu_count() or 4)) as ex:
        objs = list(ex.map(lambda s: _compile(s, verbose, ptxas_v), SOURCES))
    if not os.path.exists(LIB) or any(os.path.getmtime(o) > os.path.getmtime(LIB) for o in objs):
        tmp = LIB + ".tmp"
        cmd = [nvcc(), *ARCH, "-shared", "-o", tmp, *objs, "-cudart", "static"]
        if verbose:
            print(" ".join(cmd), flush=True)
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
        os.replace(tmp, LIB)
    return LIB


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--ptxas-v", action="store_true", help="print register/smem usage per kernel")
    args = ap.parse_args(argv)
    print(build(args.verbose, args.ptxas_v))
    return 0


if __name__ == "__main__":
    sys.exit(main())
