"""Builds libsa_sketch.so in-tree with nvcc for sm_100a.

    python -m prototype_sketch_attention_b200.build [--verbose-ptxas] [--force]

Each .cu file under csrc/ compiles to an object under _build/ (in parallel). The
objects link into prototype_sketch_attention_b200/libsa_sketch.so. The CUDA runtime
is linked statically and the driver API is reached through
cudaGetDriverEntryPoint, so the library needs no -lcuda.
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
LIB = os.path.join(PKG, "libsa_sketch.so")

SOURCES = ["sa_host.cu", "sa_prep.cu", "sa_fwd_sm100.cu", "sa_fwd_simt.cu", "sa_bwd_simt.cu",
           "sa_gemm_sm100.cu", "sa_bwd_tc.cu",
           "sa_noalloc.cu", "sa_stca.cu", "sa_codec.cu", "sa_forward_host.cu", "sa_bwd_fused.cu",
           "sa_stca_keys.cu", "sa_stca_keys_bwd.cu"]
HEADERS = ["sa_common.cuh", "sa_internal.h"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for cand in (os.environ.get("CUDA_HOME", ""), "/usr/local/cuda"):
        p = os.path.join(cand, "bin", "nvcc") if cand else ""
        if p and os.path.exists(p):
            return p
    p = shutil.which("nvcc")
    if not p:
        raise RuntimeError("nvcc not found")
    return p


def _mtime(p: str) -> float:
    return os.path.getmtime(p) if os.path.exists(p) else -1.0


def _deps_mtime() -> float:
    files = [os.path.join(CSRC, h) for h in HEADERS] + [os.path.join(INCLUDE, "sa_sketch.h"), __file__]
    return max(_mtime(f) for f in files)


def _compile(src: str, verbose_ptxas: bool) -> tuple[str, str]:
    obj = os.path.join(BUILD, os.path.splitext(src)[0] + ".o")
    cmd = [nvcc(), *ARCH, "-lineinfo", "-O3", "-std=c++17", "-Xcompiler", "-fPIC",
           "--expt-relaxed-constexpr", "-I", INCLUDE, "-I", CSRC, "-c",
           os.path.join(CSRC, src), "-o", obj]
    if verbose_ptxas:
        cmd.insert(1, "-Xptxas=-v")
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
    return obj, r.stderr


def build(force: bool = False, verbose_ptxas: bool = False) -> str:
    """Compiles every CUDA source for sm_100a and links libsa_sketch.so. Returns its path."""
    os.makedirs(BUILD, exist_ok=True)
    deps = _deps_mtime()
    stale = [s for s in SOURCES
             if force or verbose_ptxas
             or _mtime(os.path.join(BUILD, os.path.splitext(s)[0] + ".o"))
             < max(_mtime(os.path.join(CSRC, s)), deps)]
    logs = {}
    if stale:
        with cf.ThreadPoolExecutor(max_workers=len(stale)) as ex:
            for src, (obj, log) in zip(stale, ex.map(lambda s: _compile(s, verbose_ptxas), stale)):
                logs[src] = log
    objs = [os.path.join(BUILD, os.path.splitext(s)[0] + ".o") for s in SOURCES]
    if stale or _mtime(LIB) < max(_mtime(o) for o in objs):
        tmp = LIB + f".tmp{os.getpid()}"
        cmd = [nvcc(), *ARCH, "-shared", "-o", tmp, *objs]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
        os.replace(tmp, LIB)
    if verbose_ptxas:
        for src, log in logs.items():
            print(f"== {src}\n{log}")
    return LIB


def main(argv=None) -> int:
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose-ptxas", action="store_true")
    a = ap.parse_args(argv)
    print(build(force=a.force, verbose_ptxas=a.verbose_ptxas))
    return 0


if __name__ == "__main__":
    sys.exit(main())
