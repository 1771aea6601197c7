"""Build libpa.so in-tree with nvcc for sm_100a.

Usage: python -m pagedattention_decode_03_b200.build [--verbose] [--ptxas-info] [--nvtx]

Compiles every source under csrc/ (CUDA and host C++) and links one shared
library next to this file.  Objects go to csrc/_build/ (ignored by git).
Nothing needs a GPU: nvcc cross-compiles for sm_100a.

--nvtx (or PA_NVTX=1 in the environment) defines PA_NVTX: every C-ABI call
then opens an NVTX range named after it (header-only NVTX 3, nothing to link).
A change of these options rebuilds the library.
"""
from __future__ import annotations

import argparse
import concurrent.futures
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
BUILD = os.path.join(CSRC, "_build")
LIB = os.path.join(HERE, "libpa.so")
INCLUDE = os.path.join(ROOT, "include")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMMON = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-Wall",
          "-I", INCLUDE, "-I", CSRC, "--expt-relaxed-constexpr"]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _sources():
    return sorted(f for f in os.listdir(CSRC) if f.endswith((".cu", ".cpp")))


def _defines(nvtx: bool) -> list[str]:
    return ["-DPA_NVTX"] if nvtx else []


def _compile(src: str, ptxas_info: bool, nvtx: bool = False) -> tuple[str, str]:
    obj = os.path.join(BUILD, src + ".o")
    cmd = [_nvcc(), *ARCH, *COMMON, *_defines(nvtx), "-c", os.path.join(CSRC, src), "-o", obj]
    if src.endswith(".cpp"):
        cmd[1:1] = ["-x", "cu"]
    if ptxas_info and src.endswith(".cu"):
        cmd.append("-Xptxas=-v")
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed on {src}:\n{r.stdout}\n{r.stderr}")
    return obj, r.stderr


STAMP = os.path.join(BUILD, "options.txt")


def _stale(objs, options: str) -> bool:
    if not os.path.exists(LIB):
        return True
    try:
        with open(STAMP) as f:
            if f.read() != options:
                return True
    except OSError:
        return True
    lib_t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cu", ".cpp", ".h", ".cuh"))]
    deps.append(os.path.join(INCLUDE, "pa.h"))
    deps.append(os.path.abspath(__file__))
    return any(os.path.getmtime(d) > lib_t for d in deps)


def build(force: bool = False, verbose: bool = False, ptxas_info: bool = False,
          nvtx: bool | None = None) -> str:
    if nvtx is None:
        nvtx = os.environ.get("PA_NVTX", "") not in ("", "0")
    os.makedirs(BUILD, exist_ok=True)
    srcs = _sources()
    options = " ".join(_defines(nvtx))
    if not force and not ptxas_info and not _stale(srcs, options):
        return LIB
    with concurrent.futures.ThreadPoolExecutor(max_workers=min(8, len(srcs))) as ex:
        results = list(ex.map(lambda s: _compile(s, ptxas_info, nvtx), srcs))
    if verbose or ptxas_info:
        for _, log in results:
            if log.strip():
                print(log, file=sys.stderr)
    tmp = LIB + ".tmp"
    cmd = [_nvcc(), *ARCH, "-shared", "-Xcompiler", "-fPIC", "-o", tmp,
           *[o for o, _ in results], "-lcudart_static", "-ldl", "-lpthread", "-lrt"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, LIB)
    with open(STAMP, "w") as f:
        f.write(options)
    return LIB


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--ptxas-info", action="store_true")
    ap.add_argument("--nvtx", action="store_true", help="NVTX range around every C-ABI call")
    a = ap.parse_args()
    print(build(force=a.force, verbose=a.verbose, ptxas_info=a.ptxas_info, nvtx=True if a.nvtx else None))


if __name__ == "__main__":
    main()
