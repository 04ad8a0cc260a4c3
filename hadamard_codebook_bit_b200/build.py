"""Build libcq.so (the CUDA library behind include/cq.h) in-tree for sm_100a.

Usage: python -m hadamard_codebook_bit_b200.build [--force] [-v]
Each translation unit is compiled by nvcc (in parallel) into _build/, then linked into
hadamard_codebook_bit_b200/libcq.so with the static CUDA runtime.  `-v` also prints the
ptxas resource usage (registers, spills, shared memory) of every kernel.
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
BUILD = os.path.join(ROOT, "_build", "libcq")
LIB = os.path.join(PKG, "libcq.so")

SOURCES = ["cq_api.cu", "cq_quantize.cu", "cq_quantize_tc.cu", "cq_dequantize.cu",
           "cq_dequantize_tc.cu", "cq_gemv.cu",
           "cq_gemv_static.cu", "cq_codebook.cpp"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _deps() -> list[str]:
    out = [os.path.join(INCLUDE, "cq.h")]
    for f in os.listdir(CSRC):
        out.append(os.path.join(CSRC, f))
    return out


def source_hash(files=None) -> str:
    """SHA-256 over the kernel sources and the public header (identifies a kernel build), or
    over the named files only (base names under csrc/ or include/: one kernel and the headers
    it includes)."""
    import hashlib
    h = hashlib.sha256()
    paths = _deps()
    if files is not None:
        want = set(files)
        paths = [p for p in paths if os.path.basename(p) in want]
        if {os.path.basename(p) for p in paths} != want:
            raise FileNotFoundError(f"unknown sources: {sorted(want - {os.path.basename(p) for p in paths})}")
    for path in sorted(paths):
        h.update(os.path.basename(path).encode())
        with open(path, "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def _compile(src: str, verbose: bool) -> tuple[str, str]:
    path = os.path.join(CSRC, src)
    obj = os.path.join(BUILD, src + ".o")
    cmd = [nvcc(), *ARCH, "-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC",
           "-I", INCLUDE, "-I", CSRC, "-c", path, "-o", obj]
    if src.endswith(".cu"):
        cmd += ["--expt-relaxed-constexpr"]
        if verbose:
            cmd += ["-Xptxas", "-v"]
    else:
        cmd = [nvcc(), "-O2", "-std=c++17", "-Xcompiler", "-fPIC", "-I", INCLUDE, "-I", CSRC,
               "-c", path, "-o", obj]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{res.stderr}")
    return obj, res.stderr


def build(force: bool = False, verbose: bool = False) -> str:
    stale = force or not os.path.exists(LIB) or any(
        os.path.getmtime(p) > os.path.getmtime(LIB) for p in _deps())
    if not stale:
        return LIB
    os.makedirs(BUILD, exist_ok=True)
    with cf.ThreadPoolExecutor(max_workers=len(SOURCES)) as ex:
        results = list(ex.map(lambda s: _compile(s, verbose), SOURCES))
    if verbose:
        for (_, log), src in zip(results, SOURCES):
            if log.strip():
                print(f"== {src}\n{log}", file=sys.stderr)
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [nvcc(), *ARCH, "-shared", "-o", tmp, *[o for o, _ in results], "-lpthread"]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"link failed:\n{res.stderr}")
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("-v", "--verbose", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force, verbose=a.verbose))
