"""Build libifq.so in-tree for sm_100a with nvcc.

Usage: python -m bit_complex_quantized_b200.build   (or build() from Python)
Objects go to bit_complex_quantized_b200/_build/, the library next to this file.
The ptxas resource report (registers, spills, shared memory) of each kernel
file is written to _build/<file>.ptxas.txt.
"""
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
BUILD = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "libifq.so")
SOURCES = ["api.cu", "convert.cu", "quantize.cu", "dequantize.cu", "gemv.cu", "gemv_i8.cu", "gemm.cu", "product_generic.cu"]

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O2", "--expt-relaxed-constexpr",
         "-I" + os.path.join(ROOT, "include")]


def nvcc():
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _stale(obj, deps):
    if not os.path.exists(obj):
        return True
    t = os.path.getmtime(obj)
    return any(os.path.getmtime(d) > t for d in deps)


def build(verbose=False):
    os.makedirs(BUILD, exist_ok=True)
    headers = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".h", ".cuh"))]
    headers.append(os.path.join(ROOT, "include", "ifq.h"))
    objs = []
    for src in SOURCES:
        s = os.path.join(CSRC, src)
        o = os.path.join(BUILD, src.replace(".cu", ".o"))
        objs.append(o)
        if not _stale(o, [s] + headers + [__file__]):
            continue
        cmd = [nvcc()] + ARCH + FLAGS + ["-Xptxas", "-v", "-c", s, "-o", o]
        r = subprocess.run(cmd, capture_output=True, text=True)
        with open(os.path.join(BUILD, src + ".ptxas.txt"), "w") as f:
            f.write(r.stderr)
        if r.returncode != 0:
            sys.stderr.write(r.stderr)
            raise RuntimeError("nvcc failed on " + src)
        if verbose:
            print("compiled", src)
    if _stale(LIB, objs):
        cmd = [nvcc()] + ARCH + ["-shared", "-cudart", "static", "-o", LIB] + objs
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            sys.stderr.write(r.stderr)
            raise RuntimeError("link failed")
        if verbose:
            print("linked", LIB)
    return LIB


if __name__ == "__main__":
    build(verbose=True)
