"""Build ``libif4.so`` in-tree with nvcc for sm_100a (B200).

Each CUDA source is compiled to an object with its own flags, then linked
into one shared library with a static CUDA runtime, so the library loads on
a host without a GPU (the entry points then fail with a status, never crash)
and uses whatever CUDA driver the process finds at run time.

    python -m adaptive_block_scaled_b200.build [--force]
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(os.path.dirname(HERE), "include")
OUT_DIR = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "libif4.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMMON = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-Wall",
          f"-I{INCLUDE}"]

# Per-source flags.  The quantizer must not contract a*b+c into an FMA behind
# the arithmetic contract's back, so that file is built with -fmad=false.
SOURCES = [
    ("if4_quant.cu", ["-fmad=false"]),
    ("if4_linear.cu", ["-fmad=false"]),   # shares the IF4 encoder (no contraction)
    ("if4_linear_noalloc.cu", []),
    ("ifw_quant.cu", ["-fmad=false"]),    # IF6 / IF3: the same arithmetic contract
]
HEADERS = ["if4_device.cuh", "if4_encode.cuh", "if4_decode.cuh", "if4_internal.h", "exports.map"]


def _nvcc():
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    return "nvcc"


def _newest_input():
    paths = [os.path.join(CSRC, s) for s, _ in SOURCES] + [os.path.join(CSRC, h) for h in HEADERS]
    paths.append(os.path.join(INCLUDE, "if4.h"))
    paths.append(os.path.abspath(__file__))
    return max(os.path.getmtime(p) for p in paths if os.path.exists(p))


def up_to_date() -> bool:
    return os.path.exists(LIB) and os.path.getmtime(LIB) >= _newest_input()


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and up_to_date():
        return LIB
    os.makedirs(OUT_DIR, exist_ok=True)
    nvcc = _nvcc()
    objs = []
    for src, flags in SOURCES:
        path = os.path.join(CSRC, src)
        if not os.path.exists(path):
            continue
        obj = os.path.join(OUT_DIR, src.replace(".cu", ".o"))
        cmd = [nvcc, *ARCH, *COMMON, *flags, "-c", path, "-o", obj]
        if verbose:
            print(" ".join(cmd))
        subprocess.run(cmd, check=True)
        objs.append(obj)
    tmp = LIB + ".tmp"
    cmd = [nvcc, *ARCH, "-shared", "-cudart", "static", "-o", tmp, *objs,
           "-Xlinker", f"--version-script={os.path.join(CSRC, 'exports.map')}",
           "-Xlinker", "--exclude-libs,ALL", "-Xlinker", "-Bsymbolic",
           "-lpthread", "-ldl", "-lrt"]
    if verbose:
        print(" ".join(cmd))
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
