"""Build libmxfp8.so in-tree with nvcc for sm_100a.

    python -m mxfp8_w8a8_quantized_b200.build [--force] [--verbose]

Cross-compiles without a GPU.  The library links the CUDA runtime
statically and needs only the driver at run time.
"""
import hashlib
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libmxfp8.so")

PUBLIC_HEADERS = ["mxfp8.h", "fp8_rowwise.h", "nvfp4.h"]
SOURCES = ["mxfp8_quant.cu", "mxfp8_gemm.cu", "mxfp8_capi.cu", "mxfp8_noalloc.cu", "fp8_rowwise.cu", "nvfp4.cu"]
HEADERS = ["ptx.cuh", "mx_element.cuh", "tmap_host.cuh"]
# The files each profiled kernel is compiled from: a profile summary names
# the hash of its kernel's files, so that it goes stale only when they change.
KERNEL_FILES = {
    "mxfp8_gemm": ["mxfp8_gemm.cu", "ptx.cuh", "mx_element.cuh", "tmap_host.cuh"],
}

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for c in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if c and (os.path.sep not in c or os.path.exists(c)):
            return c
    return "nvcc"


def _inputs():
    return ([os.path.join(CSRC, s) for s in SOURCES + HEADERS]
            + [os.path.join(INCLUDE, h) for h in PUBLIC_HEADERS] + [os.path.abspath(__file__)])


def source_sha(kernel: str = None) -> str:
    """Hash of the library's sources, or of one kernel's files
    (KERNEL_FILES); ties a profile summary to one build."""
    if kernel is None:
        paths = ([os.path.join(CSRC, s) for s in SOURCES + HEADERS]
                 + [os.path.join(INCLUDE, h) for h in PUBLIC_HEADERS])
    else:
        paths = [os.path.join(CSRC, s) for s in KERNEL_FILES[kernel]]
    h = hashlib.sha256()
    for p in paths:
        with open(p, "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(p) <= t for p in _inputs())


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and up_to_date():
        return LIB
    cmd = [nvcc(), "-O3", "-std=c++17", *ARCH, "-lineinfo", "-shared", "-Xcompiler", "-fPIC",
           "-I", INCLUDE, "-I", CSRC, "-o", LIB + ".tmp"]
    if verbose:
        cmd += ["-Xptxas", "-v"]
    cmd += [os.path.join(CSRC, s) for s in SOURCES]
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv))
