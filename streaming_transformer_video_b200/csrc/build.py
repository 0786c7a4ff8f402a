"""Build libflashdec.so (the FlashDecoder C-ABI library) for sm_100a, and its
bounds-checked twin libflashdec_debug.so (-DFD_DEBUG: device-side range
checks on every ring row, slot, V^T column, split-partial index and pixel
offset, reported as FD_ERR_BOUNDS through fd_status).

Usage: python -m streaming_transformer_video_b200.csrc.build  [--verbose]
The shared libraries are written next to the Python binding, in-tree.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
PKG = os.path.dirname(HERE)
ROOT = os.path.dirname(PKG)
LIB = os.path.join(PKG, "libflashdec.so")
LIB_DEBUG = os.path.join(PKG, "libflashdec_debug.so")
SOURCES = ["fd_api.cu"]
HEADERS = ["fd_common.cuh", "fd_ptx.cuh", "fd_epilogue.cuh", "fd_simt.cuh", "fd_gemm_tc.cuh",
           "fd_attn_tc.cuh"]


def nvcc_cmd(out=LIB, extra=()):
    nvcc = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
    return [nvcc, "-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
            "-Xcompiler", "-fPIC,-fvisibility=hidden", "-shared", "--expt-relaxed-constexpr",
            "-I", os.path.join(ROOT, "include"), *extra,
            *[os.path.join(HERE, s) for s in SOURCES], "-o", out]


def up_to_date(lib=LIB):
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    deps = [os.path.join(HERE, f) for f in SOURCES + HEADERS]
    deps.append(os.path.join(ROOT, "include", "flashdec.h"))
    return all(os.path.getmtime(d) <= t for d in deps)


def build(force=False, verbose=False, debug=True):
    """Compile the libraries that are missing or older than their sources
    (all of them with force); the two builds run concurrently."""
    jobs = [(LIB, ())]
    if debug:
        jobs.append((LIB_DEBUG, ("-DFD_DEBUG",)))
    procs = []
    for out, extra in jobs:
        if not force and up_to_date(out):
            continue
        cmd = nvcc_cmd(out=out, extra=(*extra, *(("-Xptxas", "-v") if verbose else ())))
        procs.append((out, subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.PIPE,
                                            text=True)))
    for out, p in procs:
        o, e = p.communicate()
        if p.returncode != 0:
            sys.stderr.write(o + e)
            raise RuntimeError(f"nvcc failed building {os.path.basename(out)}")
        if verbose:
            sys.stderr.write(e)
    return LIB


if __name__ == "__main__":
    build(force=True, verbose="--verbose" in sys.argv)
    print(LIB)
