"""Build libflashdec.so (the FlashDecoder C-ABI library) for sm_100a.

Usage: python -m streaming_transformer_video_b200.csrc.build  [--verbose]
The shared library is written next to the Python binding, in-tree.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
PKG = os.path.dirname(HERE)
ROOT = os.path.dirname(PKG)
LIB = os.path.join(PKG, "libflashdec.so")
SOURCES = ["fd_api.cu"]
HEADERS = ["fd_common.cuh", "fd_ptx.cuh", "fd_epilogue.cuh", "fd_simt.cuh", "fd_gemm_tc.cuh",
           "fd_attn_tc.cuh"]


def nvcc_cmd(out=LIB, extra=()):
    nvcc = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
    return [nvcc, "-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
            "-Xcompiler", "-fPIC,-fvisibility=hidden", "-shared", "--expt-relaxed-constexpr",
            "-I", os.path.join(ROOT, "include"), *extra,
            *[os.path.join(HERE, s) for s in SOURCES], "-o", out]


def up_to_date():
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    deps = [os.path.join(HERE, f) for f in SOURCES + HEADERS]
    deps.append(os.path.join(ROOT, "include", "flashdec.h"))
    return all(os.path.getmtime(d) <= t for d in deps)


def build(force=False, verbose=False):
    if not force and up_to_date():
        return LIB
    cmd = nvcc_cmd(extra=("-Xptxas", "-v") if verbose else ())
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError("nvcc failed building libflashdec.so")
    if verbose:
        sys.stderr.write(r.stderr)
    return LIB


if __name__ == "__main__":
    build(force=True, verbose="--verbose" in sys.argv)
    print(LIB)
