"""Builds libsta.so (release) and libsta_debug.so (device bounds checks,
STA_DEBUG=1) in-tree for sm_100a with nvcc.

    python -m block_sparse_local_b200.build [--verbose]

The library is one translation unit (csrc/sta_lib.cu includes the kernel
headers) compiled with -gencode arch=compute_100a,code=sm_100a.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIB_PATH = os.path.join(HERE, "libsta.so")
DEBUG_LIB_PATH = os.path.join(HERE, "libsta_debug.so")
SOURCES = [os.path.join(HERE, "csrc", "sta_lib.cu")]
DEPENDS = SOURCES + [os.path.join(HERE, "csrc", f) for f in
                     ("device_ptx.cuh", "reorder.cuh", "tile_lists.cuh",
                      "attn_fwd.cuh", "attn_fwd_pair.cuh", "attn_bwd.cuh", "attn_bwd_dq.cuh",
                      "hilbert.cuh")] + [os.path.join(ROOT, "include", "sta.h")]


def nvcc_path():
    cuda = os.environ.get("CUDA_HOME", "/usr/local/cuda")
    p = os.path.join(cuda, "bin", "nvcc")
    return p if os.path.exists(p) else "nvcc"


def command(out=LIB_PATH, extra=()):
    return [nvcc_path(), "-gencode", "arch=compute_100a,code=sm_100a", "-O3",
            "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-shared",
            "-I" + os.path.join(ROOT, "include"), *extra, "-o", out, *SOURCES]


def up_to_date(path=LIB_PATH):
    if not os.path.exists(path):
        return False
    t = os.path.getmtime(path)
    return all(os.path.getmtime(f) <= t for f in DEPENDS)


def build(force=False, verbose=False, debug=True):
    """Builds libsta.so and (debug=True) libsta_debug.so, in parallel."""
    jobs = [(LIB_PATH, ())]
    if debug:
        jobs.append((DEBUG_LIB_PATH, ("-DSTA_DEBUG=1",)))
    procs = []
    for path, defs in jobs:
        if not force and up_to_date(path):
            continue
        extra = tuple(defs) + (("-Xptxas", "-v") if verbose else ())
        procs.append((path, subprocess.Popen(command(out=path, extra=extra),
                                             stdout=subprocess.PIPE, stderr=subprocess.PIPE,
                                             text=True)))
    for path, proc in procs:
        out, err = proc.communicate()
        if verbose or proc.returncode != 0:
            sys.stderr.write(out + err)
        if proc.returncode != 0:
            raise RuntimeError(f"nvcc failed building {os.path.basename(path)}")
    return LIB_PATH


if __name__ == "__main__":
    build(force=True, verbose="--verbose" in sys.argv)
    print(LIB_PATH)
