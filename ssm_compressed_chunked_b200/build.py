"""Build libattamba.so and libattamba_checked.so in-tree with nvcc for sm_100a.

    python -m ssm_compressed_chunked_b200.build [--verbose]

The library links the CUDA runtime statically and resolves the driver's
tensor-map encoder at run time, so it needs only libc and the NVIDIA driver.
libattamba_checked.so is the same source compiled with ATTAMBA_CHECKED: the
kernels test their index computations against the arrays they address and
report a failure in the status word (ATTAMBA_DEV_BOUNDS) instead of making the
access.  It is a debugging build, selected with ATTAMBA_LIBRARY=checked.
"""

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libattamba.so")
LIB_CHECKED = os.path.join(HERE, "libattamba_checked.so")
SOURCES = ["abi.cu", "chunk_index.cu", "kv_ssm_scan.cu", "chunk_attn.cu", "decode.cu", "handoff.cu", "proj_gemm.cu", "device.cu"]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
         "-Xcompiler", "-fPIC", "-shared", "-cudart", "static", "-I", INCLUDE, "-I", CSRC]


def _nvcc(out, extra, verbose):
    cmd = [NVCC] + FLAGS + extra + (["-Xptxas", "-v"] if verbose else []) + \
        [os.path.join(CSRC, s) for s in SOURCES] + ["-o", out + ".tmp"]
    return subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True), out


def build(verbose=False):
    jobs = [_nvcc(LIB, [], verbose), _nvcc(LIB_CHECKED, ["-DATTAMBA_CHECKED"], verbose)]
    for proc, out in jobs:
        so, se = proc.communicate()
        if proc.returncode != 0:
            sys.stderr.write(so + se)
            raise RuntimeError(f"nvcc failed for {os.path.basename(out)}")
        os.replace(out + ".tmp", out)
        if verbose:
            sys.stderr.write(se)
    return LIB


if __name__ == "__main__":
    print(build(verbose="--verbose" in sys.argv))
