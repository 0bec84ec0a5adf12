"""Build libattamba.so in-tree with nvcc for sm_100a.

    python -m ssm_compressed_chunked_b200.build [--verbose]

The library links the CUDA runtime statically and resolves the driver's
tensor-map encoder at run time, so it needs only libc and the NVIDIA driver.
"""

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libattamba.so")
SOURCES = ["abi.cu", "chunk_index.cu", "kv_ssm_scan.cu", "chunk_attn.cu", "decode.cu", "handoff.cu", "proj_gemm.cu", "device.cu"]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
         "-Xcompiler", "-fPIC", "-shared", "-cudart", "static", "-I", INCLUDE, "-I", CSRC]


def build(verbose=False):
    cmd = [NVCC] + FLAGS + (["-Xptxas", "-v"] if verbose else []) + \
        [os.path.join(CSRC, s) for s in SOURCES] + ["-o", LIB + ".tmp"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError("nvcc failed for libattamba.so")
    os.replace(LIB + ".tmp", LIB)
    if verbose:
        sys.stderr.write(r.stderr)
    return LIB


if __name__ == "__main__":
    print(build(verbose="--verbose" in sys.argv))
