"""Build the sm_100a C-ABI library in-tree: calibration_free_weight_b200/libhqq_b200.so.

nvcc cross-compiles for B200 without a GPU.  The CUDA runtime is linked
statically so the library does not depend on which libcudart torch ships.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
SOURCES = [os.path.join(CSRC, f) for f in ("hqq_kernels.cu", "hqq_api.cu", "hqq_noalloc.cu", "hqq_stream.cu",
                                                "hqq_gemv.cu", "hqq_gemm.cu")]
HEADERS = [os.path.join(CSRC, "hqq_internal.h"), os.path.join(CSRC, "hqq_device.cuh"),
           os.path.join(os.path.dirname(HERE), "include", "hqq.h")]
LIB = os.path.join(HERE, "libhqq_b200.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
         "-Xcompiler", "-fPIC", "-shared", "-cudart=static", "--expt-relaxed-constexpr"]


def build(force: bool = False, verbose: bool = False, out: str = LIB) -> str:
    newest = max(os.path.getmtime(f) for f in SOURCES + HEADERS)
    if not force and os.path.exists(out) and os.path.getmtime(out) >= newest:
        return out
    cmd = [NVCC, *FLAGS, *(["-Xptxas", "-v"] if verbose else []), *SOURCES, "-o", out]
    subprocess.run(cmd, check=True)
    return out


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
