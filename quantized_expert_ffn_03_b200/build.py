"""Build libmoe.so (CUDA, sm_100a) in the package directory.

    python quantized_expert_ffn_03_b200/build.py [--force]

nvcc cross-compiles for sm_100a without a GPU; the library links the CUDA
runtime statically so it does not depend on the runtime version loaded by
other libraries in the process.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libmoe.so")
SOURCES = ["moe_abi.cu", "moe_decode.cu", "moe_router.cu", "moe_pack.cu", "moe_noalloc.cu", "moe_stream.cu",
           "moe_grouped.cu"]
HEADERS = ["moe_device.cuh", "moe_kernels.h", "moe_layout.h", "moe_stream_policy.h", "moe_tc.cuh", "moe_grouped.h"]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _deps():
    paths = [os.path.join(CSRC, f) for f in SOURCES + HEADERS]
    paths.append(os.path.join(ROOT, "include", "moe.h"))
    paths.append(os.path.abspath(__file__))
    return paths


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(p) <= t for p in _deps() if os.path.exists(p))


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and up_to_date():
        return LIB
    cmd = [NVCC, "-O3", "-std=c++17", "-lineinfo", *ARCH, "-shared", "-Xcompiler", "-fPIC",
           "-Xcompiler", "-ffp-contract=off", "-cudart", "static", "-I", os.path.join(ROOT, "include"),
           "-o", LIB + ".tmp"]
    if verbose:
        cmd += ["-Xptxas", "-v"]
    cmd += [os.path.join(CSRC, f) for f in SOURCES] + ["-lpthread"]
    subprocess.check_call(cmd)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
