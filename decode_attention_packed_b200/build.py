"""Build libmxa.so in-tree for sm_100a.

    python -m decode_attention_packed_b200.build [--force] [--verbose]

nvcc cross-compiles without a GPU; the library links the CUDA runtime
statically and looks the tensor-map encoder up through the runtime's driver
entry point, so it loads on a machine without a GPU as well.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libmxa.so")
SOURCES = [os.path.join(CSRC, "mxa_kernels.cu"), os.path.join(CSRC, "mxa_api.cpp"),
           os.path.join(CSRC, "mxa_noalloc.cu")]
DEPS = SOURCES + [os.path.join(CSRC, f) for f in ("mxa_config.h", "mxa_device.cuh", "mxa_launch.h")] + \
    [os.path.join(INCLUDE, "mxa.h")]

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
         "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden", "--expt-relaxed-constexpr",
         "-I" + INCLUDE, "-I" + CSRC]


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(f) > t for f in DEPS)


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not _stale():
        return LIB
    objs = []
    for src in SOURCES:
        obj = os.path.join(CSRC, os.path.basename(src) + ".o")
        cmd = [NVCC, *FLAGS, "-c", src, "-o", obj]
        if verbose and src.endswith(".cu"):
            cmd += ["-Xptxas", "-v"]
        subprocess.check_call(cmd)
        objs.append(obj)
    tmp = LIB + ".tmp"
    subprocess.check_call([NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-shared",
                           "-Xcompiler", "-fPIC", *objs, "-o", tmp, "-lcudart_static", "-ldl", "-lrt",
                           "-lpthread"])
    os.replace(tmp, LIB)
    for o in objs:
        os.remove(o)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv))
