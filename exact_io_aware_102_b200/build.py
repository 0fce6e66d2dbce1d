"""Build step for libattn.so (nvcc, sm_100a, in-tree).

``python -m exact_io_aware_102_b200.build`` compiles ``csrc/attn_fwd.cu`` and
``csrc/attn_bwd.cu`` into ``libattn.so`` next to this file.  The CUDA runtime is linked statically
and the driver is reached through cudaGetDriverEntryPoint, so the library
loads on machines without a GPU (its argument checks then still work).
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRCS = [os.path.join(HERE, "csrc", f) for f in ("attn_fwd.cu", "attn_bwd.cu")]
OUT = os.path.join(HERE, "libattn.so")
NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "-I", os.path.join(ROOT, "include"),
]


def nvcc():
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    return "nvcc"


def build(verbose=False, extra=()):
    tmp = OUT + ".tmp%d" % os.getpid()
    cmd = [nvcc()] + NVCC_FLAGS + list(extra) + ["-o", tmp] + SRCS
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.check_call(cmd)
    os.replace(tmp, OUT)
    return OUT


if __name__ == "__main__":
    print(build(verbose="-v" in sys.argv))
