"""Build libqlora_nf4.so in-tree for sm_100a with nvcc.

Usage: python -m bit_nf4_quantised_b200.build  (or call build()).
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_NAME = "libqlora_nf4.so"
LIB_PATH = os.path.join(HERE, LIB_NAME)

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC,-fvisibility=hidden", "-shared",
    "-Xptxas", "-v",
]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def build(verbose: bool = False, log_path: str | None = None) -> str:
    """Compile every CUDA source of the package into LIB_PATH; returns it."""
    srcs = sorted(glob.glob(os.path.join(HERE, "csrc", "*.cu")))
    cmd = [_nvcc(), *NVCC_FLAGS, "-o", LIB_PATH + ".tmp", *srcs]
    res = subprocess.run(cmd, capture_output=True, text=True)
    out = res.stdout + res.stderr
    if log_path:
        with open(log_path, "w") as f:
            f.write(" ".join(cmd) + "\n" + out)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + out)
    os.replace(LIB_PATH + ".tmp", LIB_PATH)
    if verbose:
        print(out)
    return LIB_PATH


if __name__ == "__main__":
    build(verbose="-v" in sys.argv)
    print(LIB_PATH)
