"""Build libtl_nvfp4.so in-tree: nvcc for sm_100a, static CUDA runtime, no torch at link time.

Usage: python -m nvfp4_weight_gemm_b200.build [--force] [--debug]
--debug lowers the device wait limit (TL_WAIT_LIMIT) so the bounded-wait paths can be
exercised quickly; it is never the default.
"""

from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libtl_nvfp4.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
]


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh")) +
                  glob.glob(os.path.join(INCLUDE, "*.h")))


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    return "nvcc"


def build(force: bool = False, debug: bool = False, out: str = LIB) -> str:
    srcs = _sources()
    newest = max(os.path.getmtime(s) for s in srcs)
    if not force and not debug and os.path.exists(out) and os.path.getmtime(out) >= newest:
        return out
    tmp = out + f".tmp{os.getpid()}"
    cmd = [nvcc()] + NVCC_FLAGS + ["-I", INCLUDE, "-o", tmp, os.path.join(CSRC, "tl_nvfp4_api.cu")]
    if debug:
        cmd.insert(1, "-DTL_WAIT_LIMIT=64u")
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, debug="--debug" in sys.argv))
