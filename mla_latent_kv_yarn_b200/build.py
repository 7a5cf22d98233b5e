"""Build libxmla.so in-tree with nvcc for sm_100a.

    python -m mla_latent_kv_yarn_b200.build        (or call build())

The library is written next to this file so that it travels with the source
tree; the CUDA runtime is linked statically.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libxmla.so")
SOURCES = ["rope_append.cu", "mla_decode.cu", "absorb_combine.cu", "xmla_api.cu", "kv_produce.cu",
           "head_gemm.cu", "mla_decode_q8.cu", "q8_append.cu", "prefill.cu"]
HEADERS = ["xmla_device.cuh", "yarn.cuh", "append.cuh", "decode_chain.h", "split_kv.h", "produce.cuh",
           "prefill.h",
           os.path.join("..", "..", "include", "xmla.h")]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "--expt-relaxed-constexpr",
]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, s) for s in SOURCES] + [os.path.join(CSRC, h) for h in HEADERS]
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not _stale():
        return LIB
    tmp = LIB + ".tmp"
    cmd = [_nvcc(), *NVCC_FLAGS, *[os.path.join(CSRC, s) for s in SOURCES], "-o", tmp]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
