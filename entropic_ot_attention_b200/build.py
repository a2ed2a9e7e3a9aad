"""Build libeot.so (the C-ABI library) in-tree with nvcc for sm_100a."""
from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(os.path.dirname(HERE), "include")
LIB = os.path.join(HERE, "libeot.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(INCLUDE, "*.h"))
    return any(os.path.getmtime(f) > t for f in deps)


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile every csrc/*.cu into entropic_ot_attention_b200/libeot.so (static cudart)."""
    if not force and not _stale():
        return LIB
    cmd = [NVCC, "-O3", "-std=c++17", *ARCH, "-lineinfo", "-Xcompiler", "-fPIC", "-shared",
           "-I", INCLUDE, "-o", LIB + ".tmp", *sources()]
    if os.environ.get("EOT_NVTX", "0") == "1":   # NVTX ranges around the passes (timeline profiling)
        cmd[1:1] = ["-DEOT_NVTX"]
    if os.environ.get("EOT_ITER_PREFETCH"):      # next tile's TMEM scores loaded during this tile (tuning)
        cmd[1:1] = [f"-DEOT_ITER_PREFETCH={int(os.environ['EOT_ITER_PREFETCH'])}"]
    if os.environ.get("EOT_ITER_FMA_PAIRS"):     # exponential pairs per 32 columns on the FMA pipe (tuning)
        cmd[1:1] = [f"-DEOT_ITER_FMA_PAIRS={int(os.environ['EOT_ITER_FMA_PAIRS'])}"]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
        raise RuntimeError("nvcc failed building libeot.so")
    if verbose:
        sys.stderr.write(res.stderr)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="-v" in sys.argv)
    print(LIB)
