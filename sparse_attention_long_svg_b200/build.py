"""Builds libsvg.so (the C-ABI CUDA library) in-tree for sm_100a with nvcc."""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "csrc", "svg.cu")
OUT = os.path.join(HERE, "libsvg.so")
NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
]


def nvcc_path() -> str:
    p = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(p):
        raise RuntimeError("nvcc not found")
    return p


def sources():
    csrc = os.path.join(HERE, "csrc")
    return sorted(os.path.join(csrc, f) for f in os.listdir(csrc) if f.endswith((".cu", ".cuh")))


# The source files each profiled kernel is compiled from (its own header and
# the shared primitives); a profile's counters stay valid while these match.
KERNEL_SOURCES = {
    "kmeans_assign_tc_kernel": ("common.cuh", "kmeans_tc.cuh"),
    "sparse_attn_kernel": ("common.cuh", "attn.cuh"),
    "sparse_attn_kernel_fp8": ("common.cuh", "attn.cuh"),
}


def source_hash(kernel: str | None = None) -> str:
    """Hash of the CUDA sources and the ABI header (a whole build), or of the
    files one kernel in KERNEL_SOURCES is compiled from."""
    import hashlib
    h = hashlib.sha256()
    if kernel is None:
        paths = sources() + [os.path.join(os.path.dirname(HERE), "include", "svg.h")]
    else:
        paths = [os.path.join(HERE, "csrc", f) for f in KERNEL_SOURCES[kernel]]
    for path in paths:
        with open(path, "rb") as f:
            h.update(os.path.basename(path).encode())
            h.update(f.read())
    return h.hexdigest()[:16]


def up_to_date() -> bool:
    if not os.path.exists(OUT):
        return False
    t = os.path.getmtime(OUT)
    deps = sources() + [os.path.join(os.path.dirname(HERE), "include", "svg.h")]
    return all(os.path.getmtime(d) <= t for d in deps)


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and up_to_date():
        return OUT
    cmd = [nvcc_path(), *NVCC_FLAGS, "-o", OUT + ".tmp", SRC]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)
    os.replace(OUT + ".tmp", OUT)
    return OUT


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="-v" in sys.argv)
    print(OUT)
