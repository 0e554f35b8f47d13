"""Builds the four C-ABI libraries in-tree for sm_100a with nvcc.

    python -m sparse_moe_layer_sum_b200.build [--verbose]

Each library is one translation unit linked against the static CUDA
runtime, so the .so files depend only on the driver.  Outputs go to
sparse_moe_layer_sum_b200/lib/.
"""
from __future__ import annotations

import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIBDIR = os.path.join(PKG, "lib")
INCLUDE = os.path.join(ROOT, "include")

LIBRARIES = {
    "moe_router": "router.cu",
    "moe_dispatch": "dispatch.cu",
    "moe_experts": "experts.cu",
    "moe_combine": "combine.cu",
}

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-Xcompiler", "-fPIC,-fvisibility=hidden",
    "-shared",
]


def nvcc() -> str:
    home = os.environ.get("CUDA_HOME", "/usr/local/cuda")
    path = os.path.join(home, "bin", "nvcc")
    return path if os.path.exists(path) else "nvcc"


def _sources_mtime(src: str) -> float:
    files = [os.path.join(CSRC, src)] + [os.path.join(CSRC, f) for f in os.listdir(CSRC)
                                         if f.endswith(".cuh")]
    files += [os.path.join(INCLUDE, f) for f in os.listdir(INCLUDE)]
    return max(os.path.getmtime(f) for f in files)


def build_one(name: str, src: str, verbose: bool = False, force: bool = False) -> str:
    out = os.path.join(LIBDIR, f"lib{name}.so")
    if not force and os.path.exists(out) and os.path.getmtime(out) >= _sources_mtime(src):
        return out
    cmd = [nvcc(), *NVCC_FLAGS, "-I", INCLUDE, "-I", CSRC, "-o", out, os.path.join(CSRC, src)]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed for {name}:\n{res.stdout}\n{res.stderr}")
    if verbose:
        sys.stderr.write(res.stderr)
    return out


def build_all(verbose: bool = False, force: bool = False) -> list[str]:
    os.makedirs(LIBDIR, exist_ok=True)
    with ThreadPoolExecutor(max_workers=4) as ex:
        futs = [ex.submit(build_one, n, s, verbose, force) for n, s in LIBRARIES.items()]
        return [f.result() for f in futs]


if __name__ == "__main__":
    for p in build_all(verbose="--verbose" in sys.argv, force="--force" in sys.argv):
        print(p)
