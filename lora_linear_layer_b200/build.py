"""Build step: compile the CUDA library for sm_100a into ``_lib/``.

    python -m lora_linear_layer_b200.build [--force]

Two translation units: ``csrc/lora_api.cu`` (the entry points, with the
kernels included) and ``csrc/plan_api.cu`` (host-only launch-plan
introspection); the CUDA runtime is linked statically and the driver's tensor-map encoder is
looked up at run time, so the library loads on machines without a GPU.
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

_HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(_HERE, "csrc")
OUT = os.path.join(_HERE, "_lib", "liblora_b200.so")
HEADER = os.path.join(os.path.dirname(_HERE), "include", "lora.h")
TRANSLATION_UNITS = ("lora_api.cu", "plan_api.cu")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
]


def nvcc_path() -> str:
    p = shutil.which("nvcc")
    if p:
        return p
    cand = "/usr/local/cuda/bin/nvcc"
    if os.path.exists(cand):
        return cand
    raise RuntimeError("nvcc not found")


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh")) + [HEADER])


def build(force: bool = False, verbose: bool = True, extra_flags=None) -> str:
    """Compile if any source is newer than the library (or `force`)."""
    if not force and os.path.exists(OUT):
        newest = max(os.path.getmtime(s) for s in sources())
        if os.path.getmtime(OUT) >= newest and not extra_flags:
            return OUT
    os.makedirs(os.path.dirname(OUT), exist_ok=True)
    tmp = OUT + ".tmp"
    cmd = [nvcc_path()] + NVCC_FLAGS + list(extra_flags or []) + ["-o", tmp] + [os.path.join(CSRC, f) for f in TRANSLATION_UNITS]
    if verbose:
        print("[lora_b200 build]", " ".join(cmd), flush=True)
    subprocess.run(cmd, check=True, cwd=CSRC)
    os.replace(tmp, OUT)
    return OUT


if __name__ == "__main__":
    build(force="--force" in sys.argv)
