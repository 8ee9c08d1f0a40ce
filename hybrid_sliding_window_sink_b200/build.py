"""Builds libmimo_attn.so in this package directory with nvcc for sm_100a.

Usage: ``python -m hybrid_sliding_window_sink_b200.build`` (or call ``build()``).
The library links the CUDA runtime statically and reaches the driver's
tensor-map encoder through cudaGetDriverEntryPoint, so loading it needs no
GPU; running any entry point needs a B200.
"""

from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB_NAME = "libmimo_attn.so"
LIB_PATH = os.path.join(PKG, LIB_NAME)
SOURCES = ["mimo_attn.cu"]
HEADERS = ["ptx.cuh", "decode.cuh", "decode_warp.cuh", "decode_fp8.cuh", "decode_mq_tma.cuh", "decode_mq.cuh", "select.cuh", "prefill.cuh", "prefill_swa.cuh", "prefill_ga.cuh"]


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


#: Test builds of the same source, each a separate library next to the product one:
#:   shortwait  waits on work in progress give up after 1 ns (the 2 s exit-path drains stay),
#:              so the kernels' abort paths run; plus a hook that waits on a barrier nothing
#:              arrives on (mimo_attn_test_stuck_wait)
#:   debug      kernels record out-of-range lengths and indices in the device error word
VARIANTS = {
    "shortwait": ["-DMIMO_WAIT_LIMIT_NS=1ull", "-DMIMO_TEST_HOOKS"],
    "debug": ["-DMIMO_DEBUG"],
}


def variant_path(name: str) -> str:
    return os.path.join(PKG, f"libmimo_attn_{name}.so")


def _stale(path=LIB_PATH) -> bool:
    if not os.path.exists(path):
        return True
    t = os.path.getmtime(path)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS]
    deps.append(os.path.join(INCLUDE, "mimo_attn.h"))
    deps.append(os.path.abspath(__file__))
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False, variant: str | None = None) -> str:
    """Builds the product library, or with ``variant`` one of the test builds (VARIANTS)."""
    path = LIB_PATH if variant is None else variant_path(variant)
    if not force and not _stale(path):
        return path
    cmd = [
        nvcc_path(), "-std=c++17", "-O3", "-lineinfo",
        "-gencode", "arch=compute_100a,code=sm_100a",
        "-Xcompiler", "-fPIC,-O3", "-shared",
        "-I", INCLUDE, "-I", CSRC,
        "-o", path + ".tmp",
    ] + (VARIANTS[variant] if variant else []) + [os.path.join(CSRC, f) for f in SOURCES]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)
    os.replace(path + ".tmp", path)
    return path


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
    if "--variants" in sys.argv:
        for name in VARIANTS:
            print(build(force="--force" in sys.argv, variant=name))
