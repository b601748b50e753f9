"""Build ``libpaged_attn.so`` in-tree for sm_100a with nvcc.

    python -m paged_kv_cache_463_b200.build [--verbose]

The library links the CUDA runtime statically and resolves the one driver
entry point it needs (cuTensorMapEncodeTiled) at run time, so it loads on a
machine without a GPU (symbols can be inspected there; calls fail with
PA_ERR_CUDA).
"""

from __future__ import annotations

import argparse
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB_DIR = os.path.join(PKG, "lib")
LIB = os.path.join(LIB_DIR, "libpaged_attn.so")
SOURCES = ["paged_attn.cu", "block_manager.cpp"]
DEPS = ["paged_attn.cu", "block_manager.cpp", "decode.cuh", "prefix.cuh", "prefill.cuh", "umma.cuh", "cache_ops.cuh", "ptx.cuh"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
HEADERS = ["paged_attn.h", "block_manager.h"]


def nvcc() -> str:
    exe = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(exe):
        raise RuntimeError("nvcc not found")
    return exe


def command(out: str = LIB, extra: list[str] | None = None) -> list[str]:
    return ([nvcc()] + ARCH + ["-O3", "-lineinfo", "-std=c++17", "--shared", "-Xcompiler", "-fPIC,-fvisibility=hidden",
                              "-I", os.path.join(ROOT, "include"), "-o", out]
            + [os.path.join(CSRC, s) for s in SOURCES] + (extra or []))


def up_to_date(out: str = LIB) -> bool:
    if not os.path.exists(out):
        return False
    t = os.path.getmtime(out)
    deps = [os.path.join(CSRC, d) for d in DEPS] + [os.path.join(ROOT, "include", h) for h in HEADERS] + [__file__]
    return all(os.path.getmtime(d) <= t for d in deps)


def build(force: bool = False, verbose: bool = False, out: str = LIB, extra: list[str] | None = None) -> str:
    os.makedirs(os.path.dirname(out), exist_ok=True)
    if not force and extra is None and up_to_date(out):
        return out
    cmd = command(out, extra)
    if verbose:
        print(" ".join(cmd), flush=True)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError(f"nvcc failed ({r.returncode})")
    if verbose and (r.stdout or r.stderr):
        sys.stderr.write(r.stdout + r.stderr)
    return out


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--ptxas-info", action="store_true", help="print registers / spills / shared memory")
    a = ap.parse_args()
    extra = ["-Xptxas", "-v"] if a.ptxas_info else None
    print(build(force=a.force or a.ptxas_info, verbose=a.verbose or a.ptxas_info, extra=extra))
