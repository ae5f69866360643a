"""Build the in-tree shared library ``libattn_b200.so`` (sm_100a only)."""
from __future__ import annotations

import os
import shutil
import subprocess

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG_DIR)
CSRC = os.path.join(PKG_DIR, "csrc")
LIB_PATH = os.path.join(PKG_DIR, "libattn_b200.so")
SOURCES = [os.path.join(CSRC, f) for f in ("attn_fwd.cu", "attn_bwd.cu", "attn_decode.cu", "attn_merge.cu",
                                                "attn_fwd_host.cu")]
HEADERS = [os.path.join(CSRC, f) for f in ("attn_fwd_kernel.cuh", "attn_bwd_kernel.cuh", "attn_decode_kernel.cuh", "sm100_ptx.cuh")] + [
    os.path.join(ROOT, "include", "attn.h")]


def nvcc_path() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def nvcc_command(out: str = LIB_PATH, extra=()) -> list:
    return [nvcc_path(), "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3", "-std=c++17",
            "-Xcompiler", "-fPIC", "-shared", "-I" + os.path.join(ROOT, "include"), *extra,
            "-o", out, *SOURCES]


def needs_build(out: str = LIB_PATH) -> bool:
    if not os.path.exists(out):
        return True
    t = os.path.getmtime(out)
    return any(os.path.getmtime(s) > t for s in SOURCES + HEADERS)


def build(force: bool = False, verbose: bool = False) -> str:
    if force or needs_build():
        tmp = LIB_PATH + ".tmp"
        cmd = nvcc_command(tmp, ("-Xptxas", "-v") if verbose else ())
        res = subprocess.run(cmd, capture_output=True, text=True)
        if res.returncode != 0:
            raise RuntimeError("nvcc failed:\n" + res.stdout + res.stderr)
        if verbose:
            print(res.stdout + res.stderr)
        os.replace(tmp, LIB_PATH)
    return LIB_PATH


if __name__ == "__main__":
    import sys
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
