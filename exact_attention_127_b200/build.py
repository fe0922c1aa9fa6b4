"""Build the CUDA library in-tree: exact_attention_127_b200/libattn127.so.

One translation unit, compiled for sm_100a only, cudart linked statically so
the library needs nothing beyond the driver at run time.
"""
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
SRC = os.path.join(PKG, "csrc", "attn_fwd_sm100.cu")
SOURCES = [SRC]
HDR = os.path.join(ROOT, "include", "attn_fwd.h")
LIB = os.path.join(PKG, "libattn127.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "-cudart", "static",
    "-Xptxas", "-v",
]


def nvcc_path() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def build(force: bool = False, verbose: bool = False) -> str:
    deps = SOURCES + [os.path.join(PKG, "csrc", f) for f in ("attn_standard.cuh", "attn_bwd.cuh", "attn_decode.cuh")]
    deps.append(HDR)
    newest = max(os.path.getmtime(f) for f in deps)
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= newest:
        return LIB
    tmp = LIB + ".tmp"
    cmd = [nvcc_path(), *NVCC_FLAGS, "-I", os.path.join(ROOT, "include"), *SOURCES, "-o", tmp]
    try:
        res = subprocess.run(cmd, capture_output=True, text=True, timeout=900)
    except subprocess.TimeoutExpired:
        raise RuntimeError("nvcc timed out after 900 s:\n" + " ".join(cmd))
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + " ".join(cmd) + "\n" + res.stdout + res.stderr)
    os.replace(tmp, LIB)
    if verbose:
        sys.stderr.write(res.stdout + res.stderr)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
