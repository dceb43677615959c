"""Build the CUDA library in-tree: decode_attention_qk_b200/libqwen3_decode_attn.so.

nvcc compiles the kernels for sm_100a only (B200) and links a shared library
with a C ABI (include/qwen3_decode_attn.h). Run `python -m
decode_attention_qk_b200.build` or call build_library().
"""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIBRARY = os.path.join(PKG, "libqwen3_decode_attn.so")
SOURCES = [os.path.join(CSRC, f) for f in ("qda_decode_kernel.cu", "qda_decode_mma.cu", "qda_qkv_proj.cu", "qda_api.cu",
                                           "qda_noalloc.cu", "qda_host_stage.cu", "qda_prefill.cu")]
HEADERS = [os.path.join(CSRC, "qda_internal.h"), os.path.join(CSRC, "qda_device.cuh"), os.path.join(CSRC, "qda_tc.cuh"),
           os.path.join(CSRC, "qda_prefill.h"),
           os.path.join(INCLUDE, "qwen3_decode_attn.h")]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "-Xptxas", "-v",
]


def nvcc() -> str:
    home = os.environ.get("CUDA_HOME", "/usr/local/cuda")
    path = os.path.join(home, "bin", "nvcc")
    return path if os.path.exists(path) else "nvcc"


def needs_build() -> bool:
    if not os.path.exists(LIBRARY):
        return True
    t = os.path.getmtime(LIBRARY)
    return any(os.path.getmtime(f) > t for f in SOURCES + HEADERS)


def build_library(force: bool = False, verbose: bool = False) -> str:
    """Compile if a source is newer than the library; return the ptxas report."""
    if not force and not needs_build():
        return ""
    cmd = [nvcc(), *NVCC_FLAGS, "-I", INCLUDE, "-I", CSRC, "-o", LIBRARY, *SOURCES]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed ({' '.join(cmd)}):\n{res.stdout}\n{res.stderr}")
    report = res.stdout + res.stderr
    if verbose:
        print(report)
    return report


if __name__ == "__main__":
    print(build_library(force="--force" in sys.argv, verbose=True) or "up to date")
