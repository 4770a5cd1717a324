"""Build libnvfp4ws.so (all CUDA sources, sm_100a) next to this file.

Run ``python -m nvfp4_weight_streaming_gemm_b200.build``. ``__graft_entry__.build()``
calls the same function. The library links the CUDA runtime statically, so it
loads beside torch's own runtime without a version clash.
"""

from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libnvfp4ws.so")
SOURCES = ["api.cu", "pack.cu", "gemv.cu", "verify.cu", "mma.cu", "mxf4.cu", "noalloc.cu", "fp8.cu", "fp8q.cu",
           "xshift.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    cuda = os.environ.get("CUDA_HOME", "/usr/local/cuda")
    path = os.path.join(cuda, "bin", "nvcc")
    return path if os.path.exists(path) else "nvcc"


def build(verbose: bool = False, extra: list[str] | None = None) -> str:
    """Compile every source into libnvfp4ws.so; returns its path. Raises on failure."""
    srcs = [os.path.join(CSRC, s) for s in SOURCES]
    deps = srcs + [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".h", ".cuh"))]
    deps.append(os.path.join(ROOT, "include", "nvfp4ws.h"))
    if os.path.exists(LIB) and all(os.path.getmtime(LIB) >= os.path.getmtime(d) for d in deps) and not extra:
        return LIB
    cmd = [nvcc(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "-shared", "-Xcompiler", "-fPIC",
           "-cudart", "static", "--expt-relaxed-constexpr", "-I", os.path.join(ROOT, "include"),
           *(extra or []), "-o", LIB + ".tmp", *srcs]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + r.stdout + r.stderr)
    if verbose and (r.stdout or r.stderr):
        print(r.stdout + r.stderr, file=sys.stderr)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(verbose=True, extra=sys.argv[1:] or None))
