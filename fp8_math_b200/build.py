"""Build libbsq.so in-tree with nvcc for sm_100a.

    python -m fp8_math_b200.build [--force]

quant.cu is compiled with --fmad=false so that no multiply-add in the
quantization arithmetic is contracted (the codes must match an IEEE
operation sequence bit for bit); the GEMM and API objects use the default.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
OUT = os.path.join(HERE, "libbsq.so")
BUILD = os.path.join(HERE, "_build")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMMON = ARCH + ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
                 "--expt-relaxed-constexpr", "-I", os.path.join(HERE, "..", "include")]
SOURCES = {
    "quant.cu": ["--fmad=false"],
    "gemm.cu": [],
    "api.cu": [],
}
HEADERS = ["common.cuh", "devcache.h", "nvfp4.cuh", "quant.cuh", "gemm.cuh", "sm100.cuh"]


def _mtime(p):
    return os.path.getmtime(p) if os.path.exists(p) else 0.0


def build(force: bool = False, verbose: bool = False) -> str:
    os.makedirs(BUILD, exist_ok=True)
    hdr = max([_mtime(os.path.join(CSRC, h)) for h in HEADERS] +
              [_mtime(os.path.join(HERE, "..", "include", "bsq.h"))])
    objs = []
    procs = []
    for src, extra in SOURCES.items():
        s = os.path.join(CSRC, src)
        o = os.path.join(BUILD, src.replace(".cu", ".o"))
        objs.append(o)
        if force or _mtime(o) < max(_mtime(s), hdr):
            cmd = [NVCC, *COMMON, *extra, "-c", s, "-o", o]
            if verbose:
                cmd += ["-Xptxas", "-v"]
            procs.append((cmd, subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.STDOUT)))
    for cmd, p in procs:
        out, _ = p.communicate()
        if verbose or p.returncode:
            sys.stdout.write(out.decode(errors="replace"))
        if p.returncode:
            raise RuntimeError("nvcc failed: " + " ".join(cmd))
    if force or procs or not os.path.exists(OUT):
        tmp = OUT + f".tmp{os.getpid()}"
        subprocess.check_call([NVCC, *ARCH, "-shared", "-o", tmp, *objs, "-lcudart_static",
                               "-ldl", "-lrt", "-lpthread"])
        os.replace(tmp, OUT)
    return OUT


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="-v" in sys.argv)
    print(OUT)
