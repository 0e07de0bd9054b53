"""fp8_math_b200 -- libbsq, block-scaled (NVFP4 / MXFP8) quantization and
block-scaled GEMM for NVIDIA B200 (sm_100a), behind a C ABI (include/bsq.h).

``fp8_math_b200.bsq`` is the thin ctypes binding (same names as the C entry
points); ``fp8_math_b200.workloads`` draws the seeded synthetic inputs.
The binding loads ``fp8_math_b200/libbsq.so`` lazily and raises if it is
missing: there is no CPU fallback.
"""
__all__ = ["bsq", "workloads"]
