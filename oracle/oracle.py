"""Python face of the CPU oracle (bsq_oracle.c).

TEST INFRASTRUCTURE ONLY: imported by tests/, by ``__graft_entry__.smoke()``
and by the CPU-baseline leg of ``bench.py``.  The library in fp8_math_b200/
never imports this module, and this module imports nothing from it.

The C file is compiled on first use (gcc, ``-O2 -ffp-contract=off
-fno-fast-math``) into ``oracle/liboracle.so``; ``build()`` does the same
ahead of time.  Arrays are numpy; bf16 tensors travel as ``uint16`` bit
patterns.  Each wrapper names the C function whose header comment cites the
page and section it follows.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
import threading
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "bsq_oracle.c")
_SO = os.path.join(_HERE, "liboracle.so")
_CFLAGS = ["-std=c11", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared"]
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle into oracle/liboracle.so (if missing or stale)."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        tmp = _SO + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *_CFLAGS, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _SO)
    return _SO


_u8p = np.ctypeslib.ndpointer(np.uint8, flags="C_CONTIGUOUS")
_i8p = np.ctypeslib.ndpointer(np.int8, flags="C_CONTIGUOUS")
_u16p = np.ctypeslib.ndpointer(np.uint16, flags="C_CONTIGUOUS")
_i32p = np.ctypeslib.ndpointer(np.int32, flags="C_CONTIGUOUS")
_i64p = np.ctypeslib.ndpointer(np.int64, flags="C_CONTIGUOUS")
_f32p = np.ctypeslib.ndpointer(np.float32, flags="C_CONTIGUOUS")
_f64p = np.ctypeslib.ndpointer(np.float64, flags="C_CONTIGUOUS")
_u32p = np.ctypeslib.ndpointer(np.uint32, flags="C_CONTIGUOUS")
_i64 = C.c_int64


def lib():
    global _lib
    with _lock:
        if _lib is None:
            L = C.CDLL(build())
            sig = {
                "ora_bf16_to_f32": (C.c_float, [C.c_uint16]),
                "ora_f32_to_bf16": (C.c_uint16, [C.c_float]),
                "ora_e2m1_value": (C.c_float, [C.c_uint8]),
                "ora_e2m1_rne_sat": (C.c_uint8, [C.c_float]),
                "ora_e4m3_value": (C.c_float, [C.c_uint8]),
                "ora_e4m3_rne_sat": (C.c_uint8, [C.c_float]),
                "ora_e8m0_value": (C.c_float, [C.c_uint8]),
                "ora_e4m3_sr": (C.c_uint8, [C.c_float, C.c_uint16]),
                "ora_e2m1_sr": (C.c_uint8, [C.c_float, C.c_uint16]),
                "ora_philox4x32_10": (None, [_u32p, _u32p, _u32p]),
                "ora_sr_draw": (C.c_uint16, [C.c_uint64, C.c_uint32, C.c_uint64]),
                "ora_rht_sign_mask": (C.c_uint16, [C.c_uint64]),
                "ora_rht16": (None, [_f32p, C.c_uint16, _f32p]),
                "ora_rht_bf16": (C.c_int, [_u16p, _u16p, _i64, _i64, _i64, C.c_uint16]),
                "ora_amax": (C.c_float, [_u16p, _i64, _i64, _i64, C.c_int, C.c_uint16, C.c_void_p]),
                "ora_nvfp4_global_scale": (C.c_float, [C.c_float]),
                "ora_quant_nvfp4": (C.c_int, [_u16p, _i64, _i64, _i64, C.c_int, C.c_int, C.c_int,
                                              C.c_uint16, C.c_void_p, C.c_void_p, _f32p, _u8p, _u8p]),
                "ora_quant_nvfp4_sr": (C.c_int, [_u16p, _i64, _i64, _i64, C.c_int, C.c_int, C.c_uint16,
                                                 C.c_void_p, C.c_void_p, C.c_uint64, C.c_uint32, _f32p, _u8p,
                                                 _u8p]),
                "ora_quant_nvfp4_sr_rows": (C.c_int, [_u16p, _i64, _i64, _i64, C.c_int, C.c_int, C.c_uint16,
                                                      C.c_void_p, C.c_void_p, C.c_uint64, C.c_uint32, _i64,
                                                      _f32p, _u8p, _u8p]),
                "ora_quant_mxfp4": (C.c_int, [_u16p, _i64, _i64, _i64, C.c_int, C.c_uint64, C.c_uint32,
                                              _u8p, _u8p]),
                "ora_quant_mxfp4_rows": (C.c_int, [_u16p, _i64, _i64, _i64, C.c_int, C.c_uint64, C.c_uint32,
                                                   _i64, _u8p, _u8p]),
                "ora_rht_f32": (C.c_int, [_u16p, _f32p, _i64, _i64, C.c_uint16]),
                "ora_quant_mxfp8": (C.c_int, [_u16p, _i64, _i64, _i64, C.c_int, C.c_int,
                                              C.c_uint64, C.c_uint32, _u8p, _u8p]),
                "ora_quant_mxfp8_rows": (C.c_int, [_u16p, _i64, _i64, _i64, C.c_int, C.c_int,
                                                   C.c_uint64, C.c_uint32, _i64, _u8p, _u8p]),
                "ora_requant_transpose": (C.c_int, [_u8p, _u8p, _i64, _i64, C.c_int, C.c_uint64,
                                                    C.c_uint32, _u8p, _u8p]),
                "ora_requant_transpose_rows": (C.c_int, [_u8p, _u8p, _i64, _i64, C.c_int, C.c_uint64,
                                                         C.c_uint32, _i64, _i64, _u8p, _u8p]),
                "ora_requant_nvfp4_mxfp8_rows": (C.c_int, [_u8p, _u8p, C.c_float, _i64, _i64, C.c_int, C.c_uint64,
                                                           C.c_uint32, _i64, _i64, _u8p, _u8p]),
                "ora_quant_s2f6": (C.c_int, [_u16p, _i64, _i64, _i64, C.c_int, C.c_uint16, _i8p, _u8p]),
                "ora_combine_s2f6": (C.c_int, [_i8p, _u8p, _i64, _i32p, _i32p, _f32p, _i64, C.c_uint16, _u16p]),
                "ora_sf_swizzled_bytes": (_i64, [_i64, _i64]),
                "ora_sf_offset": (_i64, [_i64, _i64, _i64]),
                "ora_sf_swizzle": (None, [_u8p, _i64, _i64, _u8p]),
                "ora_sf_unswizzle": (None, [_u8p, _i64, _i64, _u8p]),
                "ora_dequant": (None, [C.c_int, _u8p, _u8p, C.c_float, _i64, _i64, _f64p]),
                "ora_gemm_f64": (None, [_f64p, _f64p, _i64, _i64, _i64, _f64p, _f64p]),
                "ora_gemm_points": (None, [C.c_int, _u8p, _u8p, C.c_float, _u8p, _u8p, C.c_float,
                                           _i64, _i64, _i64p, _i64p, _f64p, _f64p]),
            }
            for name, (res, args) in sig.items():
                f = getattr(L, name)
                f.restype = res
                f.argtypes = args
            _lib = L
    return _lib


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _ptr(a):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


# ---------------------------------------------------------------- threads
# Every oracle function below computes each output row on its own (the SR
# draw index is the absolute output position, the amax a maximum), so the
# rows can be split into bands and the bands run on separate threads (ctypes
# releases the GIL during the C call) with results identical to one thread.
def ncores() -> int:
    """Host cores this process may run on."""
    return len(os.sched_getaffinity(0))


def _bands(R, parts, align=1):
    units = -(-R // align)
    parts = max(1, min(parts, units))
    edges = [min(R, (units * i // parts) * align) for i in range(parts + 1)]
    edges[-1] = R
    return [(edges[i], edges[i + 1]) for i in range(parts) if edges[i] < edges[i + 1]]


def _run_bands(fn, R, threads, align=1):
    """fn(r0, r1) over bands of [0, R); returns the list of results in band order."""
    bands = _bands(R, max(1, threads) * 4 if threads > 1 else 1, align)
    if threads <= 1 or len(bands) <= 1:
        return [fn(r0, r1) for r0, r1 in bands]
    with ThreadPoolExecutor(threads) as ex:
        return list(ex.map(lambda b: fn(*b), bands))


# ---------------------------------------------------------------- formats
def bf16_to_f32(b):
    b = _c(b, np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


def f32_to_bf16(f):
    return np.array([lib().ora_f32_to_bf16(float(v)) for v in np.ravel(f)], np.uint16).reshape(np.shape(f))


def e2m1_value(code):
    return lib().ora_e2m1_value(int(code))


def e2m1_rne_sat(v):
    return lib().ora_e2m1_rne_sat(float(np.float32(v)))


def e4m3_value(code):
    return lib().ora_e4m3_value(int(code))


def e4m3_rne_sat(v):
    return lib().ora_e4m3_rne_sat(float(np.float32(v)))


def e8m0_value(code):
    return lib().ora_e8m0_value(int(code))


def e2m1_sr(v, r16):
    return lib().ora_e2m1_sr(float(v), int(r16))


def e4m3_sr(v, r16):
    return lib().ora_e4m3_sr(float(np.float32(v)), int(r16))


# ---------------------------------------------------------------- random
def philox4x32_10(ctr, key):
    out = np.zeros(4, np.uint32)
    lib().ora_philox4x32_10(_c(ctr, np.uint32), _c(key, np.uint32), out)
    return out


def sr_draw(seed, stream_id, idx):
    return lib().ora_sr_draw(int(seed), int(stream_id), int(idx))


def rht_sign_mask(seed):
    return lib().ora_rht_sign_mask(int(seed))


# ---------------------------------------------------------------- transforms
def rht16(x16, mask):
    y = np.zeros(16, np.float32)
    lib().ora_rht16(_c(x16, np.float32), int(mask), y)
    return y


def rht_bf16(x, mask):
    x = _c(x, np.uint16)
    M, K = x.shape
    y = np.zeros_like(x)
    if lib().ora_rht_bf16(x, y, M, K, K, int(mask)):
        raise ValueError("K must be a multiple of 16")
    return y


def rht_f32(x, mask):
    """The fused RHT's binary32 output y = 1/4 H16 diag(s) x for every group of
    16 along K (ora_rht_f32)."""
    x = _c(x, np.uint16)
    M, K = x.shape
    y = np.zeros((M, K), np.float32)
    if lib().ora_rht_f32(x, y, M, K, int(mask)):
        raise ValueError("K must be a multiple of 16")
    return y


def amax(x, rht_mask=None, row_index=None, threads=1):
    x = _c(x, np.uint16)
    M, K = x.shape
    ri = None if row_index is None else _c(row_index, np.int32)
    rows = M if ri is None else ri.shape[0]
    L = lib()

    def band(r0, r1):
        if ri is None:
            return L.ora_amax(x[r0:r1], r1 - r0, K, K, int(rht_mask is not None), int(rht_mask or 0), None)
        sub = ri[r0:r1]
        return L.ora_amax(x, r1 - r0, K, K, int(rht_mask is not None), int(rht_mask or 0), _ptr(sub))

    if rows == 0:
        return 0.0
    return max(_run_bands(band, rows, threads))


def nvfp4_global_scale(a):
    return lib().ora_nvfp4_global_scale(float(a))


def _nvfp4_common(x, block_2d, rht_mask, row_index, amax_in, threads, call):
    """Shared driver of quant_nvfp4 / quant_nvfp4_sr: one call on the whole
    tensor (threads == 1), or the tensor amax first and then bands of output
    rows (16-row aligned for 16x16 tiles) with that amax given."""
    x = _c(x, np.uint16)
    M, K = x.shape
    ri = None if row_index is None else _c(row_index, np.int32)
    R = M if ri is None else ri.shape[0]
    codes = np.zeros((R, K // 2), np.uint8)
    sf = np.zeros((R, K // 16), np.uint8)
    if threads <= 1 or R == 0:
        sg = np.zeros(1, np.float32)
        am = None if amax_in is None else np.array([amax_in], np.float32)
        if call(x, R, ri, am, 0, sg, codes, sf):
            raise ValueError("unsupported NVFP4 shape/options")
        return codes, sf, float(sg[0])
    if amax_in is None:
        amax_in = amax(x, rht_mask, ri, threads=threads)
    am = np.array([amax_in], np.float32)

    def band(r0, r1):
        sg = np.zeros(1, np.float32)
        xs, sub = (x[r0:r1], None) if ri is None else (x, ri[r0:r1])
        if call(xs, r1 - r0, sub, am, r0, sg, codes[r0:r1], sf[r0:r1]):
            raise ValueError("unsupported NVFP4 shape/options")
        return float(sg[0])

    sgs = _run_bands(band, R, threads, 16 if block_2d else 1)
    assert len(set(sgs)) == 1
    return codes, sf, sgs[0]


def quant_nvfp4(x, block_2d=False, four_over_six=False, rht_mask=None, row_index=None, amax_in=None, threads=1):
    """NVFP4 quantize (ora_quant_nvfp4).  Returns (codes [R,K/2] u8, sf [R,K/16] u8, s_g).
    threads > 1 splits the output rows into bands (identical results)."""
    K = np.shape(x)[1]
    L = lib()

    def call(xs, R, ri, am, row0, sg, codes, sf):
        return L.ora_quant_nvfp4(xs, R, K, K, int(block_2d), int(four_over_six), int(rht_mask is not None),
                                 int(rht_mask or 0), _ptr(ri), _ptr(am), sg, codes, sf)

    return _nvfp4_common(x, block_2d, rht_mask, row_index, amax_in, threads, call)


def quant_nvfp4_sr(x, block_2d=False, rht_mask=None, row_index=None, amax_in=None, seed=0, stream_id=0, threads=1):
    """NVFP4 quantize with stochastic rounding of the elements
    (ora_quant_nvfp4_sr_rows).  Returns (codes [R,K/2] u8, sf [R,K/16] u8, s_g)."""
    K = np.shape(x)[1]
    L = lib()

    def call(xs, R, ri, am, row0, sg, codes, sf):
        return L.ora_quant_nvfp4_sr_rows(xs, R, K, K, int(block_2d), int(rht_mask is not None), int(rht_mask or 0),
                                         _ptr(ri), _ptr(am), int(seed), int(stream_id), int(row0), sg, codes, sf)

    return _nvfp4_common(x, block_2d, rht_mask, row_index, amax_in, threads, call)


def quant_mxfp4(x, sr=False, seed=0, stream_id=0, threads=1):
    """MXFP4 quantize (ora_quant_mxfp4_rows), row-wise blocks of 32 along K.
    Returns (codes [M,K/2] u8, sf [M,K/32] u8)."""
    x = _c(x, np.uint16)
    M, K = x.shape
    codes = np.zeros((M, K // 2), np.uint8)
    sf = np.zeros((M, K // 32), np.uint8)
    L = lib()

    def band(r0, r1):
        if L.ora_quant_mxfp4_rows(x[r0:r1], r1 - r0, K, K, int(sr), int(seed), int(stream_id), int(r0),
                                  codes[r0:r1], sf[r0:r1]):
            raise ValueError("unsupported MXFP4 shape")

    _run_bands(band, M, threads)
    return codes, sf


def quant_mxfp8(x, colwise=False, sr=False, seed=0, stream_id=0, out_row0=0, threads=1):
    """MXFP8 quantize (ora_quant_mxfp8_rows).  Returns (codes, sf) in the output
    orientation.  out_row0: index of the first output row within the full
    output tensor (SR draw indices), for computing a band of rows alone.
    threads > 1 splits the output rows into bands (identical results)."""
    x = _c(x, np.uint16)
    M, K = x.shape
    R, Cc = (K, M) if colwise else (M, K)
    codes = np.zeros((R, Cc), np.uint8)
    sf = np.zeros((R, Cc // 32), np.uint8)
    L = lib()

    def band(r0, r1):
        # output rows r0..r1: input rows (row-wise) or input columns (column-wise)
        xs = x[r0:r1] if not colwise else np.ascontiguousarray(x[:, r0:r1])
        m, k = (r1 - r0, K) if not colwise else (M, r1 - r0)
        if L.ora_quant_mxfp8_rows(xs, m, k, k, int(colwise), int(sr), int(seed), int(stream_id), int(out_row0 + r0),
                                  codes[r0:r1], sf[r0:r1]):
            raise ValueError("unsupported MXFP8 shape")

    if threads <= 1:
        band(0, R)
    else:
        _run_bands(band, R, threads)
    return codes, sf


def requant_transpose(codes, sf, sr=True, seed=0, stream_id=1, threads=1):
    codes = _c(codes, np.uint8)
    sf = _c(sf, np.uint8)
    M, K = codes.shape
    cc = np.zeros((K, M), np.uint8)
    sc = np.zeros((K, M // 32), np.uint8)
    L = lib()

    def band(k0, k1):
        if L.ora_requant_transpose_rows(codes, sf, M, K, int(sr), int(seed), int(stream_id), k0, k1, cc, sc):
            raise ValueError("unsupported requant shape")

    _run_bands(band, K, threads)
    return cc, sc


def requant_nvfp4_mxfp8(codes, sf, s_g, sr=True, seed=0, stream_id=1, threads=1):
    """NVFP4 [R, C] (codes [R, C/2], canonical sf [R, C/16], s_g) ->
    dequantize (binary32), transpose, MXFP8 (ora_requant_nvfp4_mxfp8_rows).
    Returns (codes [C, R] u8, sf [C, R/32] u8)."""
    codes = _c(codes, np.uint8)
    sf = _c(sf, np.uint8)
    R, C = codes.shape[0], codes.shape[1] * 2
    cc = np.zeros((C, R), np.uint8)
    sc = np.zeros((C, R // 32), np.uint8)
    L = lib()

    def band(c0, c1):
        if L.ora_requant_nvfp4_mxfp8_rows(codes, sf, float(s_g), R, C, int(sr), int(seed), int(stream_id), c0, c1,
                                          cc, sc):
            raise ValueError("unsupported NVFP4 -> MXFP8 shape")

    _run_bands(band, C, threads)
    return cc, sc


def quant_s2f6(x, rht_mask=None, threads=1):
    """RHT (optional) + block-scaled S2F6 (ora_quant_s2f6).  Returns (codes
    [M, K] int8, sf [M, K/32] E8M0 codes)."""
    x = _c(x, np.uint16)
    M, K = x.shape
    codes = np.zeros((M, K), np.int8)
    sf = np.zeros((M, K // 32), np.uint8)
    L = lib()

    def band(r0, r1):
        if L.ora_quant_s2f6(x[r0:r1], r1 - r0, K, K, int(rht_mask is not None), int(rht_mask or 0), codes[r0:r1],
                            sf[r0:r1]):
            raise ValueError("K must be a multiple of 32")

    _run_bands(band, M, threads)
    return codes, sf


def combine_s2f6(codes, sf, token_offsets, rows, weights, mask, threads=1):
    """Weighted sum per token of S2F6 rows, inverse RHT, bf16 (ora_combine_s2f6).
    Returns bf16 bits [T, K]; threads > 1 splits the tokens into bands."""
    codes = _c(codes, np.int8)
    sf = _c(sf, np.uint8)
    off = _c(token_offsets, np.int32)
    rows = _c(rows, np.int32)
    weights = _c(weights, np.float32)
    T, K = off.shape[0] - 1, codes.shape[1]
    out = np.zeros((T, K), np.uint16)
    L = lib()

    def band(t0, t1):
        if L.ora_combine_s2f6(codes, sf, K, np.ascontiguousarray(off[t0:t1 + 1]), rows, weights, t1 - t0, int(mask),
                              out[t0:t1]):
            raise ValueError("K must be a multiple of 32")

    _run_bands(band, T, threads)
    return out


# ---------------------------------------------------------------- layout
def sf_swizzled_bytes(rows, nblk):
    return lib().ora_sf_swizzled_bytes(rows, nblk)


def sf_offset(r, b, nblk):
    return lib().ora_sf_offset(r, b, nblk)


def sf_swizzle(sf):
    sf = _c(sf, np.uint8)
    rows, nblk = sf.shape
    out = np.zeros(sf_swizzled_bytes(rows, nblk), np.uint8)
    lib().ora_sf_swizzle(sf, rows, nblk, out)
    return out


def sf_unswizzle(buf, rows, nblk):
    out = np.zeros((rows, nblk), np.uint8)
    lib().ora_sf_unswizzle(_c(buf, np.uint8), rows, nblk, out)
    return out


# ---------------------------------------------------------------- GEMM
NVFP4, MXFP8, MXFP4 = 0, 1, 2


def dequant(fmt, codes, sf, s_g=1.0, threads=1):
    codes = _c(codes, np.uint8)
    sf = _c(sf, np.uint8)
    R = codes.shape[0]
    K = codes.shape[1] * (1 if fmt == MXFP8 else 2)
    out = np.zeros((R, K), np.float64)
    L = lib()

    def band(r0, r1):
        L.ora_dequant(int(fmt), codes[r0:r1], sf[r0:r1], float(s_g), r1 - r0, K, out[r0:r1])

    _run_bands(band, R, threads)
    return out


def gemm_f64_blas(A, B):
    """C = A B^T in binary64 and sum_k |A[m,k]| |B[n,k]|, each as one call of
    the BLAS matrix product (a library primitive; it uses every core).  The
    same definition as ora_gemm_f64, summed in the library's order; the sum
    of magnitudes only scales the tolerance, so it is formed in binary32
    (relative error below 1e-5 at these lengths)."""
    A = _c(A, np.float64)
    B = _c(B, np.float64)
    Ra = np.abs(A).astype(np.float32) @ np.abs(B).astype(np.float32).T
    return A @ B.T, Ra.astype(np.float64)


def gemm_f64(A, B):
    """C = A B^T and sum |A||B| in binary64 (ora_gemm_f64)."""
    A = _c(A, np.float64)
    B = _c(B, np.float64)
    M, K = A.shape
    N = B.shape[0]
    Cm = np.zeros((M, N), np.float64)
    Ra = np.zeros((M, N), np.float64)
    lib().ora_gemm_f64(A, B, M, N, K, Cm, Ra)
    return Cm, Ra


def gemm_points(fmt, qa, qb, K, pm, pn):
    """C and sum|.| at points (pm[i], pn[i]); qa/qb = (codes, sf, s_g)."""
    ca, sa, ga = qa
    cb, sb, gb = qb
    pm = _c(pm, np.int64)
    pn = _c(pn, np.int64)
    Cm = np.zeros(pm.shape[0], np.float64)
    Ra = np.zeros(pm.shape[0], np.float64)
    lib().ora_gemm_points(int(fmt), _c(ca, np.uint8), _c(sa, np.uint8), float(ga),
                          _c(cb, np.uint8), _c(sb, np.uint8), float(gb), int(K),
                          pm.shape[0], pm, pn, Cm, Ra)
    return Cm, Ra
