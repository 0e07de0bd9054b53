"""ctypes binding of libbsq (include/bsq.h) -- argument marshalling only.

Every function has the name of its C entry point and takes torch tensors
(device tensors for the tensor arguments) or plain integers; it passes their
data pointers, sizes and the current CUDA stream to the library and raises
``BsqError`` on a nonzero status.  All computation happens in the library's
kernels.  The library is loaded from ``fp8_math_b200/libbsq.so``; if it is
missing the first call raises (build it with ``python -m fp8_math_b200.build``
or ``__graft_entry__.build()``).
"""
from __future__ import annotations

import ctypes as C
import os
import threading

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libbsq.so")

BSQ_OK, BSQ_ERR_INVALID, BSQ_ERR_ALIGN, BSQ_ERR_UNSUPPORTED, BSQ_ERR_CUDA, BSQ_ERR_TIMEOUT = range(6)
BSQ_RNE, BSQ_SR = 0, 1
BSQ_NVFP4, BSQ_MXFP8, BSQ_MXFP4 = 0, 1, 2
BSQ_OUT_F32, BSQ_OUT_BF16 = 0, 1
(BSQ_KNOB_FUSED_QUANT, BSQ_KNOB_GEMM_PAIR, BSQ_KNOB_GEMM_BN, BSQ_KNOB_STREAM_QUANT, BSQ_KNOB_GEMM_SPLITK,
 BSQ_KNOB_LAUNCH_OVERLAP) = 0, 1, 2, 3, 4, 5

_lock = threading.Lock()
_lib = None

_vp = C.c_void_p
_i64 = C.c_int64
_SIGS = {
    "bsq_status_str": (C.c_char_p, [C.c_int]),
    "bsq_sf_bytes": (C.c_size_t, [_i64, _i64]),
    "bsq_rht_sign_mask": (C.c_uint16, [C.c_uint64]),
    "bsq_amax": (C.c_int, [_vp, _i64, _i64, _i64, C.c_int, C.c_uint16, _vp, _vp, _vp]),
    "bsq_global_scale_noalloc": (C.c_int, [_vp, _i64, _i64, _i64, C.c_int, C.c_uint16, _vp, _vp]),
    "bsq_quant_nvfp4": (C.c_int, [_vp, _i64, _i64, _i64, C.c_int, C.c_int, C.c_int, C.c_uint16, _vp,
                                  C.c_int, _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "bsq_quant_mxfp8": (C.c_int, [_vp, _i64, _i64, _i64, C.c_int, C.c_int, C.c_uint64, C.c_uint32,
                                  _vp, _vp, _vp]),
    "bsq_quant_nvfp4_sr": (C.c_int, [_vp, _i64, _i64, _i64, C.c_int, C.c_int, C.c_uint16, _vp, _vp, _vp,
                                     C.c_uint64, C.c_uint32, _vp, _vp, _vp]),
    "bsq_quant_mxfp4": (C.c_int, [_vp, _i64, _i64, _i64, C.c_int, C.c_uint64, C.c_uint32, _vp, _vp, _vp]),
    "bsq_quant_mxfp8_rowcol": (C.c_int, [_vp, _i64, _i64, _i64, C.c_int, C.c_uint64, C.c_uint32, C.c_uint32,
                                         _vp, _vp, _vp, _vp, _vp]),
    "bsq_requant_nvfp4_mxfp8": (C.c_int, [_vp, _vp, _vp, _i64, _i64, C.c_int, C.c_uint64, C.c_uint32, _vp, _vp,
                                          _vp]),
    "bsq_rht": (C.c_int, [_vp, _vp, _i64, _i64, _i64, _i64, C.c_uint16, _vp]),
    "bsq_requant_transpose": (C.c_int, [_vp, _vp, _i64, _i64, C.c_int, C.c_uint64, C.c_uint32, _vp, _vp, _vp]),
    "bsq_gemm_blockscaled": (C.c_int, [C.c_int, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp, _i64,
                                       C.c_int, _vp]),
    "bsq_grouped_gemm": (C.c_int, [C.c_int, C.c_int, _vp, _vp, _i64, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64,
                                   _vp, _i64, C.c_int, _vp]),
    "bsq_grouped_gemm_nvfp4_out": (C.c_int, [C.c_int, C.c_int, _vp, _vp, _i64, _vp, _vp, _vp, _vp, _vp, _vp, _i64,
                                             _i64, _vp, C.c_int, _vp, _vp, _vp, _vp, _i64, _vp]),
    "bsq_quant_s2f6": (C.c_int, [_vp, _i64, _i64, _i64, C.c_int, C.c_uint16, _vp, _vp, _vp]),
    "bsq_combine_s2f6": (C.c_int, [_vp, _vp, _i64, _vp, _vp, _vp, _i64, C.c_uint16, _vp, _i64, _vp]),
    "bsq_gather_rows": (C.c_int, [_vp, _i64, _vp, _i64, _vp, _vp]),
    "bsq_sf_to_rows": (C.c_int, [_vp, _i64, _i64, _vp, _vp]),
    "bsq_sf_from_rows": (C.c_int, [_vp, _i64, _i64, C.c_int, _vp, _vp, _vp, _vp]),
    "bsq_quant_nvfp4_gather_workspace": (C.c_size_t, [_i64, _i64]),
    "bsq_quant_nvfp4_gather": (C.c_int, [_vp, _i64, _i64, _i64, _vp, _i64, C.c_int, C.c_int, C.c_uint16, C.c_int,
                                         _vp, _vp, _vp, _vp, _vp, _vp, _vp, C.c_size_t, _vp]),
    "bsq_check": (C.c_int, [_vp]),
    "bsq_debug_timeout_probe": (C.c_int, [C.c_uint64, _vp]),
    "bsq_debug_kernel_choice": (C.c_int, [C.c_int, C.c_int]),
}


class BsqError(RuntimeError):
    def __init__(self, fn, status):
        super().__init__(f"{fn}: status {status} ({status_str(status)})")
        self.status = status


def lib():
    """Load libbsq.so (once).  Raises if it has not been built."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(f"libbsq.so not built at {LIB_PATH}; run python -m fp8_math_b200.build")
            L = C.CDLL(LIB_PATH)
            for name, (res, args) in _SIGS.items():
                f = getattr(L, name)
                f.restype = res
                f.argtypes = args
            _lib = L
    return _lib


def _p(t):
    """Pointer of a tensor (or None / int)."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is not None:
        return stream if isinstance(stream, int) else stream.cuda_stream
    import torch
    return torch.cuda.current_stream().cuda_stream


def _check(fn, st):
    if st != BSQ_OK:
        raise BsqError(fn, st)
    return st


def status_str(status: int) -> str:
    return lib().bsq_status_str(status).decode()


def bsq_sf_bytes(rows: int, nblocks: int) -> int:
    return int(lib().bsq_sf_bytes(rows, nblocks))


def bsq_rht_sign_mask(seed: int) -> int:
    return int(lib().bsq_rht_sign_mask(seed))


def bsq_amax(x, M, K, ldx, rht_enable, rht_sign_mask, row_index, amax_out, stream=None):
    return _check("bsq_amax", lib().bsq_amax(_p(x), M, K, ldx, int(rht_enable), rht_sign_mask, _p(row_index),
                                             _p(amax_out), _stream(stream)))


def bsq_global_scale_noalloc(x, M, K, ldx, rht_enable, rht_sign_mask, gs_out, stream=None):
    return _check("bsq_global_scale_noalloc", lib().bsq_global_scale_noalloc(
        _p(x), M, K, ldx, int(rht_enable), rht_sign_mask, _p(gs_out), _stream(stream)))


def bsq_quant_nvfp4(x, M, K, ldx, block_2d, four_over_six, rht_enable, rht_sign_mask, row_index, G, row_offsets,
                    sf_row_offsets, amax_in, global_scale_out, codes, sf, stream=None):
    return _check("bsq_quant_nvfp4", lib().bsq_quant_nvfp4(
        _p(x), M, K, ldx, int(block_2d), int(four_over_six), int(rht_enable), rht_sign_mask, _p(row_index), G,
        _p(row_offsets), _p(sf_row_offsets), _p(amax_in), _p(global_scale_out), _p(codes), _p(sf), _stream(stream)))


def bsq_quant_mxfp8(x, M, K, ldx, colwise, rounding, seed, stream_id, codes, sf, stream=None):
    return _check("bsq_quant_mxfp8", lib().bsq_quant_mxfp8(_p(x), M, K, ldx, int(colwise), rounding, seed,
                                                           stream_id, _p(codes), _p(sf), _stream(stream)))


def bsq_quant_nvfp4_sr(x, M, K, ldx, block_2d, rht_enable, rht_sign_mask, row_index, amax_in, global_scale, seed,
                       stream_id, codes, sf, stream=None):
    return _check("bsq_quant_nvfp4_sr",
                  lib().bsq_quant_nvfp4_sr(_p(x), M, K, ldx, int(block_2d), int(rht_enable), rht_sign_mask,
                                           _p(row_index), _p(amax_in), _p(global_scale), seed, stream_id, _p(codes),
                                           _p(sf), _stream(stream)))


def bsq_quant_mxfp4(x, M, K, ldx, rounding, seed, stream_id, codes, sf, stream=None):
    return _check("bsq_quant_mxfp4", lib().bsq_quant_mxfp4(_p(x), M, K, ldx, rounding, seed, stream_id, _p(codes),
                                                           _p(sf), _stream(stream)))


def bsq_rht(x, y, M, K, ldx, ldy, rht_sign_mask, stream=None):
    return _check("bsq_rht", lib().bsq_rht(_p(x), _p(y), M, K, ldx, ldy, rht_sign_mask, _stream(stream)))


def bsq_requant_transpose(codes_row, sf_row, M, K, rounding, seed, stream_id, codes_col, sf_col, stream=None):
    return _check("bsq_requant_transpose", lib().bsq_requant_transpose(
        _p(codes_row), _p(sf_row), M, K, rounding, seed, stream_id, _p(codes_col), _p(sf_col), _stream(stream)))


def bsq_gemm_blockscaled(fmt, A, sfA, gsA, B, sfB, gsB, M, N, K, C_out, ldc, out_type, stream=None):
    return _check("bsq_gemm_blockscaled", lib().bsq_gemm_blockscaled(
        fmt, _p(A), _p(sfA), _p(gsA), _p(B), _p(sfB), _p(gsB), M, N, K, _p(C_out), ldc, out_type, _stream(stream)))


def bsq_grouped_gemm(fmt, G, row_offsets, sf_row_offsets, M_total, A, sfA, gsA, B, sfB, gsB, N, K, C_out, ldc,
                     out_type, stream=None):
    return _check("bsq_grouped_gemm", lib().bsq_grouped_gemm(
        fmt, G, _p(row_offsets), _p(sf_row_offsets), M_total, _p(A), _p(sfA), _p(gsA), _p(B), _p(sfB), _p(gsB), N,
        K, _p(C_out), ldc, out_type, _stream(stream)))


def bsq_check(stream=None):
    """Synchronize the stream and return the device status (no raise)."""
    return int(lib().bsq_check(_stream(stream)))


def bsq_debug_timeout_probe(timeout_ns, stream=None):
    return _check("bsq_debug_timeout_probe", lib().bsq_debug_timeout_probe(timeout_ns, _stream(stream)))


def bsq_debug_kernel_choice(knob, value):
    return _check("bsq_debug_kernel_choice", lib().bsq_debug_kernel_choice(knob, value))


def bsq_quant_mxfp8_rowcol(x, M, K, ldx, rounding, seed, stream_id_row, stream_id_col, codes_row, sf_row, codes_col,
                           sf_col, stream=None):
    return _check("bsq_quant_mxfp8_rowcol", lib().bsq_quant_mxfp8_rowcol(
        _p(x), M, K, ldx, rounding, seed, stream_id_row, stream_id_col, _p(codes_row), _p(sf_row), _p(codes_col),
        _p(sf_col), _stream(stream)))


def bsq_requant_nvfp4_mxfp8(codes, sf, gs, R, C, rounding, seed, stream_id, codes_col, sf_col, stream=None):
    return _check("bsq_requant_nvfp4_mxfp8", lib().bsq_requant_nvfp4_mxfp8(
        _p(codes), _p(sf), _p(gs), R, C, rounding, seed, stream_id, _p(codes_col), _p(sf_col), _stream(stream)))


def bsq_grouped_gemm_nvfp4_out(fmt, G, row_offsets, sf_row_offsets, M_total, A, sfA, gsA, B, sfB, gsB, N, K, out_gs,
                               four_over_six, out_codes, out_sf, out_amax, C_out, ldc, stream=None):
    return _check("bsq_grouped_gemm_nvfp4_out", lib().bsq_grouped_gemm_nvfp4_out(
        fmt, G, _p(row_offsets), _p(sf_row_offsets), M_total, _p(A), _p(sfA), _p(gsA), _p(B), _p(sfB), _p(gsB), N, K,
        _p(out_gs), int(four_over_six), _p(out_codes), _p(out_sf), _p(out_amax), _p(C_out), ldc, _stream(stream)))


def bsq_quant_s2f6(x, M, K, ldx, rht_enable, rht_sign_mask, codes, sf, stream=None):
    return _check("bsq_quant_s2f6", lib().bsq_quant_s2f6(_p(x), M, K, ldx, int(rht_enable), rht_sign_mask, _p(codes),
                                                         _p(sf), _stream(stream)))


def bsq_combine_s2f6(codes, sf, K, token_offsets, rows, weights, T, rht_sign_mask, out, ldo, stream=None):
    return _check("bsq_combine_s2f6", lib().bsq_combine_s2f6(_p(codes), _p(sf), K, _p(token_offsets), _p(rows),
                                                             _p(weights), T, rht_sign_mask, _p(out), ldo,
                                                             _stream(stream)))


def bsq_gather_rows(src, row_bytes, index, R, dst, stream=None):
    return _check("bsq_gather_rows", lib().bsq_gather_rows(_p(src), row_bytes, _p(index), R, _p(dst),
                                                           _stream(stream)))


def bsq_sf_to_rows(sf, rows, nblk, out, stream=None):
    return _check("bsq_sf_to_rows", lib().bsq_sf_to_rows(_p(sf), rows, nblk, _p(out), _stream(stream)))


def bsq_sf_from_rows(rows_in, rows, nblk, G, row_offsets, sf_row_offsets, sf, stream=None):
    return _check("bsq_sf_from_rows", lib().bsq_sf_from_rows(_p(rows_in), rows, nblk, G, _p(row_offsets),
                                                             _p(sf_row_offsets), _p(sf), _stream(stream)))


def bsq_quant_nvfp4_gather_workspace(T, K):
    return int(lib().bsq_quant_nvfp4_gather_workspace(T, K))


def bsq_quant_nvfp4_gather(x, T, K, ldx, row_index, M, four_over_six, rht_enable, rht_sign_mask, G, row_offsets,
                           sf_row_offsets, amax_in, global_scale, codes, sf, workspace, workspace_bytes, stream=None):
    return _check("bsq_quant_nvfp4_gather", lib().bsq_quant_nvfp4_gather(
        _p(x), T, K, ldx, _p(row_index), M, int(four_over_six), int(rht_enable), rht_sign_mask, G, _p(row_offsets),
        _p(sf_row_offsets), _p(amax_in), _p(global_scale), _p(codes), _p(sf), _p(workspace), workspace_bytes,
        _stream(stream)))
