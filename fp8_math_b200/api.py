"""Allocating convenience wrappers over the C ABI (torch tensors in and out).

Each helper allocates its output tensors on the input's device with
``torch.empty`` and calls one libbsq entry point through ``fp8_math_b200.bsq``;
all arithmetic runs in the library's CUDA kernels.  Shapes and layouts are
those of include/bsq.h.
"""
from __future__ import annotations

import torch

from . import bsq


def sf_bytes(rows: int, nblocks: int) -> int:
    return bsq.bsq_sf_bytes(rows, nblocks)


def _ld(x: torch.Tensor) -> int:
    assert x.dim() == 2 and x.stride(1) == 1, "row-major 2-D tensor expected"
    return x.stride(0)


def amax(x, rht_mask=None, row_index=None, out=None):
    M = x.shape[0] if row_index is None else row_index.shape[0]
    out = torch.empty(1, dtype=torch.float32, device=x.device) if out is None else out
    bsq.bsq_amax(x, M, x.shape[1], _ld(x), rht_mask is not None, rht_mask or 0, row_index, out)
    return out


def quant_nvfp4(x, block_2d=False, four_over_six=False, rht_mask=None, row_index=None, groups=None,
                amax_in=None, out=None):
    """Returns (codes [R, K/2] uint8, sf swizzled uint8, global_scale [1] fp32).
    groups = (row_offsets int32 [G+1], sf_row_offsets int32 [G+1], sf_rows)."""
    K = x.shape[1]
    R = x.shape[0] if row_index is None else row_index.shape[0]
    G, ro, so = 0, None, None
    sf_rows = R
    if groups is not None:
        ro, so, sf_rows = groups
        G = ro.shape[0] - 1
    if out is None:
        codes = torch.empty(R, K // 2, dtype=torch.uint8, device=x.device)
        sf = torch.zeros(sf_bytes(sf_rows, K // 16), dtype=torch.uint8, device=x.device)
        gs = torch.empty(1, dtype=torch.float32, device=x.device)
    else:
        codes, sf, gs = out
    bsq.bsq_quant_nvfp4(x, R, K, _ld(x), block_2d, four_over_six, rht_mask is not None, rht_mask or 0, row_index,
                        G, ro, so, amax_in, gs, codes, sf)
    return codes, sf, gs


def quant_mxfp8(x, colwise=False, sr=False, seed=0, stream_id=0, out=None):
    """Returns (codes, sf swizzled) in the output orientation ([M,K] or [K,M])."""
    M, K = x.shape
    R, Cc = (K, M) if colwise else (M, K)
    if out is None:
        codes = torch.empty(R, Cc, dtype=torch.uint8, device=x.device)
        sf = torch.zeros(sf_bytes(R, Cc // 32), dtype=torch.uint8, device=x.device)
    else:
        codes, sf = out
    bsq.bsq_quant_mxfp8(x, M, K, _ld(x), colwise, bsq.BSQ_SR if sr else bsq.BSQ_RNE, seed, stream_id, codes, sf)
    return codes, sf


def quant_mxfp8_rowcol(x, sr=False, seed=0, stream_id_row=0, stream_id_col=1, out=None):
    """Row-wise and column-wise MXFP8 in one pass.  Returns
    (codes_row [M,K], sf_row, codes_col [K,M], sf_col)."""
    M, K = x.shape
    if out is None:
        cr = torch.empty(M, K, dtype=torch.uint8, device=x.device)
        sr_ = torch.zeros(sf_bytes(M, K // 32), dtype=torch.uint8, device=x.device)
        cc = torch.empty(K, M, dtype=torch.uint8, device=x.device)
        sc = torch.zeros(sf_bytes(K, M // 32), dtype=torch.uint8, device=x.device)
    else:
        cr, sr_, cc, sc = out
    bsq.bsq_quant_mxfp8_rowcol(x, M, K, _ld(x), bsq.BSQ_SR if sr else bsq.BSQ_RNE, seed, stream_id_row,
                               stream_id_col, cr, sr_, cc, sc)
    return cr, sr_, cc, sc


def requant_nvfp4_mxfp8(codes, sf, gs, sr=True, seed=0, stream_id=1, out=None):
    """NVFP4 [R, C] (codes [R, C/2], swizzled sf, gs [1]) -> column-wise MXFP8.
    Returns (codes [C, R], sf swizzled)."""
    R, C = codes.shape[0], codes.shape[1] * 2
    if out is None:
        cc = torch.empty(C, R, dtype=torch.uint8, device=codes.device)
        sc = torch.zeros(sf_bytes(C, R // 32), dtype=torch.uint8, device=codes.device)
    else:
        cc, sc = out
    bsq.bsq_requant_nvfp4_mxfp8(codes, sf, gs, R, C, bsq.BSQ_SR if sr else bsq.BSQ_RNE, seed, stream_id, cc, sc)
    return cc, sc


def quant_nvfp4_sr(x, block_2d=False, rht_mask=None, row_index=None, amax_in=None, seed=0, stream_id=0, out=None):
    """NVFP4 with stochastic rounding of the elements.  Returns (codes
    [R, K/2] uint8, sf swizzled uint8, global_scale [1] fp32)."""
    K = x.shape[1]
    R = x.shape[0] if row_index is None else row_index.shape[0]
    if out is None:
        codes = torch.empty(R, K // 2, dtype=torch.uint8, device=x.device)
        sf = torch.zeros(sf_bytes(R, K // 16), dtype=torch.uint8, device=x.device)
        gs = torch.empty(1, dtype=torch.float32, device=x.device)
    else:
        codes, sf, gs = out
    bsq.bsq_quant_nvfp4_sr(x, R, K, _ld(x), block_2d, rht_mask is not None, rht_mask or 0, row_index, amax_in, gs,
                           seed, stream_id, codes, sf)
    return codes, sf, gs


def quant_mxfp4(x, sr=False, seed=0, stream_id=0, out=None):
    """Row-wise MXFP4.  Returns (codes [M,K/2], sf swizzled)."""
    M, K = x.shape
    if out is None:
        codes = torch.empty(M, K // 2, dtype=torch.uint8, device=x.device)
        sf = torch.zeros(sf_bytes(M, K // 32), dtype=torch.uint8, device=x.device)
    else:
        codes, sf = out
    bsq.bsq_quant_mxfp4(x, M, K, _ld(x), bsq.BSQ_SR if sr else bsq.BSQ_RNE, seed, stream_id, codes, sf)
    return codes, sf


def rht(x, mask, out=None):
    y = torch.empty_like(x) if out is None else out
    bsq.bsq_rht(x, y, x.shape[0], x.shape[1], _ld(x), _ld(y), mask)
    return y


def requant_transpose(codes_row, sf_row, sr=True, seed=0, stream_id=1, out=None):
    M, K = codes_row.shape
    if out is None:
        cc = torch.empty(K, M, dtype=torch.uint8, device=codes_row.device)
        sc = torch.zeros(sf_bytes(K, M // 32), dtype=torch.uint8, device=codes_row.device)
    else:
        cc, sc = out
    bsq.bsq_requant_transpose(codes_row, sf_row, M, K, bsq.BSQ_SR if sr else bsq.BSQ_RNE, seed, stream_id, cc, sc)
    return cc, sc


def _out(M, N, dtype, device):
    """[M, N] output whose row stride is a multiple of 16 bytes (a view of a
    padded buffer when N needs it)."""
    per = 16 // torch.tensor([], dtype=dtype).element_size()
    ld = -(-N // per) * per
    return torch.empty(M, ld, dtype=dtype, device=device)[:, :N]


def gemm(fmt, A, sfA, B, sfB, M, N, K, gsA=None, gsB=None, out_dtype=torch.bfloat16, out=None):
    C_out = _out(M, N, out_dtype, A.device) if out is None else out
    ot = bsq.BSQ_OUT_BF16 if C_out.dtype == torch.bfloat16 else bsq.BSQ_OUT_F32
    bsq.bsq_gemm_blockscaled(fmt, A, sfA, gsA, B, sfB, gsB, M, N, K, C_out, C_out.stride(0), ot)
    return C_out


def grouped_gemm(fmt, row_offsets, sf_row_offsets, A, sfA, B, sfB, M_total, N, K, gsA=None, gsB=None,
                 out_dtype=torch.bfloat16, out=None):
    G = row_offsets.shape[0] - 1
    C_out = _out(M_total, N, out_dtype, A.device) if out is None else out
    ot = bsq.BSQ_OUT_BF16 if C_out.dtype == torch.bfloat16 else bsq.BSQ_OUT_F32
    bsq.bsq_grouped_gemm(fmt, G, row_offsets, sf_row_offsets, M_total, A, sfA, gsA, B, sfB, gsB, N, K, C_out,
                         C_out.stride(0), ot)
    return C_out


def grouped_gemm_nvfp4_out(row_offsets, sf_row_offsets, A, sfA, B, sfB, M_total, N, K, out_gs, sf_rows,
                           gsA=None, gsB=None, four_over_six=True, amax=True, bf16_out=False, out=None):
    """Grouped NVFP4 GEMM with the output quantized to NVFP4 in the epilogue
    (given global scale out_gs [1]).  Returns (codes [M_total, N/2], sf
    swizzled with sf_rows rows, amax [1] or None, C bf16 or None)."""
    G = row_offsets.shape[0] - 1
    if out is None:
        codes = torch.empty(M_total, N // 2, dtype=torch.uint8, device=A.device)
        sf = torch.zeros(sf_bytes(sf_rows, N // 16), dtype=torch.uint8, device=A.device)
        am = torch.empty(1, dtype=torch.float32, device=A.device) if amax else None
        C_out = _out(M_total, N, torch.bfloat16, A.device) if bf16_out else None
    else:
        codes, sf, am, C_out = out
    bsq.bsq_grouped_gemm_nvfp4_out(bsq.BSQ_NVFP4, G, row_offsets, sf_row_offsets, M_total, A, sfA, gsA, B, sfB, gsB,
                                   N, K, out_gs, four_over_six, codes, sf, am, C_out,
                                   C_out.stride(0) if C_out is not None else 0)
    return codes, sf, am, C_out


def quant_s2f6(x, rht_mask=None, out=None):
    """RHT (optional) + block-scaled S2F6.  Returns (codes [M, K] int8, sf [M, K/32] uint8)."""
    M, K = x.shape
    if out is None:
        codes = torch.empty(M, K, dtype=torch.int8, device=x.device)
        sf = torch.empty(M, K // 32, dtype=torch.uint8, device=x.device)
    else:
        codes, sf = out
    bsq.bsq_quant_s2f6(x, M, K, _ld(x), rht_mask is not None, rht_mask or 0, codes, sf)
    return codes, sf


def combine_s2f6(codes, sf, token_offsets, rows, weights, rht_mask, out=None):
    """Per token: weighted sum of its S2F6 rows, inverse RHT, bf16 [T, K]."""
    K = codes.shape[1]
    T = token_offsets.shape[0] - 1
    y = torch.empty(T, K, dtype=torch.bfloat16, device=codes.device) if out is None else out
    bsq.bsq_combine_s2f6(codes, sf, K, token_offsets, rows, weights, T, rht_mask, y, _ld(y))
    return y


def quant_nvfp4_gather(x, row_index, four_over_six=False, rht_mask=None, groups=None, amax_in=None, out=None,
                       workspace=None):
    """bsq_quant_nvfp4 of the rows x[row_index] (same bytes), computed by
    quantizing each source row once.  Returns (codes, sf, global_scale)."""
    T, K = x.shape
    R = row_index.shape[0]
    G, ro, so = 0, None, None
    sf_rows = R
    if groups is not None:
        ro, so, sf_rows = groups
        G = ro.shape[0] - 1
    if out is None:
        codes = torch.empty(R, K // 2, dtype=torch.uint8, device=x.device)
        sf = torch.zeros(sf_bytes(sf_rows, K // 16), dtype=torch.uint8, device=x.device)
        gs = torch.empty(1, dtype=torch.float32, device=x.device)
    else:
        codes, sf, gs = out
    nbytes = bsq.bsq_quant_nvfp4_gather_workspace(T, K)
    if workspace is None:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=x.device)
    bsq.bsq_quant_nvfp4_gather(x, T, K, _ld(x), row_index, R, four_over_six, rht_mask is not None, rht_mask or 0, G,
                               ro, so, amax_in, gs, codes, sf, workspace, workspace.numel())
    return codes, sf, gs
