"""CPU checks of the C-ABI library: it loads, exports every entry point that
include/bsq.h declares, and its host-only helpers and argument validation
behave (no device work is issued by these calls)."""
import ctypes as C
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from fp8_math_b200 import bsq
    if not os.path.exists(bsq.LIB_PATH):
        from fp8_math_b200 import build
        build.build()
    return bsq


def declared_symbols():
    with open(os.path.join(ROOT, "include", "bsq.h")) as f:
        text = f.read()
    return sorted(set(re.findall(r"BSQ_API[^;(]*?\b(bsq_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_symbols()
    for n in ["bsq_amax", "bsq_quant_nvfp4", "bsq_quant_mxfp8", "bsq_rht", "bsq_requant_transpose",
              "bsq_gemm_blockscaled", "bsq_grouped_gemm", "bsq_check"]:
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    L = C.CDLL(lib.LIB_PATH)
    for n in declared_symbols():
        assert hasattr(L, n), n


def test_sf_bytes_matches_oracle_layout(lib, ora):
    for rows, nb in [(1, 1), (128, 16), (8192, 256), (131, 3), (0, 5)]:
        assert lib.bsq_sf_bytes(rows, nb) == ora.sf_swizzled_bytes(rows, nb)


def test_rht_sign_mask_matches_oracle(lib, ora):
    for seed in [0, 1, 2, 3, 4, 2**40 + 17, 2**64 - 1]:
        assert lib.bsq_rht_sign_mask(seed) == ora.rht_sign_mask(seed)


def test_validation_rejects_before_any_device_work(lib):
    L = lib.lib()
    # NULL / misaligned pointers and bad shapes are refused on the host
    assert L.bsq_quant_nvfp4(None, 16, 16, 16, 0, 0, 0, 0, None, 0, None, None, None, None, None, None,
                             None) == lib.BSQ_ERR_INVALID
    assert L.bsq_quant_nvfp4(16, 16, 24, 24, 0, 0, 0, 0, None, 0, None, None, None, 64, 64, 64,
                             None) == lib.BSQ_ERR_INVALID  # K % 16
    assert L.bsq_quant_nvfp4(16, 16, 32, 32, 1, 1, 0, 0, None, 0, None, None, None, 64, 64, 64,
                             None) == lib.BSQ_ERR_INVALID  # 2-D with Four Over Six
    assert L.bsq_quant_nvfp4(8, 16, 32, 32, 0, 0, 0, 0, None, 0, None, None, None, 64, 64, 64,
                             None) == lib.BSQ_ERR_ALIGN    # x not 16-byte aligned
    assert L.bsq_quant_mxfp8(16, 4, 48, 48, 0, 0, 0, 0, 64, 64, None) == lib.BSQ_ERR_INVALID  # K % 32
    assert L.bsq_quant_mxfp8(16, 4, 64, 64, 0, 7, 0, 0, 64, 64, None) == lib.BSQ_ERR_INVALID  # rounding
    assert L.bsq_gemm_blockscaled(0, 16, 16, None, 16, 16, None, 4, 4, 96, 16, 4, 0, None) == lib.BSQ_ERR_INVALID
    assert L.bsq_gemm_blockscaled(5, 16, 16, None, 16, 16, None, 4, 4, 128, 16, 4, 0, None) == lib.BSQ_ERR_INVALID
    assert L.bsq_requant_transpose(16, 16, 48, 32, 0, 0, 0, 16, 16, None) == lib.BSQ_ERR_INVALID  # M % 32
    assert L.bsq_debug_timeout_probe(0, None) == lib.BSQ_ERR_INVALID
    assert lib.status_str(lib.BSQ_ERR_TIMEOUT) == "device-side wait timed out"


def declared_parameter_counts():
    """name -> number of parameters, from each BSQ_API declaration."""
    with open(os.path.join(ROOT, "include", "bsq.h")) as f:
        text = re.sub(r"/\*.*?\*/", "", f.read(), flags=re.S)
    out = {}
    for m in re.finditer(r"BSQ_API[^;(]*?\b(bsq_\w+)\s*\(([^)]*)\)\s*;", text, flags=re.S):
        params = m.group(2).strip()
        out[m.group(1)] = 0 if params in ("", "void") else params.count(",") + 1
    return out


def test_binding_matches_header_signatures(lib):
    """Every declared entry point has a ctypes binding with the header's
    number of parameters, and the binding names nothing the header lacks."""
    decl = declared_parameter_counts()
    assert set(decl) == set(lib._SIGS), (sorted(set(decl) ^ set(lib._SIGS)))
    for name, n in decl.items():
        assert len(lib._SIGS[name][1]) == n, (name, n, len(lib._SIGS[name][1]))


def test_validation_of_the_fp4_variants(lib):
    L = lib.lib()
    # MXFP4: K % 32, rounding mode, alignment
    assert L.bsq_quant_mxfp4(16, 4, 48, 48, 0, 0, 0, 64, 64, None) == lib.BSQ_ERR_INVALID
    assert L.bsq_quant_mxfp4(16, 4, 64, 64, 7, 0, 0, 64, 64, None) == lib.BSQ_ERR_INVALID
    assert L.bsq_quant_mxfp4(8, 4, 64, 64, 0, 0, 0, 64, 64, None) == lib.BSQ_ERR_ALIGN
    assert L.bsq_quant_mxfp4(16, 4, 64, 60, 0, 0, 0, 64, 64, None) == lib.BSQ_ERR_INVALID  # ldx < K
    # NVFP4 with stochastic rounding: K % 16, 2-D needs M % 16 and no gather, alignment
    assert L.bsq_quant_nvfp4_sr(16, 16, 24, 24, 0, 0, 0, None, None, 64, 0, 0, 64, 64, None) == lib.BSQ_ERR_INVALID
    assert L.bsq_quant_nvfp4_sr(16, 8, 32, 32, 1, 0, 0, None, None, 64, 0, 0, 64, 64, None) == lib.BSQ_ERR_INVALID
    assert L.bsq_quant_nvfp4_sr(16, 16, 32, 32, 1, 0, 0, 64, None, 64, 0, 0, 64, 64, None) == lib.BSQ_ERR_INVALID
    assert L.bsq_quant_nvfp4_sr(16, 16, 32, 32, 0, 0, 0, None, None, 66, 0, 0, 64, 64, None) == lib.BSQ_ERR_ALIGN
    assert L.bsq_quant_nvfp4_sr(None, 16, 32, 32, 0, 0, 0, None, None, 64, 0, 0, 64, 64, None) == lib.BSQ_ERR_INVALID


def test_kernel_choice_knobs_validate(lib):
    L = lib.lib()
    assert L.bsq_debug_kernel_choice(7, 0) == lib.BSQ_ERR_INVALID
    assert L.bsq_debug_kernel_choice(lib.BSQ_KNOB_FUSED_QUANT, 2) == lib.BSQ_ERR_INVALID
    assert L.bsq_debug_kernel_choice(lib.BSQ_KNOB_GEMM_BN, 64) == lib.BSQ_ERR_INVALID
    assert L.bsq_debug_kernel_choice(lib.BSQ_KNOB_GEMM_SPLITK, 3) == lib.BSQ_ERR_INVALID
    assert L.bsq_debug_kernel_choice(lib.BSQ_KNOB_LAUNCH_OVERLAP, 2) == lib.BSQ_ERR_INVALID
    for knob, value in [(lib.BSQ_KNOB_FUSED_QUANT, 0), (lib.BSQ_KNOB_GEMM_PAIR, 1), (lib.BSQ_KNOB_GEMM_BN, 256),
                        (lib.BSQ_KNOB_LAUNCH_OVERLAP, 0)]:
        assert L.bsq_debug_kernel_choice(knob, value) == lib.BSQ_OK
        assert L.bsq_debug_kernel_choice(knob, -1) == lib.BSQ_OK


def test_gathered_quantize_bounds_the_group_count(lib):
    """bsq_quant_nvfp4_gather moves scale words with the group offsets held in
    shared memory (at most 1024 groups): more is refused on the host, before
    any CUDA call.  The pointers are placeholders that are never dereferenced."""
    L = lib.lib()
    p = 256
    ws = lib.bsq_quant_nvfp4_gather_workspace(4, 64)
    args = lambda G: (p, 4, 64, 64, p, 4, 0, 0, 0, G, p, p, None, p, p, p, p, ws, None)
    assert L.bsq_quant_nvfp4_gather(*args(1025)) == lib.BSQ_ERR_UNSUPPORTED
    assert L.bsq_quant_nvfp4_gather(*args(-1)) == lib.BSQ_ERR_INVALID


def test_scale_row_movers_bound_their_size(lib):
    """bsq_sf_to_rows / bsq_sf_from_rows index with 32-bit arithmetic and
    refuse rows * nblk >= 2^31 on the host, before any CUDA call (the
    pointers are placeholders that are never dereferenced)."""
    L = lib.lib()
    assert L.bsq_sf_to_rows(256, 1 << 20, 1 << 11, 256, None) == lib.BSQ_ERR_UNSUPPORTED
    assert L.bsq_sf_from_rows(256, 1 << 20, 1 << 11, 0, None, None, 256, None) == lib.BSQ_ERR_UNSUPPORTED
    assert L.bsq_sf_to_rows(256, -1, 4, 256, None) == lib.BSQ_ERR_INVALID


def test_noalloc_rejects_requests_beyond_its_scratch(lib):
    """The no-allocation entry point holds one partial maximum per 65536
    elements in a 4096-word array (one word is the counter): 4095 CTAs are
    the most it can take.  A larger request is refused on the host, before
    any CUDA call (on this GPU-less machine a request that fits reaches the
    runtime and fails there instead)."""
    L = lib.lib()
    K = 4096
    fits = 4095 * 65536 // K              # 65520 rows: exactly 4095 CTAs
    assert L.bsq_global_scale_noalloc(16, fits + 1, K, K, 0, 0, 64, None) == lib.BSQ_ERR_UNSUPPORTED
    assert L.bsq_global_scale_noalloc(16, 1 << 41, 16, 16, 0, 0, 64, None) == lib.BSQ_ERR_UNSUPPORTED
    assert L.bsq_global_scale_noalloc(16, 4, 40, 40, 0, 0, 64, None) == lib.BSQ_ERR_INVALID   # K % 16
    assert L.bsq_global_scale_noalloc(8, 4, 64, 64, 0, 0, 64, None) == lib.BSQ_ERR_ALIGN      # x alignment
    import torch
    if not torch.cuda.is_available():
        assert L.bsq_global_scale_noalloc(16, fits, K, K, 0, 0, 64, None) == lib.BSQ_ERR_CUDA


def test_validation_of_the_backward_input_entry_points(lib):
    L = lib.lib()
    # one-pass row + column MXFP8: M % 32, K % 32, rounding, alignment
    assert L.bsq_quant_mxfp8_rowcol(16, 48, 64, 64, 0, 0, 0, 1, 64, 64, 64, 64, None) == lib.BSQ_ERR_INVALID
    assert L.bsq_quant_mxfp8_rowcol(16, 64, 48, 48, 0, 0, 0, 1, 64, 64, 64, 64, None) == lib.BSQ_ERR_INVALID
    assert L.bsq_quant_mxfp8_rowcol(16, 64, 64, 64, 2, 0, 0, 1, 64, 64, 64, 64, None) == lib.BSQ_ERR_INVALID
    assert L.bsq_quant_mxfp8_rowcol(16, 64, 64, 64, 0, 0, 0, 1, 64, 64, 72, 64, None) == lib.BSQ_ERR_ALIGN
    # NVFP4 -> MXFP8: R % 32, C % 16, the global scale pointer
    assert L.bsq_requant_nvfp4_mxfp8(16, 16, 64, 48, 64, 1, 0, 0, 64, 64, None) == lib.BSQ_ERR_INVALID
    assert L.bsq_requant_nvfp4_mxfp8(16, 16, 64, 64, 40, 1, 0, 0, 64, 64, None) == lib.BSQ_ERR_INVALID
    assert L.bsq_requant_nvfp4_mxfp8(16, 16, None, 64, 64, 1, 0, 0, 64, 64, None) == lib.BSQ_ERR_INVALID
    assert L.bsq_requant_nvfp4_mxfp8(16, 16, 66, 64, 64, 1, 0, 0, 64, 64, None) == lib.BSQ_ERR_ALIGN
