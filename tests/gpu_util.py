"""Shared helpers for the GPU parity tests: move seeded inputs to the device,
bring outputs back, unswizzle scale factors with the oracle's layout function
and compare."""
import numpy as np
import torch

from fp8_math_b200 import workloads as W


def dev(t):
    return t.cuda()


def host_u8(t):
    return t.cpu().numpy().view(np.uint8)


def sf_canonical(ora, sf_dev, rows, nblk):
    """Swizzled device SF buffer -> canonical [rows][nblk] via the oracle's layout."""
    return ora.sf_unswizzle(host_u8(sf_dev), rows, nblk)


def assert_codes_equal(got, want, what):
    got = np.asarray(got)
    want = np.asarray(want)
    assert got.shape == want.shape, (what, got.shape, want.shape)
    bad = np.argwhere(got != want)
    assert bad.size == 0, f"{what}: {len(bad)} mismatches, first at {bad[:5].tolist()}: " \
                          f"got {got[tuple(bad[0])]} want {want[tuple(bad[0])]}"


def bits(t):
    return W.bf16_bits(t)


def gemm_tolerance(C_ref, ref_abs, out_bf16):
    """|gpu - C| <= 1e-3 * sum|a||b| (fp32 accumulation of exact products);
    a bf16 output adds one bf16 rounding: 2^-8 * (|C| + 1e-3 sum|a||b|)."""
    tol = 1e-3 * ref_abs
    if out_bf16:
        tol = tol + 2.0 ** -8 * (np.abs(C_ref) + 1e-3 * ref_abs)
    return tol + 1e-30


def assert_gemm_close(got, C_ref, ref_abs, out_bf16, what):
    got = np.asarray(got, np.float64)
    tol = gemm_tolerance(C_ref, ref_abs, out_bf16)
    err = np.abs(got - C_ref)
    bad = np.argwhere(~(err <= tol))
    assert bad.size == 0, f"{what}: {len(bad)} of {err.size} outside tolerance; first {bad[:5].tolist()}, " \
                          f"got {got[tuple(bad[0])]} want {C_ref[tuple(bad[0])]} tol {tol[tuple(bad[0])]}"


def assert_gemm_full(ora, Cg, dequant_a_rows, B64, out_bf16, what, chunk=2048):
    """Every element of the device output Cg [M, N] against the oracle's
    binary64 GEMM (BLAS form): rows r0..r1 of A decoded by
    dequant_a_rows(r0, r1), B decoded once (B64 [N, K])."""
    M = Cg.shape[0]
    for r0 in range(0, M, chunk):
        r1 = min(M, r0 + chunk)
        Cr, Ra = ora.gemm_f64_blas(dequant_a_rows(r0, r1), B64)
        got = Cg[r0:r1].float().cpu().numpy().astype(np.float64)
        assert_gemm_close(got, Cr, Ra, out_bf16, f"{what} rows {r0}..{r1}")


def assert_quant_full(ora, codes_dev, sf_dev, want, sf_rows, nblk, what, sf_row_of=None, gs_dev=None):
    """Codes (every byte), canonical scale factors (every row) and, for
    NVFP4, the global scale of a device quantization against the oracle's
    want = (codes, sf[, s_g]).  sf_row_of maps output rows to SF rows
    (expert groups); None means the identity."""
    assert_codes_equal(host_u8(codes_dev), want[0], f"{what} codes")
    can = sf_canonical(ora, sf_dev, sf_rows, nblk)
    if sf_row_of is not None:
        can = can[sf_row_of]
    assert_codes_equal(can, want[1], f"{what} scales")
    if gs_dev is not None:
        assert np.float32(gs_dev.item()) == np.float32(want[2]), f"{what} s_g {gs_dev.item()} vs {want[2]}"
