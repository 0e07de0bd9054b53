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
