"""Canary bytes around every output buffer: each call writes only inside its
outputs.  The outputs are views into larger buffers filled with a canary
byte; after the call, the bytes before and after each view are unchanged,
and so are the scale-factor padding bytes (rows past the tensor's last row
within a 128-row atom, blocks past the last block within a 4-block group),
which the quantizers never write."""
import numpy as np
import pytest
import torch

from fp8_math_b200 import api, bsq
from fp8_math_b200 import workloads as W
from gpu_util import dev

pytestmark = pytest.mark.gpu

CANARY = 0xA5
PAD = 256  # guard bytes on each side (a multiple of 16 keeps the views aligned)


def guarded(nbytes):
    """(whole buffer, view of nbytes in its middle), canary-filled."""
    buf = torch.full((PAD + nbytes + PAD,), CANARY, dtype=torch.uint8, device="cuda")
    return buf, buf[PAD:PAD + nbytes]


def check_guards(buf, nbytes, what):
    h = buf.cpu().numpy()
    assert (h[:PAD] == CANARY).all(), f"{what}: bytes before the output changed"
    assert (h[PAD + nbytes:] == CANARY).all(), f"{what}: bytes after the output changed"


def sf_padding_mask(rows, nblk):
    """True at the bytes of a swizzled SF buffer that no (row, block) maps to."""
    used = np.zeros(bsq.bsq_sf_bytes(rows, nblk), bool)
    bt = (nblk + 3) // 4
    r = np.arange(rows)[:, None]
    b = np.arange(nblk)[None, :]
    off = ((r // 128) * bt + b // 4) * 512 + (r % 32) * 16 + ((r // 32) % 4) * 4 + (b % 4)
    used[off.ravel()] = True
    return ~used


def check_sf(buf, rows, nblk, what):
    n = bsq.bsq_sf_bytes(rows, nblk)
    check_guards(buf, n, what + " sf")
    body = buf.cpu().numpy()[PAD:PAD + n]
    assert (body[sf_padding_mask(rows, nblk)] == CANARY).all(), f"{what}: SF padding written"


def edge(M, K, seed):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(M, K, generator=g)
    x[0, :16] = 0.0
    return x.to(torch.bfloat16)


@pytest.mark.parametrize("M,K,two_d,fos,rht", [(37, 80, False, False, False), (130, 1024, False, True, True),
                                               (48, 80, True, False, True), (256, 4096, True, False, True),
                                               (200, 4096, False, False, True)])
def test_nvfp4_writes_only_its_outputs(M, K, two_d, fos, rht):
    x = dev(edge(M, K, M + K))
    cb, c = guarded(M * K // 2)
    sb, s = guarded(bsq.bsq_sf_bytes(M, K // 16))
    gb, g = guarded(16)
    api.quant_nvfp4(x, block_2d=two_d, four_over_six=fos, rht_mask=0x1234 if rht else None,
                    out=(c.view(M, K // 2), s, g[:4].view(torch.float32)))
    assert bsq.bsq_check() == bsq.BSQ_OK
    check_guards(cb, M * K // 2, "nvfp4 codes")
    check_sf(sb, M, K // 16, "nvfp4")
    assert (gb.cpu().numpy()[PAD + 4:] == CANARY).all() and (gb.cpu().numpy()[:PAD] == CANARY).all()


@pytest.mark.parametrize("two_d", [False, True])
def test_nvfp4_sr_writes_only_its_outputs(two_d):
    M, K = 48, 272
    x = dev(edge(M, K, 5))
    cb, c = guarded(M * K // 2)
    sb, s = guarded(bsq.bsq_sf_bytes(M, K // 16))
    gb, g = guarded(16)
    api.quant_nvfp4_sr(x, block_2d=two_d, rht_mask=0x00F0, seed=3, out=(c.view(M, K // 2), s, g[:4].view(torch.float32)))
    assert bsq.bsq_check() == bsq.BSQ_OK
    check_guards(cb, M * K // 2, "nvfp4 sr codes")
    check_sf(sb, M, K // 16, "nvfp4 sr")


@pytest.mark.parametrize("M,K,colwise,sr", [(100, 96, False, True), (64, 4096, False, False), (33, 3072, False, True),
                                            (96, 200, True, True), (160, 40, True, False), (2048, 72, True, True)])
def test_mxfp8_writes_only_its_outputs(M, K, colwise, sr):
    x = dev(edge(M, K, 7 * M + K))
    R, C = (K, M) if colwise else (M, K)
    cb, c = guarded(R * C)
    sb, s = guarded(bsq.bsq_sf_bytes(R, C // 32))
    api.quant_mxfp8(x, colwise=colwise, sr=sr, seed=1, out=(c.view(R, C), s))
    assert bsq.bsq_check() == bsq.BSQ_OK
    check_guards(cb, R * C, "mxfp8 codes")
    check_sf(sb, R, C // 32, "mxfp8")


def test_requant_and_mxfp4_write_only_their_outputs():
    M, K = 96, 160
    x = dev(edge(M, K, 9))
    c1, s1 = api.quant_mxfp8(x, sr=True, seed=1)
    cb, c = guarded(K * M)
    sb, s = guarded(bsq.bsq_sf_bytes(K, M // 32))
    api.requant_transpose(c1, s1, sr=True, seed=1, out=(c.view(K, M), s))
    check_guards(cb, K * M, "requant codes")
    check_sf(sb, K, M // 32, "requant")
    cb, c = guarded(M * K // 2)
    sb, s = guarded(bsq.bsq_sf_bytes(M, K // 32))
    api.quant_mxfp4(x, sr=True, seed=2, out=(c.view(M, K // 2), s))
    assert bsq.bsq_check() == bsq.BSQ_OK
    check_guards(cb, M * K // 2, "mxfp4 codes")
    check_sf(sb, M, K // 32, "mxfp4")


def test_rht_writes_only_its_output():
    M, K = 37, 80
    x = dev(edge(M, K, 11))
    yb, y = guarded(M * K * 2)
    api.rht(x, 0x0F0F, out=y.view(torch.bfloat16).view(M, K))
    assert bsq.bsq_check() == bsq.BSQ_OK
    check_guards(yb, M * K * 2, "rht")


@pytest.mark.parametrize("fmt,M,N,K,out_bf16", [(0, 200, 264, 256, True), (0, 300, 512, 512, True),
                                                (1, 130, 256, 128, False), (0, 64, 1000, 256, True)])
def test_gemm_writes_only_its_tile_of_c(fmt, M, N, K, out_bf16):
    """C is a strided view (ldc = N + 8) one row into a larger buffer: the
    rows around it and the columns past N stay untouched."""
    A = dev(edge(M, K, 1))
    B = dev(edge(N, K, 2))
    if fmt == 0:
        qa, qb = api.quant_nvfp4(A), api.quant_nvfp4(B, block_2d=N % 16 == 0)
        gsa, gsb = qa[2], qb[2]
    else:
        qa, qb = api.quant_mxfp8(A), api.quant_mxfp8(B)
        gsa = gsb = None
    dt = torch.bfloat16 if out_bf16 else torch.float32
    ldc = N + 8
    big = torch.full((M + 2, ldc), float("nan"), dtype=dt, device="cuda")
    C = big[1:M + 1, :N]
    api.gemm(fmt, qa[0], qa[1], qb[0], qb[1], M, N, K, gsA=gsa, gsB=gsb, out=C)
    assert bsq.bsq_check() == bsq.BSQ_OK
    h = big.float().cpu().numpy()
    assert np.isnan(h[0]).all() and np.isnan(h[M + 1]).all(), "rows around C written"
    assert np.isnan(h[1:M + 1, N:]).all(), "columns past N written"
    assert np.isfinite(h[1:M + 1, :N]).all(), "C not fully written"
