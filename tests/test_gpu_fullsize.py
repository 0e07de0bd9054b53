"""Parity at the workloads' full sizes, in the launch configuration the bench
times (same entry points, shapes and options), checked in full.

Quantizers: the GPU quantizes the whole tensor and the oracle (its threaded
form: bands of rows on every host core, byte-identical to one thread)
quantizes the whole tensor too; every code byte, every scale factor and the
global scale must match.

GEMMs: the operands are the oracle's quantizations of the workload's
tensors (identical to the GPU's, which the quantizer tests establish), so
no oracle input comes from the CUDA path; the GPU multiplies them and every
output element is compared with the oracle's binary64 product of the decoded
operands within |gpu - C| <= 1e-3 sum |a||b| (+ one bf16 rounding for bf16
outputs).

The MoE forward is also run as one chain on the device (gathered Four Over
Six quantize of X, grouped up GEMM, grouped Four Over Six quantize of the
GPU's own up output H, grouped down GEMM).  Its H is the up GEMM checked
above (the same inputs, bit for bit); the quantization of that H and the
down GEMM that consumes it are checked by properties that hold at any size
(nearest E2M1 codes under candidate scales, and the down product against a
binary64 product of the GPU's codes decoded in the test), because an oracle
run on the GPU's H would take its input from the CUDA path.  The same two
kernels are checked against the oracle on the oracle's own H.
"""
import time

import numpy as np
import pytest
import torch

from fp8_math_b200 import api, bsq
from fp8_math_b200 import workloads as W
from gpu_util import assert_gemm_close, assert_gemm_full, assert_quant_full, bits, dev, host_u8

pytestmark = pytest.mark.gpu

NV, MX = 0, 1


@pytest.fixture(scope="module")
def T(ora):
    return ora.ncores()


def _log(what, t0):
    print(f"[fullsize] {what}: {time.perf_counter() - t0:.1f} s", flush=True)


def _upload(ora, q):
    """Oracle quantization (codes, canonical sf[, s_g]) -> device codes, swizzled sf[, s_g]."""
    out = [dev(torch.from_numpy(np.ascontiguousarray(q[0]))), dev(torch.from_numpy(ora.sf_swizzle(q[1])))]
    if len(q) > 2:
        out.append(dev(torch.tensor([q[2]], dtype=torch.float32)))
    return out


# ---------------------------------------------------------------- NVFP4 linear with RHT
@pytest.fixture(scope="module")
def linear_rht(ora, T):
    t0 = time.perf_counter()
    A, Wt, seed = W.nvfp4_linear_rht()
    mask = bsq.bsq_rht_sign_mask(seed)
    qa = ora.quant_nvfp4(bits(A), rht_mask=mask, threads=T)
    qw = ora.quant_nvfp4(bits(Wt), block_2d=True, rht_mask=mask, threads=T)
    _log("oracle quantize A 8192x4096 (1x16) and W 14336x4096 (16x16), RHT", t0)
    return A, Wt, mask, qa, qw


def test_nvfp4_linear_rht_quantizers_full(ora, linear_rht):
    """A 8192x4096 (1x16, amax pass + quantize pass) and W 14336x4096 (16x16,
    one cooperative launch), both with the RHT: every byte."""
    A, Wt, mask, qa, qw = linear_rht
    M, K = A.shape
    N = Wt.shape[0]
    ca, sa, ga = api.quant_nvfp4(dev(A), rht_mask=mask)
    cw, sw, gw = api.quant_nvfp4(dev(Wt), block_2d=True, rht_mask=mask)
    assert bsq.bsq_check() == bsq.BSQ_OK
    assert_quant_full(ora, ca, sa, qa, M, K // 16, "A", gs_dev=ga)
    assert_quant_full(ora, cw, sw, qw, N, K // 16, "W", gs_dev=gw)


def test_nvfp4_linear_rht_gemm_full(ora, linear_rht, T):
    """C = A W^T, 8192x14336x4096, bf16 output: every element."""
    A, Wt, mask, qa, qw = linear_rht
    M, K = A.shape
    N = Wt.shape[0]
    a = _upload(ora, qa)
    w = _upload(ora, qw)
    Cg = api.gemm(NV, a[0], a[1], w[0], w[1], M, N, K, gsA=a[2], gsB=w[2], out_dtype=torch.bfloat16)
    assert bsq.bsq_check() == bsq.BSQ_OK
    t0 = time.perf_counter()
    B64 = ora.dequant(NV, qw[0], qw[1], qw[2], threads=T)
    assert_gemm_full(ora, Cg, lambda r0, r1: ora.dequant(NV, qa[0][r0:r1], qa[1][r0:r1], qa[2], threads=T), B64,
                     True, "NVFP4 GEMM 8192x14336x4096")
    _log("oracle GEMM check 8192x14336x4096", t0)


# ---------------------------------------------------------------- MXFP8 backward + rollout
@pytest.fixture(scope="module")
def backward(ora, T):
    t0 = time.perf_counter()
    dY, Wt, X, A_roll = W.mxfp8_backward()
    xdy, xw, xx = bits(dY), bits(Wt), bits(X)
    q = {
        "dy_row": ora.quant_mxfp8(xdy, sr=True, seed=4, stream_id=0, threads=T),
        "dy_col": ora.quant_mxfp8(xdy, colwise=True, sr=True, seed=4, stream_id=1, threads=T),
        "w_col": ora.quant_mxfp8(xw, colwise=True, sr=True, seed=4, stream_id=2, threads=T),
        "x_col": ora.quant_mxfp8(xx, colwise=True, sr=True, seed=4, stream_id=3, threads=T),
    }
    _log("oracle MXFP8 SR quantize of dY (row, column), W and X (column)", t0)
    return dY, Wt, X, A_roll, q


def test_mxfp8_backward_quantizers_full(ora, backward):
    """dY 8192x14336 row- and column-wise, W 14336x4096 and X 8192x4096
    column-wise, stochastic rounding (seed 4, streams 0..3): every byte."""
    dY, Wt, X, _, q = backward
    M, N = dY.shape
    K = Wt.shape[1]
    dY_d = dev(dY)
    c, s = api.quant_mxfp8(dY_d, sr=True, seed=4, stream_id=0)
    assert bsq.bsq_check() == bsq.BSQ_OK
    assert_quant_full(ora, c, s, q["dy_row"], M, N // 32, "dY row-wise")
    del c, s
    c, s = api.quant_mxfp8(dY_d, colwise=True, sr=True, seed=4, stream_id=1)
    assert bsq.bsq_check() == bsq.BSQ_OK
    assert_quant_full(ora, c, s, q["dy_col"], N, M // 32, "dY column-wise")
    del c, s, dY_d
    c, s = api.quant_mxfp8(dev(Wt), colwise=True, sr=True, seed=4, stream_id=2)
    assert bsq.bsq_check() == bsq.BSQ_OK
    assert_quant_full(ora, c, s, q["w_col"], K, N // 32, "W column-wise")
    c, s = api.quant_mxfp8(dev(X), colwise=True, sr=True, seed=4, stream_id=3)
    assert bsq.bsq_check() == bsq.BSQ_OK
    assert_quant_full(ora, c, s, q["x_col"], K, M // 32, "X column-wise")


def test_mxfp8_rowcol_full(ora, backward):
    """dY 8192x14336 row- and column-wise in one pass (seed 4, streams 0 and
    1): every byte equals the two separate quantizations' oracle."""
    dY, _, _, _, q = backward
    M, N = dY.shape
    cr, sr_, cc, sc = api.quant_mxfp8_rowcol(dev(dY), sr=True, seed=4, stream_id_row=0, stream_id_col=1)
    assert bsq.bsq_check() == bsq.BSQ_OK
    assert_quant_full(ora, cr, sr_, q["dy_row"], M, N // 32, "dY row-wise (one pass)")
    assert_quant_full(ora, cc, sc, q["dy_col"], N, M // 32, "dY column-wise (one pass)")


def test_requant_saved_nvfp4_weight_full(ora, linear_rht, T):
    """The RHT linear's W 14336x4096 saved in NVFP4 (16x16) -> MXFP8
    column-wise [4096, 14336] with stochastic rounding: every byte."""
    _, Wt, _, _, qw = linear_rht
    N, K = Wt.shape
    codes = dev(torch.from_numpy(qw[0]))
    sf = dev(torch.from_numpy(ora.sf_swizzle(qw[1])))
    gs = dev(torch.tensor([qw[2]], dtype=torch.float32))
    cc, sc = api.requant_nvfp4_mxfp8(codes, sf, gs, sr=True, seed=4, stream_id=2)
    assert bsq.bsq_check() == bsq.BSQ_OK
    want = ora.requant_nvfp4_mxfp8(*qw, sr=True, seed=4, stream_id=2, threads=T)
    assert_quant_full(ora, cc, sc, want, K, N // 32, "W NVFP4 -> MXFP8 column-wise")


def test_mxfp8_dgrad_full(ora, backward, T):
    """dX = dY . W: A = dY row-wise [8192, 14336], B = W column-wise
    [4096, 14336], bf16 output: every element."""
    dY, Wt, _, _, q = backward
    M, N = dY.shape
    K = Wt.shape[1]
    a = _upload(ora, q["dy_row"])
    b = _upload(ora, q["w_col"])
    Cg = api.gemm(MX, a[0], a[1], b[0], b[1], M, K, N, out_dtype=torch.bfloat16)
    assert bsq.bsq_check() == bsq.BSQ_OK
    del a, b
    t0 = time.perf_counter()
    B64 = ora.dequant(MX, *q["w_col"], threads=T)
    A = q["dy_row"]
    assert_gemm_full(ora, Cg, lambda r0, r1: ora.dequant(MX, A[0][r0:r1], A[1][r0:r1], threads=T), B64, True,
                     "dgrad 8192x4096x14336")
    _log("oracle dgrad check", t0)


def test_mxfp8_wgrad_full(ora, backward, T):
    """dW = dY^T . X: A = dY column-wise [14336, 8192], B = X column-wise
    [4096, 8192], fp32 output: every element."""
    dY, Wt, X, _, q = backward
    M, N = dY.shape
    K = Wt.shape[1]
    a = _upload(ora, q["dy_col"])
    b = _upload(ora, q["x_col"])
    Cg = api.gemm(MX, a[0], a[1], b[0], b[1], N, K, M, out_dtype=torch.float32)
    assert bsq.bsq_check() == bsq.BSQ_OK
    del a, b
    t0 = time.perf_counter()
    B64 = ora.dequant(MX, *q["x_col"], threads=T)
    A = q["dy_col"]
    assert_gemm_full(ora, Cg, lambda r0, r1: ora.dequant(MX, A[0][r0:r1], A[1][r0:r1], threads=T), B64, False,
                     "wgrad 14336x4096x8192")
    _log("oracle wgrad check", t0)


def test_rollout_gemm_full(ora, backward, T):
    """Rollout decode: C [64, 14336] = A_roll (NVFP4 1x16) . W (NVFP4 16x16)^T,
    K = 4096, bf16 output (the swap-AB kernel): every element."""
    _, Wt, _, A_roll, _ = backward
    N, K = Wt.shape
    qa = ora.quant_nvfp4(bits(A_roll))
    qw = ora.quant_nvfp4(bits(Wt), block_2d=True, threads=T)
    ca, sa, ga = api.quant_nvfp4(dev(A_roll))
    cw, sw, gw = api.quant_nvfp4(dev(Wt), block_2d=True)
    assert bsq.bsq_check() == bsq.BSQ_OK
    assert_quant_full(ora, ca, sa, qa, 64, K // 16, "rollout A", gs_dev=ga)
    assert_quant_full(ora, cw, sw, qw, N, K // 16, "rollout W", gs_dev=gw)
    a = _upload(ora, qa)
    w = _upload(ora, qw)
    Cg = api.gemm(NV, a[0], a[1], w[0], w[1], 64, N, K, gsA=a[2], gsB=w[2], out_dtype=torch.bfloat16)
    assert bsq.bsq_check() == bsq.BSQ_OK
    assert_gemm_full(ora, Cg, lambda r0, r1: ora.dequant(NV, qa[0][r0:r1], qa[1][r0:r1], qa[2]),
                     ora.dequant(NV, *qw, threads=T), True, "rollout 64x14336x4096")


# ---------------------------------------------------------------- NVFP4 / MXFP4 next-row formats at full size
def test_nvfp4_sr_workload_full(ora, linear_rht, T):
    """NVFP4 with stochastic rounding (seed 2, stream 1) of the whole RHT
    linear's A (1x16) and W (16x16): every byte."""
    A, Wt, mask, _, _ = linear_rht
    K = A.shape[1]
    for t, two_d in ((A, False), (Wt, True)):
        c, s, g = api.quant_nvfp4_sr(dev(t), block_2d=two_d, rht_mask=mask, seed=2, stream_id=1)
        assert bsq.bsq_check() == bsq.BSQ_OK
        want = ora.quant_nvfp4_sr(bits(t), block_2d=two_d, rht_mask=mask, seed=2, stream_id=1, threads=T)
        assert_quant_full(ora, c, s, want, t.shape[0], K // 16, f"nvfp4 sr 2d={two_d}", gs_dev=g)


# ---------------------------------------------------------------- MoE forward
def _experts_oracle(ora, Wx, T):
    """Oracle 16x16 quantization of every expert weight [E, N, K]."""
    return [ora.quant_nvfp4(bits(Wx[e]), block_2d=True, threads=T) for e in range(Wx.shape[0])]


def _experts_device(ora, qs, N, K):
    """Expert quantizations -> device codes [E, N, K/2], concatenated swizzled
    SF buffers and global scales [E]."""
    codes = dev(torch.from_numpy(np.stack([q[0] for q in qs])))
    sfb = dev(torch.from_numpy(np.concatenate([ora.sf_swizzle(q[1]) for q in qs])))
    gsb = dev(torch.tensor([q[2] for q in qs], dtype=torch.float32))
    return codes, sfb, gsb


def _grouped_sf(ora, q, offs, sfo, K):
    """Oracle codes/canonical SF of routed rows -> device codes and the
    swizzled SF buffer with each expert's rows at its SF offset."""
    can = np.zeros((int(sfo[-1]), K // 16), np.uint8)
    for e in range(len(offs) - 1):
        can[sfo[e]:sfo[e] + offs[e + 1] - offs[e]] = q[1][offs[e]:offs[e + 1]]
    return dev(torch.from_numpy(q[0])), dev(torch.from_numpy(ora.sf_swizzle(can)))


def _sf_rows_of(offs, sfo):
    rows = np.arange(int(offs[-1]))
    e = np.searchsorted(offs, rows, side="right") - 1
    return rows - offs[e] + sfo[e]


def _check_grouped_full(ora, Cg, qa, qws, offs, out_bf16, what, T):
    """Every row of every expert's output against the oracle's binary64 GEMM."""
    for e in range(len(offs) - 1):
        r0, r1 = int(offs[e]), int(offs[e + 1])
        if r0 == r1:
            continue
        B64 = ora.dequant(NV, *qws[e], threads=T)
        A64 = ora.dequant(NV, qa[0][r0:r1], qa[1][r0:r1], qa[2], threads=T)
        Cr, Ra = ora.gemm_f64_blas(A64, B64)
        got = Cg[r0:r1].float().cpu().numpy().astype(np.float64)
        assert_gemm_close(got, Cr, Ra, out_bf16, f"{what} expert {e}")


def test_moe_forward_chain_full(ora, T):
    """16384 tokens, hidden 4096, 64 experts of ffn 1536, top-8 (131072
    routed rows), every output checked:
      1. gathered Four Over Six quantize of X with per-expert SF rows, and the
         16x16 quantize of every expert weight, against the oracle;
      2. grouped up GEMM (N 1536, K 4096) on those operands against the
         oracle's binary64 GEMM;
      3. the device chain: its H is that up output; the grouped Four Over Six
         quantize of H (131072x1536) checked by the NVFP4 properties, and the
         grouped down GEMM (N 4096, K 1536) on it checked against binary64
         products of its decoded operands;
      4. the same quantize and down GEMM on the oracle's own H (its binary64
         up output rounded to bf16) against the oracle."""
    from nvfp4_props import check_nvfp4, decode_nvfp4
    t0 = time.perf_counter()
    moe = W.moe_forward()
    Tk, H = moe.X.shape
    E, F, _ = moe.W_up.shape
    ri, offs, sfo = moe.row_index, moe.row_offsets, moe.sf_row_offsets
    Mt, sf_rows = int(offs[-1]), int(sfo[-1])
    ri_d, offs_d, sfo_d = dev(torch.from_numpy(ri)), dev(torch.from_numpy(offs)), dev(torch.from_numpy(sfo))
    sf_row_of = _sf_rows_of(offs, sfo)
    _log("MoE inputs", t0)

    # 1. quantizers
    t0 = time.perf_counter()
    qx = ora.quant_nvfp4(bits(moe.X), four_over_six=True, row_index=ri, threads=T)
    qup = _experts_oracle(ora, moe.W_up, T)
    qdn = _experts_oracle(ora, moe.W_dn, T)
    _log("oracle quantize X (gathered 4/6) and 128 expert weights", t0)
    cx, sx, gx = api.quant_nvfp4(dev(moe.X), four_over_six=True, row_index=ri_d, groups=(offs_d, sfo_d, sf_rows))
    assert bsq.bsq_check() == bsq.BSQ_OK
    assert_quant_full(ora, cx, sx, qx, sf_rows, H // 16, "X gathered 4/6", sf_row_of=sf_row_of, gs_dev=gx)
    # the same bytes by quantizing each token once and moving its rows
    cg, sg_, gg = api.quant_nvfp4_gather(dev(moe.X), ri_d, four_over_six=True, groups=(offs_d, sfo_d, sf_rows))
    assert bsq.bsq_check() == bsq.BSQ_OK
    assert torch.equal(cg, cx) and torch.equal(sg_, sx) and gg.item() == gx.item()
    del cg, sg_, gg
    up_dev = _experts_device(ora, qup, F, H)
    dn_dev = _experts_device(ora, qdn, H, F)
    for e in (0, E // 2, E - 1):   # the device's own weight quantization gives the same bytes
        cw, sw, gw = api.quant_nvfp4(dev(moe.W_up[e]), block_2d=True)
        assert_quant_full(ora, cw, sw, qup[e], F, H // 16, f"W_up[{e}]", gs_dev=gw)
    del moe

    # 2. up GEMM (its inputs are the device quantizations, equal to the oracle's)
    Hg = api.grouped_gemm(NV, offs_d, sfo_d, cx, sx, up_dev[0], up_dev[1], Mt, F, H, gsA=gx, gsB=up_dev[2],
                          out_dtype=torch.bfloat16)
    assert bsq.bsq_check() == bsq.BSQ_OK
    t0 = time.perf_counter()
    _check_grouped_full(ora, Hg, qx, qup, offs, True, "up", T)
    _log("oracle check of the up GEMM", t0)
    del up_dev

    # 3. the device chain: 4/6 quantize of the device's H, then the down GEMM
    ch, sh, gh = api.quant_nvfp4(Hg, four_over_six=True, groups=(offs_d, sfo_d, sf_rows))
    # the up GEMM with the quantizing epilogue, given the chain's global scale,
    # writes the same bytes without storing H
    up_dev = _experts_device(ora, qup, F, H)
    fc, fs, fa, _ = api.grouped_gemm_nvfp4_out(offs_d, sfo_d, cx, sx, up_dev[0], up_dev[1], Mt, F, H, gh, sf_rows,
                                               gsA=gx, gsB=up_dev[2], four_over_six=True)
    assert bsq.bsq_check() == bsq.BSQ_OK
    assert torch.equal(fc, ch) and torch.equal(fs, sh)
    assert fa.item() == api.amax(Hg).item()
    del fc, fs, fa, up_dev
    Cd = api.grouped_gemm(NV, offs_d, sfo_d, ch, sh, dn_dev[0], dn_dev[1], Mt, H, F, gsA=gh, gsB=dn_dev[2],
                          out_dtype=torch.bfloat16)
    assert bsq.bsq_check() == bsq.BSQ_OK
    t0 = time.perf_counter()
    yh = (bits(Hg.cpu()).astype(np.uint32) << 16).view(np.float32)
    sh_can = ora.sf_unswizzle(host_u8(sh), sf_rows, F // 16)[sf_row_of]
    ch_h = host_u8(ch)
    picked4 = check_nvfp4(yh, ch_h, sh_can, gh.item(), four_over_six=True, what="H (device chain) 4/6")
    assert picked4 > 0
    _log("property check of the chain's H quantization", t0)
    t0 = time.perf_counter()
    for e in range(E):
        r0, r1 = int(offs[e]), int(offs[e + 1])
        if r0 == r1:
            continue
        A64 = decode_nvfp4(ch_h[r0:r1], sh_can[r0:r1], gh.item())
        B64 = decode_nvfp4(qdn[e][0], qdn[e][1], qdn[e][2])
        Cr, Ra = A64 @ B64.T, np.abs(A64) @ np.abs(B64).T
        assert_gemm_close(Cd[r0:r1].float().cpu().numpy().astype(np.float64), Cr, Ra, True,
                          f"down (device chain) expert {e}")
    _log("binary64 check of the chain's down GEMM", t0)
    del ch, sh, Cd, yh, ch_h, sh_can, cx, sx

    # 4. the oracle's own H through the same two kernels
    t0 = time.perf_counter()
    Hb = torch.zeros(Mt, F, dtype=torch.bfloat16)
    for e in range(E):
        r0, r1 = int(offs[e]), int(offs[e + 1])
        if r0 == r1:
            continue
        A64 = ora.dequant(NV, qx[0][r0:r1], qx[1][r0:r1], qx[2], threads=T)
        Hb[r0:r1] = torch.from_numpy(ora.gemm_f64_blas(A64, ora.dequant(NV, *qup[e], threads=T))[0]).to(torch.bfloat16)
    qh = ora.quant_nvfp4(bits(Hb), four_over_six=True, threads=T)
    _log("oracle H (binary64 up output, bf16) and its 4/6 quantize", t0)
    ch, sh, gh = api.quant_nvfp4(dev(Hb), four_over_six=True, groups=(offs_d, sfo_d, sf_rows))
    assert bsq.bsq_check() == bsq.BSQ_OK
    assert_quant_full(ora, ch, sh, qh, sf_rows, F // 16, "H (oracle) 4/6", sf_row_of=sf_row_of, gs_dev=gh)
    a, sa = _grouped_sf(ora, qh, offs, sfo, F)
    Cd = api.grouped_gemm(NV, offs_d, sfo_d, a, sa, dn_dev[0], dn_dev[1], Mt, H, F,
                          gsA=dev(torch.tensor([qh[2]], dtype=torch.float32)), gsB=dn_dev[2],
                          out_dtype=torch.bfloat16)
    assert bsq.bsq_check() == bsq.BSQ_OK
    t0 = time.perf_counter()
    _check_grouped_full(ora, Cd, qh, qdn, offs, True, "down", T)
    _log("oracle check of the down GEMM", t0)
