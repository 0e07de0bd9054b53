"""Parity at the workloads' full sizes, in the launch configuration the bench
times (same entry points, same shapes and options).

Quantizers: the GPU quantizes the whole tensor; the oracle quantizes sampled
rows (with the oracle's own amax of the whole tensor, and the SR draw index
offset of the sampled band) and every sampled code, scale and the global
scale must match bit for bit.

GEMMs: the operands are built on the host -- sampled rows are the oracle's
quantization of the workload's real rows, every other row is seeded random
codes with finite scales -- so no input comes from the CUDA path; the GPU
multiplies the full-size operands and outputs are checked at sampled points
(all pairs of sampled rows, ragged edges, random points) against the
oracle's binary64 point GEMM.
"""
import numpy as np
import pytest
import torch

from fp8_math_b200 import api, bsq
from fp8_math_b200 import workloads as W
from gpu_util import assert_codes_equal, assert_gemm_close, bits, dev, host_u8

pytestmark = pytest.mark.gpu

NV, MX = 0, 1


def _sample_rows(R, n, seed, align=1):
    rng = np.random.default_rng(seed)
    rows = set(int(r) for r in rng.integers(0, R // align, n)) | {0, R // align - 1}
    return np.array(sorted(rows), np.int64) * align


def _canon_sf_rows(ora, sf_dev, rows_total, nblk, rows):
    can = ora.sf_unswizzle(host_u8(sf_dev), rows_total, nblk)
    return can[rows]


def sparse_operand(fmt, R, K, real_rows, real_q, seed):
    """Codes/canonical SF of an R x K operand: rows in real_rows come from the
    oracle quantization real_q=(codes, sf[, g]) (same row order), the rest are
    seeded random codes with scales in a finite, moderate range."""
    rng = np.random.default_rng(seed)
    if fmt == NV:
        codes = rng.integers(0, 256, (R, K // 2), dtype=np.uint8)
        sf = rng.integers(0x28, 0x48, (R, K // 16), dtype=np.uint8)   # E4M3 ~0.125 .. 4
    else:
        codes = rng.integers(0, 256, (R, K), dtype=np.uint8)
        codes[(codes & 0x7F) == 0x7F] = 0x01                           # no E4M3 NaN codes
        sf = rng.integers(120, 134, (R, K // 32), dtype=np.uint8)      # 2^-7 .. 2^6
    codes[real_rows] = real_q[0]
    sf[real_rows] = real_q[1]
    return codes, sf


def upload_q(ora, codes, sf):
    return dev(torch.from_numpy(np.ascontiguousarray(codes))), dev(torch.from_numpy(ora.sf_swizzle(sf)))


def check_points(ora, fmt, Cg, qa, qb, K, pm, pn, out_bf16, what):
    Cr, Ra = ora.gemm_points(fmt, qa, qb, K, pm, pn)
    got = Cg[torch.from_numpy(pm), torch.from_numpy(pn)].float().cpu().numpy().astype(np.float64)
    assert_gemm_close(got, Cr, Ra, out_bf16, what)


def pair_points(ra, rb, M, N, n_random, seed):
    pm, pn = np.meshgrid(ra, rb, indexing="ij")
    pm, pn = pm.ravel(), pn.ravel()
    return pm, pn


# ---------------------------------------------------------------- NVFP4 linear with RHT
def test_nvfp4_linear_rht_full_size(ora):
    """8192x4096 A (1x16, RHT) and 14336x4096 W (16x16, RHT); GEMM 8192x14336x4096 bf16."""
    A, Wt, seed = W.nvfp4_linear_rht()
    mask = bsq.bsq_rht_sign_mask(seed)
    M, K = A.shape
    N = Wt.shape[0]
    xa, xw = bits(A), bits(Wt)
    # -- quantizers, full size on the GPU
    ca, sa, ga = api.quant_nvfp4(dev(A), rht_mask=mask)
    cw, sw, gw = api.quant_nvfp4(dev(Wt), block_2d=True, rht_mask=mask)
    assert bsq.bsq_check() == bsq.BSQ_OK
    amax_a = ora.amax(xa, rht_mask=mask)
    amax_w = ora.amax(xw, rht_mask=mask)
    ra = _sample_rows(M, 384, 1)
    rw = _sample_rows(N, 24, 2, align=16)
    rw = np.concatenate([np.arange(r, r + 16) for r in rw])
    qa = ora.quant_nvfp4(xa[ra], rht_mask=mask, amax_in=amax_a)
    qw = ora.quant_nvfp4(xw[rw], block_2d=True, rht_mask=mask, amax_in=amax_w)
    assert np.float32(ga.item()) == np.float32(qa[2]) and np.float32(gw.item()) == np.float32(qw[2])
    assert_codes_equal(host_u8(ca)[ra], qa[0], "A codes (sampled rows)")
    assert_codes_equal(_canon_sf_rows(ora, sa, M, K // 16, ra), qa[1], "A scales (sampled rows)")
    assert_codes_equal(host_u8(cw)[rw], qw[0], "W codes (sampled 16-row tiles)")
    assert_codes_equal(_canon_sf_rows(ora, sw, N, K // 16, rw), qw[1], "W scales (sampled tiles)")
    # -- GEMM at full size on host-built operands
    gA = ra[::6][:64]
    gW = rw[::16][:64]
    codes_a, sf_a = sparse_operand(NV, M, K, gA, (qa[0][::6][:64], qa[1][::6][:64]), 11)
    codes_w, sf_w = sparse_operand(NV, N, K, gW, (qw[0][::16][:64], qw[1][::16][:64]), 12)
    a_d, sa_d = upload_q(ora, codes_a, sf_a)
    w_d, sw_d = upload_q(ora, codes_w, sf_w)
    gsa = dev(torch.tensor([qa[2]], dtype=torch.float32))
    gsw = dev(torch.tensor([qw[2]], dtype=torch.float32))
    Cg = api.gemm(NV, a_d, sa_d, w_d, sw_d, M, N, K, gsA=gsa, gsB=gsw, out_dtype=torch.bfloat16)
    assert bsq.bsq_check() == bsq.BSQ_OK
    pm, pn = pair_points(gA, gW, M, N, 0, 0)
    sm, sn = W.sample_points(M, N, 512, seed=5)
    pm = np.concatenate([pm, sm])
    pn = np.concatenate([pn, sn])
    check_points(ora, NV, Cg, (codes_a, sf_a, qa[2]), (codes_w, sf_w, qw[2]), K, pm, pn, True, "NVFP4 GEMM full size")


# ---------------------------------------------------------------- MXFP8 backward + rollout
def test_mxfp8_backward_and_rollout_full_size(ora):
    """dY 8192x14336 row- and column-wise, W and X column-wise (SR, seed 4,
    streams 0..3); dgrad 8192x4096 (K=14336, bf16), wgrad 14336x4096
    (K=8192, fp32); rollout NVFP4 64x14336 (K=4096, bf16)."""
    dY, Wt, X, A_roll = W.mxfp8_backward()
    M, N = dY.shape          # 8192, 14336
    K = Wt.shape[1]          # 4096
    xdy, xw, xx = bits(dY), bits(Wt), bits(X)
    dY_d, W_d, X_d = dev(dY), dev(Wt), dev(X)
    seed = 4
    c_dy_r, s_dy_r = api.quant_mxfp8(dY_d, sr=True, seed=seed, stream_id=0)   # [M, N], blocks along N
    c_dy_c, s_dy_c = api.quant_mxfp8(dY_d, colwise=True, sr=True, seed=seed, stream_id=1)  # [N, M]
    c_w_c, s_w_c = api.quant_mxfp8(W_d, colwise=True, sr=True, seed=seed, stream_id=2)     # [K, N]
    c_x_c, s_x_c = api.quant_mxfp8(X_d, colwise=True, sr=True, seed=seed, stream_id=3)     # [K, M]
    assert bsq.bsq_check() == bsq.BSQ_OK
    # sampled bands of output rows (SR draw indices offset by the band start)
    r0 = 4000
    q_dy_r = ora.quant_mxfp8(xdy[r0:r0 + 64], sr=True, seed=seed, stream_id=0, out_row0=r0)
    assert_codes_equal(host_u8(c_dy_r)[r0:r0 + 64], q_dy_r[0], "dY row codes")
    assert_codes_equal(_canon_sf_rows(ora, s_dy_r, M, N // 32, np.arange(r0, r0 + 64)), q_dy_r[1], "dY row sf")
    k0 = 14336 - 64
    q_dy_c = ora.quant_mxfp8(np.ascontiguousarray(xdy[:, k0:k0 + 64]), colwise=True, sr=True, seed=seed,
                             stream_id=1, out_row0=k0)
    assert_codes_equal(host_u8(c_dy_c)[k0:k0 + 64], q_dy_c[0], "dY col codes")
    assert_codes_equal(_canon_sf_rows(ora, s_dy_c, N, M // 32, np.arange(k0, k0 + 64)), q_dy_c[1], "dY col sf")
    k1 = 2048
    q_w_c = ora.quant_mxfp8(np.ascontiguousarray(xw[:, k1:k1 + 32]), colwise=True, sr=True, seed=seed,
                            stream_id=2, out_row0=k1)
    assert_codes_equal(host_u8(c_w_c)[k1:k1 + 32], q_w_c[0], "W col codes")
    q_x_c = ora.quant_mxfp8(np.ascontiguousarray(xx[:, 0:32]), colwise=True, sr=True, seed=seed, stream_id=3)
    assert_codes_equal(host_u8(c_x_c)[0:32], q_x_c[0], "X col codes")

    # dgrad: dX[M, K] = dY[M, N] . W[N, K]  ->  A = dY row-wise [M, N], B = W column-wise [K, N]
    ra = np.arange(r0, r0 + 64)
    rb = np.arange(k1, k1 + 32)
    ca, sa = sparse_operand(MX, M, N, ra, q_dy_r, 21)
    cb, sb = sparse_operand(MX, K, N, rb, q_w_c, 22)
    a_d, sa_d = upload_q(ora, ca, sa)
    b_d, sb_d = upload_q(ora, cb, sb)
    Cg = api.gemm(MX, a_d, sa_d, b_d, sb_d, M, K, N, out_dtype=torch.bfloat16)
    assert bsq.bsq_check() == bsq.BSQ_OK
    pm, pn = pair_points(ra[::4], rb, M, K, 0, 0)
    sm, sn = W.sample_points(M, K, 256, seed=6)
    check_points(ora, MX, Cg, (ca, sa, 1.0), (cb, sb, 1.0), N, np.concatenate([pm, sm]), np.concatenate([pn, sn]),
                 True, "dgrad")
    del a_d, b_d, Cg

    # wgrad: dW[N, K] = dY^T[N, M] . X[M, K] -> A = dY column-wise [N, M], B = X column-wise [K, M]
    ra = np.arange(k0, k0 + 64)
    rb = np.arange(0, 32)
    ca, sa = sparse_operand(MX, N, M, ra, q_dy_c, 23)
    cb, sb = sparse_operand(MX, K, M, rb, q_x_c, 24)
    a_d, sa_d = upload_q(ora, ca, sa)
    b_d, sb_d = upload_q(ora, cb, sb)
    Cg = api.gemm(MX, a_d, sa_d, b_d, sb_d, N, K, M, out_dtype=torch.float32)
    assert bsq.bsq_check() == bsq.BSQ_OK
    pm, pn = pair_points(ra[::4], rb, N, K, 0, 0)
    sm, sn = W.sample_points(N, K, 256, seed=7)
    check_points(ora, MX, Cg, (ca, sa, 1.0), (cb, sb, 1.0), M, np.concatenate([pm, sm]), np.concatenate([pn, sn]),
                 False, "wgrad")
    del a_d, b_d, Cg

    # rollout decode: C[64, N] = A_roll (NVFP4 1x16) . W (NVFP4 16x16)^T (swap-AB path)
    qa = ora.quant_nvfp4(bits(A_roll))
    amax_w = ora.amax(xw)
    rw = _sample_rows(N, 16, 3, align=16)
    rw = np.concatenate([np.arange(r, r + 16) for r in rw])
    qw = ora.quant_nvfp4(xw[rw], block_2d=True, amax_in=amax_w)
    cw, sw = sparse_operand(NV, N, K, rw, qw, 25)
    a_d, sa_d = upload_q(ora, qa[0], qa[1])
    w_d, sw_d = upload_q(ora, cw, sw)
    Cg = api.gemm(NV, a_d, sa_d, w_d, sw_d, 64, N, K, gsA=dev(torch.tensor([qa[2]], dtype=torch.float32)),
                  gsB=dev(torch.tensor([qw[2]], dtype=torch.float32)), out_dtype=torch.bfloat16)
    assert bsq.bsq_check() == bsq.BSQ_OK
    pm, pn = pair_points(np.arange(64), rw[::2], 64, N, 0, 0)
    sm, sn = W.sample_points(64, N, 256, seed=8)
    check_points(ora, NV, Cg, (qa[0], qa[1], qa[2]), (cw, sw, qw[2]), K, np.concatenate([pm, sm]),
                 np.concatenate([pn, sn]), True, "rollout")


# ---------------------------------------------------------------- MoE forward
def test_moe_forward_full_size(ora):
    """16384 tokens, 64 experts, top-8 (131072 routed rows): gathered 4/6
    quantize of X with per-expert scale rows, grouped up (N=1536, K=4096)
    and down (N=4096, K=1536) GEMMs."""
    moe = W.moe_forward()
    T, H = moe.X.shape
    E, F, _ = moe.W_up.shape
    ri, offs, sfo = moe.row_index, moe.row_offsets, moe.sf_row_offsets
    Mt = int(offs[-1])
    xX = bits(moe.X)
    ri_d = dev(torch.from_numpy(ri))
    offs_d = dev(torch.from_numpy(offs))
    sfo_d = dev(torch.from_numpy(sfo))
    cx, sx, gx = api.quant_nvfp4(dev(moe.X), four_over_six=True, row_index=ri_d, groups=(offs_d, sfo_d, int(sfo[-1])))
    assert bsq.bsq_check() == bsq.BSQ_OK
    amax_x = ora.amax(xX, row_index=ri)
    rows = _sample_rows(Mt, 512, 4)
    qx = ora.quant_nvfp4(xX, four_over_six=True, row_index=ri[rows], amax_in=amax_x)
    assert np.float32(gx.item()) == np.float32(qx[2])
    assert_codes_equal(host_u8(cx)[rows], qx[0], "X gathered codes")
    expert = np.searchsorted(offs, rows, side="right") - 1
    sf_rows = rows - offs[expert] + sfo[expert]
    assert_codes_equal(_canon_sf_rows(ora, sx, int(sfo[-1]), H // 16, sf_rows), qx[1], "X gathered scales")

    def grouped_case(K, N, Wexp, real_rows, real_q, g_a, exp_sel, what, seed):
        # A: routed rows [Mt, K]; its SF rows at the per-expert offsets
        ca, sa = sparse_operand(NV, Mt, K, real_rows, real_q, seed)
        can = np.zeros((int(sfo[-1]), K // 16), np.uint8)
        for e in range(E):
            can[sfo[e]:sfo[e] + offs[e + 1] - offs[e]] = sa[offs[e]:offs[e + 1]]
        # B: per-expert weights; real rows for the selected experts' first 64 rows
        rng = np.random.default_rng(seed + 1)
        cb = rng.integers(0, 256, (E, N, K // 2), dtype=np.uint8)
        sb = rng.integers(0x28, 0x48, (E, N, K // 16), dtype=np.uint8)
        gsb = np.full(E, 1e-3, np.float32)
        for e in exp_sel:
            qw = ora.quant_nvfp4(bits(Wexp[e, :64].contiguous()), block_2d=True, amax_in=ora.amax(bits(Wexp[e])))
            cb[e, :64] = qw[0]
            sb[e, :64] = qw[1]
            gsb[e] = qw[2]
        sfb = np.concatenate([ora.sf_swizzle(sb[e]) for e in range(E)])
        Cg = api.grouped_gemm(NV, offs_d, sfo_d, dev(torch.from_numpy(ca)), dev(torch.from_numpy(ora.sf_swizzle(can))),
                              dev(torch.from_numpy(cb)), dev(torch.from_numpy(sfb)), Mt, N, K,
                              gsA=dev(torch.tensor([g_a], dtype=torch.float32)), gsB=dev(torch.from_numpy(gsb)),
                              out_dtype=torch.bfloat16)
        assert bsq.bsq_check() == bsq.BSQ_OK
        for e in exp_sel:
            r = real_rows[(real_rows >= offs[e]) & (real_rows < offs[e + 1])][:16]
            if len(r) == 0:
                r = np.array([offs[e], offs[e + 1] - 1])
            pm, pn = np.meshgrid(r, np.arange(0, 64, 3), indexing="ij")
            pm, pn = pm.ravel(), pn.ravel()
            Cr, Ra = ora.gemm_points(NV, (ca, sa, g_a), (cb[e], sb[e], gsb[e]), K, pm, pn)
            got = Cg[torch.from_numpy(pm), torch.from_numpy(pn)].float().cpu().numpy().astype(np.float64)
            assert_gemm_close(got, Cr, Ra, True, f"{what} expert {e}")
        return Cg

    exp_sel = [int(expert[0]), int(expert[len(expert) // 2]), int(expert[-1])]
    grouped_case(H, F, moe.W_up, rows, (qx[0], qx[1]), qx[2], exp_sel, "up", 31)
    # down: A = H rows (a seeded bf16 stand-in for the up output), 4/6 grouped quantize
    g = torch.Generator().manual_seed(33)
    Hs = (torch.randn(len(rows), F, generator=g) * 0.5).to(torch.bfloat16)
    qh = ora.quant_nvfp4(bits(Hs), four_over_six=True)
    grouped_case(F, H, moe.W_dn, rows, (qh[0], qh[1]), qh[2], exp_sel, "down", 41)
