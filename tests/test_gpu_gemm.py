"""GPU block-scaled GEMM and grouped GEMM against the CPU oracle.

Operands are quantized by the ORACLE (so these tests do not depend on the
GPU quantizers), uploaded, multiplied by the tcgen05 kernels and compared
element by element with the oracle's binary64 GEMM of the decoded operands:
|gpu - C| <= 1e-3 * sum_k |a_mk b_nk| (plus one bf16 rounding for bf16
outputs).  Small shapes are checked in full (several tiles, ragged M/N/K
tails, the swap-AB path for skinny M); the full-size workloads on sampled
outputs.
"""
import numpy as np
import pytest
import torch

from fp8_math_b200 import api, bsq
from fp8_math_b200 import workloads as W
from gpu_util import assert_gemm_close, bits, dev

pytestmark = pytest.mark.gpu

NV, MX, MX4 = 0, 1, 2


def oracle_operands(ora, fmt, A, B, rht=None, fos=False, b2d=True, sr=False, seed=0):
    """Quantize A [M,K] and B [N,K] with the oracle; returns host tuples
    (codes, canonical sf, s_g)."""
    if fmt == NV:
        qa = ora.quant_nvfp4(bits(A), rht_mask=rht, four_over_six=fos)
        qb = ora.quant_nvfp4(bits(B), block_2d=b2d and B.shape[0] % 16 == 0, rht_mask=rht)
    elif fmt == MX4:
        qa = (*ora.quant_mxfp4(bits(A), sr=sr, seed=seed, stream_id=0), 1.0)
        qb = (*ora.quant_mxfp4(bits(B), sr=sr, seed=seed, stream_id=1), 1.0)
    else:
        qa = (*ora.quant_mxfp8(bits(A), sr=sr, seed=seed, stream_id=0), 1.0)
        qb = (*ora.quant_mxfp8(bits(B), sr=sr, seed=seed, stream_id=1), 1.0)
    return qa, qb


def upload(ora, q):
    c, s, g = q
    return (dev(torch.from_numpy(np.ascontiguousarray(c))), dev(torch.from_numpy(ora.sf_swizzle(s))),
            dev(torch.tensor([g], dtype=torch.float32)))


def run_gemm(ora, fmt, qa, qb, M, N, K, out_dtype):
    a, sa, ga = upload(ora, qa)
    b, sb, gb = upload(ora, qb)
    Cg = api.gemm(fmt, a, sa, b, sb, M, N, K, gsA=ga if fmt == NV else None, gsB=gb if fmt == NV else None,
                  out_dtype=out_dtype)
    assert bsq.bsq_check() == bsq.BSQ_OK
    return Cg.float().cpu().numpy().astype(np.float64)


# kernel: 0 = single-CTA tiles, 1 = the CTA-pair (cta_group::2) kernel,
# forced through the dispatch's tuning switch (the default picks pairs for
# operands of 256+ rows)
@pytest.mark.parametrize("pair", [0, 1])
@pytest.mark.parametrize("fmt", [NV, MX, MX4])
@pytest.mark.parametrize("M,N,K,out", [
    (128, 256, 256, torch.float32),     # the small NVFP4 linear workload shape
    (256, 512, 512, torch.bfloat16),    # BN = 256 path, several tiles
    (200, 136, 384, torch.float32),     # ragged M, N; K % 256 = 128
    (300, 520, 1024, torch.bfloat16),   # ragged, several k-tiles
    (129, 129, 128, torch.bfloat16),    # one-past-tile edges
    (64, 1024, 512, torch.bfloat16),    # swap-AB (skinny M)
    (1, 256, 256, torch.float32),       # M = 1
    (17, 384, 640, torch.float32),      # swap-AB ragged
])
def test_gemm_full_compare(ora, knobs, pair, fmt, M, N, K, out):
    knobs(bsq.BSQ_KNOB_GEMM_PAIR, pair)
    A, Bm = W.nvfp4_linear_small(M=M, N=N, K=K, seed=M * 7 + N + K)
    qa, qb = oracle_operands(ora, fmt, A, Bm)
    Cg = run_gemm(ora, fmt, qa, qb, M, N, K, out)
    da = ora.dequant(fmt, *qa)
    db = ora.dequant(fmt, *qb)
    Cr, Ra = ora.gemm_f64(da, db)
    assert_gemm_close(Cg, Cr, Ra, out == torch.bfloat16, f"gemm pair={pair} fmt={fmt} {M}x{N}x{K}")


# the skinny (swap-AB) GEMM split over K: clusters of S CTAs, partial sums
# added in the rank-0 CTA; S = 1 is the unsplit kernel, -1 the automatic
# choice.  K runs that do not divide evenly (K / 256 = 7, 9), more CTAs than
# k-tiles (clamped), several W tiles, ragged token and W-row counts.
@pytest.mark.parametrize("split", [-1, 1, 2, 4, 8])
@pytest.mark.parametrize("fmt", [NV, MX, MX4])
@pytest.mark.parametrize("M,N,K,out", [
    (64, 1024, 2048, torch.bfloat16),
    (37, 400, 1792, torch.float32),
    (8, 256, 2304, torch.bfloat16),
    (64, 384, 512, torch.float32),
])
def test_gemm_splitk_compare(ora, knobs, split, fmt, M, N, K, out):
    knobs(bsq.BSQ_KNOB_GEMM_SPLITK, split)
    A, Bm = W.nvfp4_linear_small(M=M, N=N, K=K, seed=M * 5 + N + K)
    qa, qb = oracle_operands(ora, fmt, A, Bm)
    Cg = run_gemm(ora, fmt, qa, qb, M, N, K, out)
    Cr, Ra = ora.gemm_f64(ora.dequant(fmt, *qa), ora.dequant(fmt, *qb))
    assert_gemm_close(Cg, Cr, Ra, out == torch.bfloat16, f"split-K {split} fmt={fmt} {M}x{N}x{K}")


def test_gemm_small_linear_workload_exact_inputs(ora):
    """NVFP4 linear, 128x256 (1x16) times 256x256 (16x16), fp32 output."""
    A, Wt = W.nvfp4_linear_small()
    qa, qb = oracle_operands(ora, NV, A, Wt)
    Cg = run_gemm(ora, NV, qa, qb, 128, 256, 256, torch.float32)
    Cr, Ra = ora.gemm_f64(ora.dequant(NV, *qa), ora.dequant(NV, *qb))
    assert_gemm_close(Cg, Cr, Ra, False, "small linear")


@pytest.mark.parametrize("pair", [0, 1])
@pytest.mark.parametrize("fmt", [NV, MX, MX4])
def test_grouped_gemm_compare(ora, knobs, pair, fmt):
    """Small MoE: routed rows grouped by expert (uneven counts, one expert
    possibly empty), per-expert B and global scales."""
    knobs(bsq.BSQ_KNOB_GEMM_PAIR, pair)
    E, T, H, F = 6, 96, 256, 192
    g = torch.Generator().manual_seed(5)
    logits = torch.randn(T, E, generator=g)
    logits[:, 5] = -1e9  # expert 5 receives no rows
    ri, offs, sfo = W.route_topk(logits, 2)
    X = torch.randn(T, H, generator=g).to(torch.bfloat16)
    Wup = (torch.randn(E, F, H, generator=g) * 0.02).to(torch.bfloat16)
    Mt = int(offs[-1])
    Xg = X[torch.from_numpy(ri.astype(np.int64))]
    if fmt == NV:
        qa = ora.quant_nvfp4(bits(Xg), four_over_six=True)
        qbs = [ora.quant_nvfp4(bits(Wup[e]), block_2d=True) for e in range(E)]
    elif fmt == MX4:
        qa = (*ora.quant_mxfp4(bits(Xg)), 1.0)
        qbs = [(*ora.quant_mxfp4(bits(Wup[e])), 1.0) for e in range(E)]
    else:
        qa = (*ora.quant_mxfp8(bits(Xg)), 1.0)
        qbs = [(*ora.quant_mxfp8(bits(Wup[e])), 1.0) for e in range(E)]
    vec = 16 if fmt == NV else 32
    # A's SF rows per expert at 128-aligned offsets
    sfA = np.zeros(int(sfo[-1]) * W.round_up(H // vec, 4), np.uint8)
    can = np.zeros((int(sfo[-1]), H // vec), np.uint8)
    for e in range(E):
        can[sfo[e]:sfo[e] + offs[e + 1] - offs[e]] = qa[1][offs[e]:offs[e + 1]]
    sfA[:] = ora.sf_swizzle(can)
    Bc = np.stack([q[0] for q in qbs])
    sfB = np.concatenate([ora.sf_swizzle(q[1]) for q in qbs])
    gsB = np.array([q[2] for q in qbs], np.float32)
    Cg = api.grouped_gemm(fmt, dev(torch.from_numpy(offs)), dev(torch.from_numpy(sfo)),
                          dev(torch.from_numpy(qa[0])), dev(torch.from_numpy(sfA)),
                          dev(torch.from_numpy(Bc)), dev(torch.from_numpy(sfB)), Mt, F, H,
                          gsA=dev(torch.tensor([qa[2]], dtype=torch.float32)) if fmt == NV else None,
                          gsB=dev(torch.from_numpy(gsB)) if fmt == NV else None, out_dtype=torch.bfloat16)
    assert bsq.bsq_check() == bsq.BSQ_OK
    Cg = Cg.float().cpu().numpy().astype(np.float64)
    da = ora.dequant(fmt, *qa)
    for e in range(E):
        r0, r1 = offs[e], offs[e + 1]
        if r1 == r0:
            continue
        Cr, Ra = ora.gemm_f64(da[r0:r1], ora.dequant(fmt, *qbs[e]))
        assert_gemm_close(Cg[r0:r1], Cr, Ra, True, f"grouped fmt={fmt} expert {e}")


def test_gemm_invalid_arguments():
    z = torch.zeros(256, dtype=torch.uint8, device="cuda")
    Cm = torch.zeros(4, 4, device="cuda")
    with pytest.raises(bsq.BsqError) as e:
        bsq.bsq_gemm_blockscaled(NV, z, z, None, z, z, None, 4, 4, 100, Cm, 4, bsq.BSQ_OUT_F32)
    assert e.value.status == bsq.BSQ_ERR_INVALID
    assert bsq.bsq_check() == bsq.BSQ_OK


@pytest.mark.parametrize("fos", [True, False])
def test_grouped_gemm_nvfp4_output(ora, fos):
    """The quantizing epilogue: a grouped NVFP4 GEMM (small MoE up
    projection, K = 256, N = 192) writing NVFP4 with a given global scale.
    With the scale of the output's own amax it reproduces, byte for byte, the
    plain GEMM's bf16 output quantized by bsq_quant_nvfp4 (same groups, same
    Four Over Six); its amax is that output's; and its codes and scales have
    the NVFP4 properties (nearest E2M1 codes under candidate scales) on that
    output.  A different scale gives the same properties under that scale."""
    from nvfp4_props import check_nvfp4
    E, T, H, F = 6, 160, 256, 192
    g = torch.Generator().manual_seed(21)
    logits = torch.randn(T, E, generator=g)
    logits[:, 4] = -1e9  # expert 4 receives no rows
    ri, offs, sfo = W.route_topk(logits, 2)
    X = torch.randn(T, H, generator=g).to(torch.bfloat16)
    Wup = (torch.randn(E, F, H, generator=g) * 0.02).to(torch.bfloat16)
    Mt, sf_rows = int(offs[-1]), int(sfo[-1])
    Xg = X[torch.from_numpy(ri.astype(np.int64))]
    qa = ora.quant_nvfp4(bits(Xg), four_over_six=True)
    qbs = [ora.quant_nvfp4(bits(Wup[e]), block_2d=True) for e in range(E)]
    can = np.zeros((sf_rows, H // 16), np.uint8)
    for e in range(E):
        can[sfo[e]:sfo[e] + offs[e + 1] - offs[e]] = qa[1][offs[e]:offs[e + 1]]
    offs_d, sfo_d = dev(torch.from_numpy(offs)), dev(torch.from_numpy(sfo))
    A, sA = dev(torch.from_numpy(qa[0])), dev(torch.from_numpy(ora.sf_swizzle(can)))
    B = dev(torch.from_numpy(np.stack([q[0] for q in qbs])))
    sB = dev(torch.from_numpy(np.concatenate([ora.sf_swizzle(q[1]) for q in qbs])))
    gA = dev(torch.tensor([qa[2]], dtype=torch.float32))
    gB = dev(torch.tensor([q[2] for q in qbs], dtype=torch.float32))
    Hp = api.grouped_gemm(NV, offs_d, sfo_d, A, sA, B, sB, Mt, F, H, gsA=gA, gsB=gB, out_dtype=torch.bfloat16)
    amax = api.amax(Hp)
    gs = dev(torch.tensor([np.float32(np.float32(amax.item()) / np.float32(2688.0))], dtype=torch.float32))
    codes, sf, am, Hq = api.grouped_gemm_nvfp4_out(offs_d, sfo_d, A, sA, B, sB, Mt, F, H, gs, sf_rows, gsA=gA,
                                                   gsB=gB, four_over_six=fos, bf16_out=True)
    assert bsq.bsq_check() == bsq.BSQ_OK
    assert torch.equal(Hq.view(torch.int16), Hp.view(torch.int16))
    assert am.item() == amax.item()
    rc, rs, rg = api.quant_nvfp4(Hp, four_over_six=fos, groups=(offs_d, sfo_d, sf_rows), amax_in=amax)
    assert bsq.bsq_check() == bsq.BSQ_OK
    assert torch.equal(codes, rc) and torch.equal(sf, rs) and rg.item() == gs.item()
    rows = np.arange(Mt)
    ex = np.searchsorted(offs, rows, side="right") - 1
    sf_row_of = rows - offs[ex] + sfo[ex]
    y = (bits(Hp.cpu()).astype(np.uint32) << 16).view(np.float32)
    can_out = ora.sf_unswizzle(sf.cpu().numpy(), sf_rows, F // 16)[sf_row_of]
    check_nvfp4(y, codes.cpu().numpy(), can_out, gs.item(), four_over_six=fos, what="fused epilogue")
    # another scale (as from an earlier step): the same properties under it
    gs2 = dev(torch.tensor([gs.item() * 1.75], dtype=torch.float32))
    codes2, sf2, am2, _ = api.grouped_gemm_nvfp4_out(offs_d, sfo_d, A, sA, B, sB, Mt, F, H, gs2, sf_rows, gsA=gA,
                                                     gsB=gB, four_over_six=fos)
    assert bsq.bsq_check() == bsq.BSQ_OK
    assert am2.item() == amax.item()
    can2 = ora.sf_unswizzle(sf2.cpu().numpy(), sf_rows, F // 16)[sf_row_of]
    check_nvfp4(y, codes2.cpu().numpy(), can2, gs2.item(), four_over_six=fos, check_sg=False,
                what="fused epilogue, earlier scale")
