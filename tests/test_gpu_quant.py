"""GPU parity of the codec kernels against the CPU oracle (bit-exact).

Inputs are the seeded workloads at sizes the oracle finishes in seconds, plus
edge tensors (zero blocks, exact E2M1 midpoints, saturating blocks, negative
values that round to zero, ragged shapes), and the full-size workloads where
the oracle still runs in seconds.  Codes, scale factors (unswizzled with the
oracle's layout function) and the global scale must match exactly.
"""
import numpy as np
import pytest
import torch

from fp8_math_b200 import api, bsq
from fp8_math_b200 import workloads as W
from gpu_util import assert_codes_equal, bits, dev, host_u8, sf_canonical

pytestmark = pytest.mark.gpu


def edge_tensor(M, K, seed=0):
    """N(0,1) plus: an all-zero block, tiny negatives beside a large value,
    exact E2M1 midpoints under a power-of-two global scale (amax = 2688),
    a saturating column and a block of subnormal-range values."""
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(M, K, generator=g)
    x[0, :16] = 0.0
    if M > 1:
        x[1, 16:32] = -1e-6
        if K >= 32:
            x[1, 20] = 3.0
    mids = torch.tensor([6.0, 2.5, 0.25, 0.75, 1.25, 1.75, 3.5, 5.0, -2.5, -0.25, -0.75, -1.25, -1.75, -3.5, -5.0, 1.0])
    for r in range(2, min(M, 10)):
        x[r, :16] = mids * (2.0 ** (r - 6))
    x[M - 1, K - 1] = 2688.0
    if K > 48:
        x[:, 47] *= 1000.0
        x[M - 1, K - 1] = float(x.abs().max()) * 1.0
    if M > 12 and K >= 32:
        x[12, 16:32] = 1e-30
    return x.to(torch.bfloat16)


def _nvfp4_check(ora, x, block_2d=False, fos=False, rht=None, row_index=None, groups=None, amax_in=None, what=""):
    xd = dev(x)
    ri = None if row_index is None else dev(torch.from_numpy(row_index))
    gr = None
    if groups is not None:
        ro, so = groups
        gr = (dev(torch.from_numpy(ro)), dev(torch.from_numpy(so)), int(so[-1]))
    am = None if amax_in is None else dev(torch.tensor([amax_in], dtype=torch.float32))
    codes, sf, gs = api.quant_nvfp4(xd, block_2d=block_2d, four_over_six=fos, rht_mask=rht, row_index=ri,
                                    groups=gr, amax_in=am)
    assert bsq.bsq_check() == 0
    oc, osf, og = ora.quant_nvfp4(bits(x), block_2d=block_2d, four_over_six=fos, rht_mask=rht,
                                  row_index=row_index, amax_in=amax_in)
    R, K = oc.shape[0], x.shape[1]
    assert np.float32(gs.item()) == np.float32(og), (what, gs.item(), og)
    assert_codes_equal(host_u8(codes), oc, what + " codes")
    if groups is None:
        assert_codes_equal(sf_canonical(ora, sf, R, K // 16), osf, what + " sf")
    else:
        ro, so = groups
        can = ora.sf_unswizzle(host_u8(sf), int(so[-1]), K // 16)
        for e in range(len(ro) - 1):
            n = ro[e + 1] - ro[e]
            assert_codes_equal(can[so[e]:so[e] + n], osf[ro[e]:ro[e + 1]], f"{what} sf group {e}")


# ------------------------------------------------------------------ NVFP4
@pytest.mark.parametrize("M,K", [(128, 256), (1, 16), (3, 48), (37, 80), (256, 512), (130, 1024)])
def test_nvfp4_1d_parity(ora, M, K):
    x = edge_tensor(M, K, seed=M + K)
    _nvfp4_check(ora, x, what=f"nvfp4 1d {M}x{K}")


@pytest.mark.parametrize("rht", [None, 0x5A5A])
@pytest.mark.parametrize("fos", [False, True])
def test_nvfp4_input_16_byte_aligned(ora, rht, fos):
    """A contiguous input that starts 16 bytes past a 32-byte boundary (the
    least alignment the boundary accepts) goes through the flat amax and 1x16
    kernels like an aligned one, and the result is the oracle's."""
    M, K = 64, 512
    x = edge_tensor(M, K, seed=77)
    buf = torch.zeros(M * K + 8, dtype=torch.bfloat16, device="cuda")
    xd = buf[8:].view(M, K)
    xd.copy_(dev(x))
    assert xd.data_ptr() % 32 == 16
    codes, sf, gs = api.quant_nvfp4(xd, four_over_six=fos, rht_mask=rht)
    a = api.amax(xd, rht_mask=rht)
    assert bsq.bsq_check() == 0
    oc, osf, og = ora.quant_nvfp4(bits(x), four_over_six=fos, rht_mask=rht)
    assert np.float32(gs.item()) == np.float32(og)
    assert np.float32(a.item()) == np.float32(ora.amax(bits(x), rht_mask=rht))
    assert_codes_equal(host_u8(codes), oc, "codes (16-byte aligned input)")
    assert_codes_equal(sf_canonical(ora, sf, M, K // 16), osf, "sf (16-byte aligned input)")


@pytest.mark.parametrize("block_2d", [False, True])
def test_nvfp4_two_pass_path(ora, knobs, block_2d):
    """The separate amax and quantize kernels (what gathered, grouped and 4/6
    inputs use), forced for contiguous tensors that otherwise go through the
    fused cooperative kernel."""
    knobs(bsq.BSQ_KNOB_FUSED_QUANT, 0)
    for M, K in [(128, 256), (48, 1040) if block_2d else (37, 80), (160, 4096)]:
        x = edge_tensor(M, K, seed=5 * M + K)
        _nvfp4_check(ora, x, block_2d=block_2d, what=f"two-pass {M}x{K}")
        _nvfp4_check(ora, x, block_2d=block_2d, rht=0x1234, what=f"two-pass rht {M}x{K}")


@pytest.mark.parametrize("M,K", [(16, 64), (48, 576), (1040, 1088), (512, 4096)])
@pytest.mark.parametrize("block_2d", [False, True])
@pytest.mark.parametrize("stream,fused", [(1, 1), (1, 0), (0, 1), (0, 0)])
def test_nvfp4_contiguous_kernel_paths(ora, knobs, stream, fused, block_2d, M, K):
    """Contiguous tensors through each kernel family: the bulk-copy streaming
    kernels (fused amax + quantize in one cooperative launch, or an amax
    launch and a quantize launch) and the register-streaming ones; shapes with
    a partial last chunk, a partial last 512-column span and more chunks than
    CTAs; with and without the RHT and with a given amax."""
    knobs(bsq.BSQ_KNOB_STREAM_QUANT, stream)
    knobs(bsq.BSQ_KNOB_FUSED_QUANT, fused)
    x = edge_tensor(M, K, seed=M + K + block_2d)
    tag = f"stream={stream} fused={fused} 2d={block_2d} {M}x{K}"
    _nvfp4_check(ora, x, block_2d=block_2d, what=tag)
    _nvfp4_check(ora, x, block_2d=block_2d, rht=0x1234, what=tag + " rht")
    _nvfp4_check(ora, x, block_2d=block_2d, rht=0x0F0F, amax_in=float(x.float().abs().max()) * 1.5,
                 what=tag + " given amax")
    xd = dev(x)
    for rht in (None, 0xBEEF):
        a = api.amax(xd, rht_mask=rht)
        assert np.float32(a.item()) == np.float32(ora.amax(bits(x), rht_mask=rht)), tag


def test_nvfp4_small_linear_workload(ora):
    A, Wt = W.nvfp4_linear_small()
    _nvfp4_check(ora, A, what="A 1x16")
    _nvfp4_check(ora, Wt, block_2d=True, what="W 16x16")


@pytest.mark.parametrize("M,K", [(16, 16), (32, 48), (256, 256), (48, 1040), (160, 4096)])
def test_nvfp4_2d_parity(ora, M, K):
    x = edge_tensor(M, K, seed=3 * M + K)
    _nvfp4_check(ora, x, block_2d=True, what=f"nvfp4 2d {M}x{K}")


def _midpoint_tensor(rows_per_block, seed):
    """Blocks whose scale t = (bamax / 6) / s_g sits on an E4M3 rounding
    midpoint (or one bf16 step away): amax = 7168 gives s_g = 7168 / 2688,
    and a block maximum of 16 m makes bamax / (6 s_g) = m exactly in real
    arithmetic, so the fp32 result lands within an ulp or two of the tie.
    Covers every normal-range midpoint (k + 1/2) 2^(e-3) and the subnormal
    ones (k + 1/2) 2^-9."""
    mids = [(k + 0.5) * 2.0 ** (e - 3) for e in range(-6, 9) for k in range(8, 16)]
    mids = [m for m in mids if m < 448] + [(k + 0.5) * 2.0 ** -9 for k in range(8)]
    targets = []
    for m in mids:
        b = torch.tensor([16 * m], dtype=torch.float32).to(torch.bfloat16)
        up = (b.view(torch.int16) + 1).view(torch.bfloat16)
        dn = (b.view(torch.int16) - 1).view(torch.bfloat16)
        targets += [b.item(), up.item(), dn.item()]
    nb = len(targets) + 1
    g = torch.Generator().manual_seed(seed)
    x = torch.empty(rows_per_block, 16 * nb)
    for j in range(nb):
        peak = 7168.0 if j == 0 else targets[j - 1]
        blk = (torch.rand(rows_per_block, 16, generator=g) * 2 - 1) * peak * 0.9
        blk[0, int(j % 16)] = -peak if j % 3 == 1 else peak
        x[:, 16 * j:16 * (j + 1)] = blk
    return x.to(torch.bfloat16)


def test_nvfp4_scale_rounding_midpoints(ora):
    x1 = _midpoint_tensor(1, 11)
    _nvfp4_check(ora, x1, what="1x16 scale midpoints")
    _nvfp4_check(ora, x1, fos=True, what="4/6 scale midpoints")
    x2 = _midpoint_tensor(16, 12)
    _nvfp4_check(ora, x2, block_2d=True, what="16x16 scale midpoints")


@pytest.mark.parametrize("block_2d", [False, True])
def test_nvfp4_rht_parity(ora, block_2d):
    A, Wt, seed = W.nvfp4_linear_rht(M=256, N=272, K=512)
    mask = ora.rht_sign_mask(seed)
    assert bsq.bsq_rht_sign_mask(seed) == mask
    _nvfp4_check(ora, A if not block_2d else Wt, block_2d=block_2d, rht=mask, what="rht")


@pytest.mark.parametrize("M,K", [(64, 256), (200, 1536), (5, 32)])
def test_nvfp4_four_over_six_parity(ora, M, K):
    x = edge_tensor(M, K, seed=7 * M)
    _nvfp4_check(ora, x, fos=True, what="4/6")
    _nvfp4_check(ora, x, fos=True, rht=0x5A5A, what="4/6 + rht")


@pytest.mark.parametrize("rht", [False, True])
@pytest.mark.parametrize("M,K", [(128, 256), (1, 16), (3, 48), (37, 80), (256, 512)])
def test_nvfp4_sr_1d_parity(ora, M, K, rht):
    """NVFP4 with stochastic rounding of the elements, 1x16 blocks."""
    x = edge_tensor(M, K, seed=M + 3 * K)
    mask = 0x5A3C if rht else None
    c, s, g = api.quant_nvfp4_sr(dev(x), rht_mask=mask, seed=11, stream_id=2)
    assert bsq.bsq_check() == 0
    oc, osf, og = ora.quant_nvfp4_sr(bits(x), rht_mask=mask, seed=11, stream_id=2)
    assert np.float32(g.item()) == np.float32(og)
    assert_codes_equal(host_u8(c), oc, "nvfp4 sr codes")
    assert_codes_equal(sf_canonical(ora, s, M, K // 16), osf, "nvfp4 sr sf")


@pytest.mark.parametrize("rht", [False, True])
@pytest.mark.parametrize("M,K", [(32, 256), (48, 80), (16, 16), (64, 1024)])
def test_nvfp4_sr_2d_parity(ora, M, K, rht):
    """NVFP4 with stochastic rounding of the elements, 16x16 tiles."""
    x = edge_tensor(M, K, seed=M * 5 + K)
    mask = 0x3C5A if rht else None
    c, s, g = api.quant_nvfp4_sr(dev(x), block_2d=True, rht_mask=mask, seed=12, stream_id=3)
    oc, osf, og = ora.quant_nvfp4_sr(bits(x), block_2d=True, rht_mask=mask, seed=12, stream_id=3)
    assert np.float32(g.item()) == np.float32(og)
    assert_codes_equal(host_u8(c), oc, "nvfp4 sr 2d codes")
    assert_codes_equal(sf_canonical(ora, s, M, K // 16), osf, "nvfp4 sr 2d sf")


def test_nvfp4_sr_gather_and_given_amax(ora):
    """Gathered rows and a caller-given amax (in place and separate)."""
    x = edge_tensor(64, 128, seed=4)
    ri = np.array([5, 0, 63, 7, 7, 12, 1, 40, 33, 2], np.int32)
    c, s, g = api.quant_nvfp4_sr(dev(x), row_index=dev(torch.from_numpy(ri)), seed=13)
    oc, osf, og = ora.quant_nvfp4_sr(bits(x), row_index=ri, seed=13)
    assert np.float32(g.item()) == np.float32(og)
    assert_codes_equal(host_u8(c), oc, "nvfp4 sr gather codes")
    assert_codes_equal(sf_canonical(ora, s, 10, 8), osf, "nvfp4 sr gather sf")
    am = dev(torch.tensor([3.5], dtype=torch.float32))
    c, s, g = api.quant_nvfp4_sr(dev(x), amax_in=am, seed=14)
    oc, osf, og = ora.quant_nvfp4_sr(bits(x), amax_in=3.5, seed=14)
    assert np.float32(g.item()) == np.float32(og)
    assert_codes_equal(host_u8(c), oc, "nvfp4 sr amax codes")
    gs = dev(torch.tensor([3.5], dtype=torch.float32))
    c2 = torch.empty(64, 64, dtype=torch.uint8, device="cuda")
    s2 = torch.zeros(bsq.bsq_sf_bytes(64, 8), dtype=torch.uint8, device="cuda")
    api.quant_nvfp4_sr(dev(x), amax_in=gs, seed=14, out=(c2, s2, gs))
    assert np.float32(gs.item()) == np.float32(og)
    assert_codes_equal(host_u8(c2), oc, "nvfp4 sr in-place amax codes")


def test_nvfp4_sr_workload_rows(ora):
    """The first 1024 rows of the RHT linear's activation A (1x16) and of
    its weight W (16x16), at K = 4096."""
    A, Wt, seed = W.nvfp4_linear_rht()
    mask = bsq.bsq_rht_sign_mask(seed)
    for t, two_d in ((A[:1024], False), (Wt[:1024], True)):
        c, s, g = api.quant_nvfp4_sr(dev(t), block_2d=two_d, rht_mask=mask, seed=2, stream_id=1)
        oc, osf, og = ora.quant_nvfp4_sr(bits(t), block_2d=two_d, rht_mask=mask, seed=2, stream_id=1)
        assert np.float32(g.item()) == np.float32(og)
        assert_codes_equal(host_u8(c), oc, f"nvfp4 sr 2d={two_d} codes")
        assert_codes_equal(sf_canonical(ora, s, 1024, 256), osf, f"nvfp4 sr 2d={two_d} sf")


def test_nvfp4_given_amax_and_zero_tensor(ora):
    x = edge_tensor(64, 128, seed=5)
    _nvfp4_check(ora, x, amax_in=float(x.float().abs().max()) * 2.0, what="given amax")
    _nvfp4_check(ora, torch.zeros(32, 64, dtype=torch.bfloat16), what="zeros")
    _nvfp4_check(ora, torch.zeros(32, 64, dtype=torch.bfloat16), block_2d=True, what="zeros 2d")


def test_nvfp4_moe_gather_groups_parity(ora):
    """MoE activations: gather by routing, Four Over Six, per-expert SF rows
    padded to 128 (small version of the MoE workload's shapes)."""
    moe = W.moe_forward(T=512, H=256, E=8, F=128, weights=False)
    _nvfp4_check(ora, moe.X, fos=True, row_index=moe.row_index,
                 groups=(moe.row_offsets, moe.sf_row_offsets), what="moe gather")


@pytest.mark.parametrize("fos,rht,given", [(True, None, False), (False, 0x9A3C, False), (True, 0x0F1E, True)])
def test_nvfp4_gather_by_source_rows(ora, fos, rht, given):
    """bsq_quant_nvfp4_gather (each source row quantized once, the results
    moved to the gathered rows) gives the oracle's bytes for the gathered
    rows, and the same bytes as bsq_quant_nvfp4 with the row index."""
    moe = W.moe_forward(T=512, H=256, E=8, F=128, weights=False)
    X = moe.X
    ri, offs, sfo = moe.row_index, moe.row_offsets, moe.sf_row_offsets
    K = X.shape[1]
    groups = (dev(torch.from_numpy(offs)), dev(torch.from_numpy(sfo)), int(sfo[-1]))
    am_val = float(ora.amax(bits(X), rht_mask=rht, row_index=ri)) * 1.25 if given else None
    am = None if am_val is None else dev(torch.tensor([am_val], dtype=torch.float32))
    xd, rid = dev(X), dev(torch.from_numpy(ri))
    c, s_, g = api.quant_nvfp4_gather(xd, rid, four_over_six=fos, rht_mask=rht, groups=groups, amax_in=am)
    c2, s2, g2 = api.quant_nvfp4(xd, four_over_six=fos, rht_mask=rht, row_index=rid, groups=groups, amax_in=am)
    assert bsq.bsq_check() == 0
    assert torch.equal(c, c2) and torch.equal(s_, s2) and g.item() == g2.item()
    oc, osf, og = ora.quant_nvfp4(bits(X), four_over_six=fos, rht_mask=rht, row_index=ri, amax_in=am_val)
    assert np.float32(g.item()) == np.float32(og)
    assert_codes_equal(host_u8(c), oc, "gather codes")
    can = ora.sf_unswizzle(host_u8(s_), int(sfo[-1]), K // 16)
    for e in range(len(offs) - 1):
        assert_codes_equal(can[sfo[e]:sfo[e] + offs[e + 1] - offs[e]], osf[offs[e]:offs[e + 1]], f"gather sf {e}")


def test_amax_parity(ora):
    x = edge_tensor(96, 160, seed=11)
    xd = dev(x)
    for rht in (None, 0xBEEF):
        for ri in (None, np.array([5, 0, 95, 5, 17], np.int32)):
            a = api.amax(xd, rht_mask=rht, row_index=None if ri is None else dev(torch.from_numpy(ri)))
            want = ora.amax(bits(x), rht_mask=rht, row_index=ri)
            assert np.float32(a.item()) == np.float32(want)


# ------------------------------------------------------------------ RHT
@pytest.mark.parametrize("M,K", [(1, 16), (64, 256), (33, 4096)])
def test_rht_bf16_parity(ora, M, K):
    x = edge_tensor(M, K, seed=M)
    mask = ora.rht_sign_mask(2)
    y = api.rht(dev(x), mask)
    assert_codes_equal(y.cpu().view(torch.int16).numpy().view(np.uint16), ora.rht_bf16(bits(x), mask), "rht")


# ------------------------------------------------------------------ MXFP8
def mx_edge_tensor(M, K, seed=0):
    g = torch.Generator().manual_seed(seed)
    x = W.student_t((M, K), 3, g)
    w = min(K, 32)
    x[0, :w] = 0.0
    if M > 1:
        x[1, :w] = torch.linspace(-1, 1, w) * 1e-38  # subnormal range, includes -0 outcomes
    if M > 2:
        x[2, :w] = 480.0  # (448, 512) x 2^0 saturates
        x[2, min(5, w - 1)] = 300.0
    if M > 3:
        x[3, :w] = -1e-3
    return x.to(torch.bfloat16)


@pytest.mark.parametrize("sr", [False, True])
@pytest.mark.parametrize("M,K", [(64, 128), (3, 32), (100, 96), (256, 4096), (48, 1024), (33, 3072)])
def test_mxfp8_rowwise_parity(ora, M, K, sr):
    x = mx_edge_tensor(M, K, seed=M * 3 + K)
    c, s = api.quant_mxfp8(dev(x), sr=sr, seed=1, stream_id=0)
    oc, osf = ora.quant_mxfp8(bits(x), sr=sr, seed=1, stream_id=0)
    assert_codes_equal(host_u8(c), oc, "mx row codes")
    assert_codes_equal(sf_canonical(ora, s, M, K // 32), osf, "mx row sf")


@pytest.mark.parametrize("sr", [False, True])
@pytest.mark.parametrize("M,K", [(128, 64), (32, 8), (96, 200), (512, 256), (160, 40), (64, 1000), (2048, 72)])
def test_mxfp8_colwise_parity(ora, M, K, sr):
    x = mx_edge_tensor(M, K, seed=M + 5 * K)
    c, s = api.quant_mxfp8(dev(x), colwise=True, sr=sr, seed=4, stream_id=3)
    oc, osf = ora.quant_mxfp8(bits(x), colwise=True, sr=sr, seed=4, stream_id=3)
    assert_codes_equal(host_u8(c), oc, "mx col codes")
    assert_codes_equal(sf_canonical(ora, s, K, M // 32), osf, "mx col sf")


@pytest.mark.parametrize("sr", [False, True])
@pytest.mark.parametrize("M,K", [(128, 64), (32, 32), (96, 160), (256, 512), (64, 1056)])
def test_requant_transpose_parity(ora, M, K, sr):
    x = mx_edge_tensor(M, K, seed=M + K)
    oc, osf = ora.quant_mxfp8(bits(x), sr=True, seed=1, stream_id=0)
    # the oracle's row-wise output is the input of both sides
    codes = dev(torch.from_numpy(oc))
    sf = dev(torch.from_numpy(ora.sf_swizzle(osf)))
    cc, sc = api.requant_transpose(codes, sf, sr=sr, seed=1, stream_id=1)
    wc, ws = ora.requant_transpose(oc, osf, sr=sr, seed=1, stream_id=1)
    assert_codes_equal(host_u8(cc), wc, "requant codes")
    assert_codes_equal(sf_canonical(ora, sc, K, M // 32), ws, "requant sf")


@pytest.mark.parametrize("sr", [False, True])
@pytest.mark.parametrize("M,K", [(64, 128), (3, 32), (100, 96), (256, 4096), (33, 3072)])
def test_mxfp4_rowwise_parity(ora, M, K, sr):
    """MXFP4 (E2M1 in blocks of 32, E8M0 scale): edge tensors with zero,
    subnormal-range, saturating and small negative blocks."""
    x = mx_edge_tensor(M, K, seed=M * 7 + K)
    c, s = api.quant_mxfp4(dev(x), sr=sr, seed=2, stream_id=5)
    oc, osf = ora.quant_mxfp4(bits(x), sr=sr, seed=2, stream_id=5)
    assert_codes_equal(host_u8(c), oc, "mxfp4 codes")
    assert_codes_equal(sf_canonical(ora, s, M, K // 32), osf, "mxfp4 sf")


def test_mxfp4_strided_rows_parity(ora):
    """A row stride larger than K (a column slice of a wider tensor)."""
    x = mx_edge_tensor(40, 320, seed=5)
    xd = dev(x)[:, :256]
    c, s = api.quant_mxfp4(xd, sr=True, seed=8)
    oc, osf = ora.quant_mxfp4(bits(x[:, :256].contiguous()), sr=True, seed=8)
    assert_codes_equal(host_u8(c), oc, "mxfp4 strided codes")
    assert_codes_equal(sf_canonical(ora, s, 40, 8), osf, "mxfp4 strided sf")


def test_mxfp4_workload_full_size(ora):
    """The Student-t 4096x4096 workload at full size, RNE and SR."""
    x = W.mxfp8_requant()
    xb = bits(x)
    xd = dev(x)
    for sr in (False, True):
        c, s = api.quant_mxfp4(xd, sr=sr, seed=1)
        oc, osf = ora.quant_mxfp4(xb, sr=sr, seed=1)
        assert_codes_equal(host_u8(c), oc, f"mxfp4 sr={sr} codes")
        assert_codes_equal(sf_canonical(ora, s, 4096, 128), osf, f"mxfp4 sr={sr} sf")


def test_mxfp8_requant_workload_full_size(ora):
    """The Student-t 4096x4096 workload at full size: RNE, SR, then the
    requant-transpose of the SR output -- all bit-exact."""
    x = W.mxfp8_requant()
    xb = bits(x)
    xd = dev(x)
    for sr in (False, True):
        c, s = api.quant_mxfp8(xd, sr=sr, seed=1, stream_id=0)
        oc, osf = ora.quant_mxfp8(xb, sr=sr, seed=1, stream_id=0)
        assert_codes_equal(host_u8(c), oc, f"cfg1 sr={sr} codes")
        assert_codes_equal(sf_canonical(ora, s, 4096, 128), osf, f"cfg1 sr={sr} sf")
    cc, sc = api.requant_transpose(c, s, sr=True, seed=1, stream_id=1)
    wc, ws = ora.requant_transpose(oc, osf, sr=True, seed=1, stream_id=1)
    assert_codes_equal(host_u8(cc), wc, "cfg1 requant codes")
    assert_codes_equal(sf_canonical(ora, sc, 4096, 128), ws, "cfg1 requant sf")


# ------------------------------------------------------------------ errors
@pytest.mark.parametrize("sr", [False, True])
@pytest.mark.parametrize("M,K", [(32, 32), (64, 96), (256, 512), (96, 4096)])
def test_mxfp8_rowcol_parity(ora, M, K, sr):
    """One pass, both orientations: byte-identical to the row-wise (stream 3)
    and column-wise (stream 5) quantizations."""
    x = W.mxfp8_requant(M=M, K=K, seed=M + K)
    x[0, :32] = 0.0
    cr, sr_, cc, sc = api.quant_mxfp8_rowcol(dev(x), sr=sr, seed=9, stream_id_row=3, stream_id_col=5)
    assert bsq.bsq_check() == 0
    wr = ora.quant_mxfp8(bits(x), sr=sr, seed=9, stream_id=3)
    wc = ora.quant_mxfp8(bits(x), colwise=True, sr=sr, seed=9, stream_id=5)
    assert_codes_equal(host_u8(cr), wr[0], "rowcol: row codes")
    assert_codes_equal(sf_canonical(ora, sr_, M, K // 32), wr[1], "rowcol: row sf")
    assert_codes_equal(host_u8(cc), wc[0], "rowcol: col codes")
    assert_codes_equal(sf_canonical(ora, sc, K, M // 32), wc[1], "rowcol: col sf")


@pytest.mark.parametrize("sr", [False, True])
@pytest.mark.parametrize("R,C,two_d", [(32, 16, True), (64, 96, True), (256, 512, True), (96, 4096, False)])
def test_requant_nvfp4_mxfp8_parity(ora, R, C, two_d, sr):
    """Saved NVFP4 -> dequantize -> transpose -> MXFP8: the oracle's NVFP4
    tensor uploaded, byte-identical output."""
    x = W.nvfp4_linear_rht(M=R, N=16, K=C, seed=R + C)[0]
    q = ora.quant_nvfp4(bits(x), block_2d=two_d)
    codes = dev(torch.from_numpy(q[0]))
    sf = dev(torch.from_numpy(ora.sf_swizzle(q[1])))
    gs = dev(torch.tensor([q[2]], dtype=torch.float32))
    cc, sc = api.requant_nvfp4_mxfp8(codes, sf, gs, sr=sr, seed=11, stream_id=2)
    assert bsq.bsq_check() == 0
    want = ora.requant_nvfp4_mxfp8(*q, sr=sr, seed=11, stream_id=2)
    assert_codes_equal(host_u8(cc), want[0], "nvfp4->mxfp8 codes")
    assert_codes_equal(sf_canonical(ora, sc, C, R // 32), want[1], "nvfp4->mxfp8 sf")


def test_invalid_arguments_launch_nothing():
    x = torch.zeros(16, 24, dtype=torch.bfloat16, device="cuda")
    codes = torch.empty(16, 12, dtype=torch.uint8, device="cuda")
    sf = torch.empty(4096, dtype=torch.uint8, device="cuda")
    gs = torch.empty(1, dtype=torch.float32, device="cuda")
    with pytest.raises(bsq.BsqError) as e:
        bsq.bsq_quant_nvfp4(x, 16, 24, 24, 0, 0, 0, 0, None, 0, None, None, None, gs, codes, sf)
    assert e.value.status == bsq.BSQ_ERR_INVALID
    with pytest.raises(bsq.BsqError) as e:
        bsq.bsq_quant_nvfp4(x, 16, 16, 24, 1, 1, 0, 0, None, 0, None, None, None, gs, codes, sf)
    assert e.value.status == bsq.BSQ_ERR_INVALID
    with pytest.raises(bsq.BsqError) as e:  # MXFP4 blocks are 32 wide
        bsq.bsq_quant_mxfp4(x, 16, 24, 24, bsq.BSQ_RNE, 0, 0, codes, sf)
    assert e.value.status == bsq.BSQ_ERR_INVALID
    with pytest.raises(bsq.BsqError) as e:  # unknown rounding mode
        bsq.bsq_quant_mxfp4(x, 16, 0, 24, 7, 0, 0, codes, sf)
    assert e.value.status == bsq.BSQ_ERR_INVALID
    assert bsq.bsq_check() == bsq.BSQ_OK


def test_bounded_wait_times_out_and_context_survives():
    """A device wait on a barrier nobody arrives at runs out (short limit),
    reports BSQ_ERR_TIMEOUT through bsq_check, and the context stays usable."""
    bsq.bsq_debug_timeout_probe(50_000_000)  # 50 ms
    assert bsq.bsq_check() == bsq.BSQ_ERR_TIMEOUT
    assert bsq.bsq_check() == bsq.BSQ_OK  # the word was cleared
    y = torch.ones(4, device="cuda") * 2
    assert float(y.sum()) == 8.0
