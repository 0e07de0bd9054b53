"""The MoE combine exchange's codec on the GPU against the oracle: RHT +
block-scaled S2F6 on the sender, weighted combine + inverse RHT on the
receiver (Thinking Machines page, section "Why communication became the
next bottleneck").  Every code, scale and output bit must match."""
import numpy as np
import pytest
import torch

from fp8_math_b200 import api, bsq
from fp8_math_b200 import workloads as W
from gpu_util import assert_codes_equal, bits, dev

pytestmark = pytest.mark.gpu


def _edge(M, K, seed):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(M, K, generator=g) * 3
    x[0, :32] = 0.0
    if M > 2:
        x[1, :64] = 1e-38            # subnormal-range values (bf16 keeps them)
        x[2, 32:64] = 2.0            # block maximum exactly at a power of two
    return x.to(torch.bfloat16)


@pytest.mark.parametrize("rht", [None, 0xC3A5])
@pytest.mark.parametrize("M,K", [(1, 32), (33, 96), (64, 4096), (300, 544)])
def test_s2f6_quant_parity(ora, M, K, rht):
    x = _edge(M, K, M + K)
    c, s = api.quant_s2f6(dev(x), rht_mask=rht)
    assert bsq.bsq_check() == bsq.BSQ_OK
    wc, ws = ora.quant_s2f6(bits(x), rht_mask=rht)
    assert_codes_equal(c.cpu().numpy(), wc, "s2f6 codes")
    assert_codes_equal(s.cpu().numpy(), ws, "s2f6 scales")


def _routing(T, E, k, seed):
    g = torch.Generator().manual_seed(seed)
    logits = torch.randn(T, E, generator=g)
    ri, offs, _ = W.route_topk(logits, k)
    probs = torch.softmax(logits, dim=1).numpy()
    # rows of each token, in routed-row order, with the token's routing weight
    order = np.argsort(ri, kind="stable")
    counts = np.bincount(ri, minlength=T)
    tok_off = np.zeros(T + 1, np.int32)
    tok_off[1:] = np.cumsum(counts)
    expert_of_row = np.searchsorted(offs, np.arange(len(ri)), side="right") - 1
    weights = probs[ri[order], expert_of_row[order]].astype(np.float32)
    return ri, tok_off, order.astype(np.int32), weights


@pytest.mark.parametrize("T,E,k,K", [(7, 4, 2, 64), (96, 8, 3, 512), (256, 16, 8, 1024)])
def test_s2f6_combine_parity(ora, T, E, k, K):
    ri, tok_off, rows, w = _routing(T, E, k, T + K)
    R = len(ri)
    y = _edge(R, K, 3 * T)
    mask = 0x5AC3
    c, s = api.quant_s2f6(dev(y), rht_mask=mask)
    out = api.combine_s2f6(c, s, dev(torch.from_numpy(tok_off)), dev(torch.from_numpy(rows)),
                           dev(torch.from_numpy(w)), mask)
    assert bsq.bsq_check() == bsq.BSQ_OK
    wc, ws = ora.quant_s2f6(bits(y), rht_mask=mask)
    want = ora.combine_s2f6(wc, ws, tok_off, rows, w, mask)
    assert_codes_equal(bits(out.cpu()), want, "combine output")


def test_s2f6_combine_moe_workload(ora):
    """The MoE workload's combine: 16384 tokens x 8 routed rows, hidden 4096
    (the down projection's output shape; its values a seeded stand-in drawn
    like the routed activations), every output bit."""
    ri, tok_off, rows, w = _routing(16384, 64, 8, 3)
    R, K = len(ri), 4096
    g = torch.Generator().manual_seed(33)
    y = (torch.randn(R, K, generator=g) * 0.05).to(torch.bfloat16)
    mask = bsq.bsq_rht_sign_mask(3)
    c, s = api.quant_s2f6(dev(y), rht_mask=mask)
    out = api.combine_s2f6(c, s, dev(torch.from_numpy(tok_off)), dev(torch.from_numpy(rows)),
                           dev(torch.from_numpy(w)), mask)
    assert bsq.bsq_check() == bsq.BSQ_OK
    T = ora.ncores()
    wc, ws = ora.quant_s2f6(bits(y), rht_mask=mask, threads=T)
    assert_codes_equal(c.cpu().numpy(), wc, "combine codes")
    want = ora.combine_s2f6(wc, ws, tok_off, rows, w, mask, threads=T)
    assert_codes_equal(bits(out.cpu()), want, "combine output")


def test_ep_exchange_on_one_gpu(ora):
    """The exchange with the library's GPU codec on a one-rank NCCL group:
    the dispatched rows are the oracle's NVFP4 quantization of the routed rows
    (every byte, in expert order); the grouped GEMM consumes them through the
    scale-row mover; the combine of expert outputs (the oracle's, rounded to
    bf16) equals the oracle's combine bit for bit."""
    import socket

    import torch.distributed as dist

    from fp8_math_b200 import ep

    with socket.socket() as so:
        so.bind(("127.0.0.1", 0))
        port = so.getsockname()[1]
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1)
    try:
        T, H, E, k = 64, 256, 4, 2
        g = torch.Generator().manual_seed(5)
        x = torch.randn(T, H, generator=g).to(torch.bfloat16)
        probs = torch.softmax(torch.randn(T, E, generator=g), dim=1)
        w, ex = torch.topk(probs, k, dim=1)
        plan = ep.make_plan(ex.numpy(), w.numpy().astype(np.float32), E, device="cuda")
        codec = ep.GpuCodec()
        codes, sf_rows, gs = ep.dispatch(dev(x), plan, codec)
        assert bsq.bsq_check() == bsq.BSQ_OK
        toks = plan.send_tokens[plan.recv_order]
        amax = ora.amax(bits(x), row_index=plan.send_tokens)
        qc, qs, qg = ora.quant_nvfp4(bits(x), four_over_six=True, row_index=toks, amax_in=amax)
        assert_codes_equal(codes.cpu().numpy(), qc, "dispatched codes")
        assert_codes_equal(sf_rows.cpu().numpy(), qs, "dispatched scale rows")
        assert np.float32(gs.item()) == np.float32(qg)
        # the grouped GEMM on the dispatched rows (scale rows moved into the GEMM's layout)
        offs = plan.expert_offsets.astype(np.int32)
        counts = np.diff(offs)
        sfo = np.zeros(E + 1, np.int32)
        sfo[1:] = np.cumsum((counts + 127) // 128 * 128)
        offs_d, sfo_d = dev(torch.from_numpy(offs)), dev(torch.from_numpy(sfo))
        sfA = torch.zeros(api.sf_bytes(int(sfo[-1]), H // 16), dtype=torch.uint8, device="cuda")
        bsq.bsq_sf_from_rows(sf_rows, int(offs[-1]), H // 16, E, offs_d, sfo_d, sfA)
        Wts = [(torch.randn(H, H, generator=g) * 0.05).to(torch.bfloat16) for _ in range(E)]
        qw = [ora.quant_nvfp4(bits(Wt), block_2d=True) for Wt in Wts]
        Bc = dev(torch.from_numpy(np.stack([q[0] for q in qw])))
        sB = dev(torch.from_numpy(np.concatenate([ora.sf_swizzle(q[1]) for q in qw])))
        gB = dev(torch.tensor([q[2] for q in qw], dtype=torch.float32))
        Y = api.grouped_gemm(0, offs_d, sfo_d, codes, sfA, Bc, sB, int(offs[-1]), H, H, gsA=gs, gsB=gB,
                             out_dtype=torch.bfloat16)
        assert bsq.bsq_check() == bsq.BSQ_OK
        from gpu_util import assert_gemm_close
        y_ora = []
        for e in range(E):
            r0, r1 = int(offs[e]), int(offs[e + 1])
            Cr, Ra = ora.gemm_f64(ora.dequant(0, qc[r0:r1], qs[r0:r1], qg), ora.dequant(0, *qw[e]))
            assert_gemm_close(Y[r0:r1].float().cpu().numpy().astype(np.float64), Cr, Ra, True, f"expert {e}")
            y_ora.append(torch.from_numpy(Cr.astype(np.float32)).to(torch.bfloat16))
        y_ora = torch.cat(y_ora)
        mask = 0x2E71
        out = ep.combine(dev(y_ora), plan, codec, mask)
        assert bsq.bsq_check() == bsq.BSQ_OK
        yc, ys = ora.quant_s2f6(bits(y_ora), rht_mask=mask)
        want = ora.combine_s2f6(yc, ys, plan.token_offsets, plan.token_rows, plan.token_weights, mask)
        assert_codes_equal(bits(out.cpu()), want, "combined output")
    finally:
        dist.destroy_process_group()
