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
