"""The expert-parallel exchange (fp8_math_b200.ep) on two gloo ranks on the
CPU: dispatch in NVFP4 with one all-reduced global scale, the experts'
outputs back in RHT + S2F6, combined per token.  The device work is done by
a CPU stand-in codec built on the oracle (test infrastructure; the library's
codec is the GPU one), so what is checked is the exchange itself: every
rank's combined output equals, bit for bit, the same layer computed in one
process over all ranks' tokens (no row may be lost, duplicated, misrouted,
reordered within a token, or quantized with another scale)."""
import os
import socket
import sys

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

WORLD, T, H, E, K_TOP = 2, 24, 64, 4, 2
MASK = 0x6B19


def _bits(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def _from_bits(b):
    return torch.from_numpy(np.ascontiguousarray(b).view(np.int16)).view(torch.bfloat16)


class OracleCodec:
    """CPU stand-in for the GPU codec (same interface), on the oracle."""

    def __init__(self):
        from oracle import oracle as ora
        self.ora = ora

    @staticmethod
    def index(a, device):
        return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32))

    def amax(self, x, rows):
        return torch.tensor([self.ora.amax(_bits(x), row_index=rows.numpy())], dtype=torch.float32)

    def quant_nvfp4_rows(self, x, rows, amax, four_over_six):
        c, s, g = self.ora.quant_nvfp4(_bits(x), four_over_six=four_over_six, row_index=rows.numpy(),
                                       amax_in=float(amax.item()))
        return torch.from_numpy(c), torch.from_numpy(s), torch.tensor([g], dtype=torch.float32)

    def gather_rows(self, src, index):
        return src[index.long()]

    def quant_s2f6(self, y, rht_mask):
        c, s = self.ora.quant_s2f6(_bits(y), rht_mask=rht_mask)
        return torch.from_numpy(c), torch.from_numpy(s)

    def combine_s2f6(self, codes, sf, token_offsets, rows, weights, rht_mask):
        out = self.ora.combine_s2f6(codes.numpy(), sf.numpy(), token_offsets.numpy(), rows.numpy(),
                                    weights.numpy(), rht_mask)
        return _from_bits(out)


def _problem(rank):
    g = torch.Generator().manual_seed(100 + rank)
    x = torch.randn(T, H, generator=g).to(torch.bfloat16)
    logits = torch.randn(T, E, generator=g)
    probs = torch.softmax(logits, dim=1)
    w, ex = torch.topk(probs, K_TOP, dim=1)
    return x, ex.numpy(), w.numpy().astype(np.float32)


def _experts():
    g = torch.Generator().manual_seed(7)
    return [(torch.randn(H, H, generator=g) * 0.1).to(torch.bfloat16) for _ in range(E)]


def _expert_rows(ora, codes, sf, gs, Wb):
    """Expert output rows: decoded NVFP4 rows times W^T, binary64 per element
    (the oracle's scalar loop), rounded to bf16."""
    a = ora.dequant(0, codes, sf, gs)
    Wq = ora.quant_nvfp4(_bits(Wb), block_2d=True)
    Cm, _ = ora.gemm_f64(a, ora.dequant(0, *Wq))
    return torch.from_numpy(Cm.astype(np.float32)).to(torch.bfloat16)


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        from fp8_math_b200 import ep
        codec = OracleCodec()
        x, ex, w = _problem(rank)
        plan = ep.make_plan(ex, w, E)
        codes, sf_rows, gs = ep.dispatch(x, plan, codec)
        epr = E // world
        ys = []
        for le in range(epr):
            r0, r1 = int(plan.expert_offsets[le]), int(plan.expert_offsets[le + 1])
            ys.append(_expert_rows(codec.ora, codes[r0:r1].numpy(), sf_rows[r0:r1].numpy(), float(gs.item()),
                                   _experts()[rank * epr + le]))
        y = torch.cat(ys) if ys else torch.zeros(0, H, dtype=torch.bfloat16)
        res = ep.combine(y, plan, codec, MASK)
        out[rank] = _bits(res).copy()
        dist.barrier()
    finally:
        dist.destroy_process_group()


def _reference():
    """The same layer in one process: all ranks' routed rows quantized with
    the global amax, each row through its expert, S2F6 and the combine, every
    token's rows in expert order."""
    from oracle import oracle as ora
    probs = [_problem(r) for r in range(WORLD)]
    rows_all = [np.repeat(np.arange(T), K_TOP) for _ in range(WORLD)]
    amax = max(ora.amax(_bits(p[0]), row_index=rows_all[i].astype(np.int32)) for i, p in enumerate(probs))
    Ws = _experts()
    outs = []
    for x, ex, w in probs:
        order = np.lexsort((np.repeat(np.arange(T), K_TOP), ex.reshape(-1)))   # by expert, then token
        toks, exps, wts = np.repeat(np.arange(T), K_TOP)[order], ex.reshape(-1)[order], w.reshape(-1)[order]
        c, s, g = ora.quant_nvfp4(_bits(x), four_over_six=True, row_index=toks.astype(np.int32), amax_in=amax)
        y = torch.cat([_expert_rows(ora, c[i:i + 1], s[i:i + 1], g, Ws[int(exps[i])]) for i in range(len(toks))])
        yc, ys = ora.quant_s2f6(_bits(y), rht_mask=MASK)
        by_tok = np.argsort(toks, kind="stable")
        off = np.zeros(T + 1, np.int32)
        off[1:] = np.cumsum(np.bincount(toks, minlength=T))
        outs.append(ora.combine_s2f6(yc, ys, off, by_tok.astype(np.int32), wts[by_tok].astype(np.float32), MASK))
    return outs


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_rank_dispatch_and_combine_match_one_process():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_rank_main, args=(WORLD, _free_port(), out), nprocs=WORLD, join=True,
                           start_method="spawn")
        res = dict(out)
    ref = _reference()
    for r in range(WORLD):
        assert np.array_equal(res[r], ref[r]), f"rank {r}"
