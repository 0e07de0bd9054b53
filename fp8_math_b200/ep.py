"""Expert-parallel dispatch and combine of a mixture-of-experts layer.

The pages (Thinking Machines, section "Why communication became the next
bottleneck") describe the exchange: tokens are dispatched to the GPUs that
hold their selected experts with the values in NVFP4, and the experts'
outputs come back rotated by a random Hadamard transform and compressed to
block-scaled S2F6 (8.25 bits per value); the receiver combines them and
reverses the transform.  This module is the host side of that exchange over
``torch.distributed`` (NCCL between GPUs): the routing plan, the one
collective the NVFP4 scale needs (an all-reduce of the amax, so that every
rank quantizes with the same global scale), and the all-to-all of the byte
buffers.  All arithmetic and every byte move on the device run in libbsq's
kernels through a codec object; ``GpuCodec`` is the library's.

Layout.  Experts are split evenly: rank r holds experts
[r * E / W, (r + 1) * E / W).  A rank sends its routed rows ordered by
(destination rank, expert, token); the receiver regroups what arrives by
local expert (stable in arrival order) for the grouped GEMM, and the
combine sends each output row back to where its token came from.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch
import torch.distributed as dist


@dataclass
class EPPlan:
    rank: int
    world: int
    n_experts: int
    send_tokens: np.ndarray     # [R_send] local token of each row this rank sends (send order)
    send_counts: np.ndarray     # [world] rows sent to each rank
    recv_counts: np.ndarray     # [world] rows received from each rank
    recv_order: np.ndarray      # [R_recv] arrival index of each row in local-expert order
    expert_offsets: np.ndarray  # [E / W + 1] rows of each local expert in that order
    token_offsets: np.ndarray   # [T + 1] combine CSR: rows (send order) of each local token
    token_rows: np.ndarray      # [R_send]
    token_weights: np.ndarray   # [R_send] routing weight of each listed row

    @property
    def experts_per_rank(self) -> int:
        return self.n_experts // self.world


def _all_to_all_int(values: np.ndarray, send_counts, recv_counts, group, device):
    out = torch.empty(int(np.sum(recv_counts)), dtype=torch.int64, device=device)
    dist.all_to_all_single(out, torch.from_numpy(values.astype(np.int64)).to(device),
                           output_split_sizes=[int(c) for c in recv_counts],
                           input_split_sizes=[int(c) for c in send_counts], group=group)
    return out.cpu().numpy()


def make_plan(topk_experts: np.ndarray, topk_weights: np.ndarray, n_experts: int, group=None,
              device="cpu") -> EPPlan:
    """Routing of this rank's tokens (top-k expert ids [T, k] and weights
    [T, k]) -> the exchange plan.  Every rank calls it (it exchanges counts)."""
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    assert n_experts % world == 0
    epr = n_experts // world
    T, k = topk_experts.shape
    tok = np.repeat(np.arange(T), k)
    exp = topk_experts.reshape(-1).astype(np.int64)
    wgt = topk_weights.reshape(-1).astype(np.float32)
    dest = exp // epr
    order = np.lexsort((tok, exp, dest))            # by destination, then expert, then token
    send_tokens, send_exp, send_w = tok[order], exp[order], wgt[order]
    send_counts = np.bincount(dest[order], minlength=world).astype(np.int64)
    recv_counts = _all_to_all_int(send_counts, np.ones(world, np.int64), np.ones(world, np.int64), group, device)
    recv_exp = _all_to_all_int(send_exp, send_counts, recv_counts, group, device) - rank * epr
    recv_order = np.argsort(recv_exp, kind="stable")
    expert_offsets = np.zeros(epr + 1, np.int64)
    expert_offsets[1:] = np.cumsum(np.bincount(recv_exp, minlength=epr))
    # combine: each token's rows in send order
    by_tok = np.argsort(send_tokens, kind="stable")
    token_offsets = np.zeros(T + 1, np.int32)
    token_offsets[1:] = np.cumsum(np.bincount(send_tokens, minlength=T))
    return EPPlan(rank, world, n_experts, send_tokens.astype(np.int32), send_counts, recv_counts,
                  recv_order.astype(np.int32), expert_offsets.astype(np.int32), token_offsets,
                  by_tok.astype(np.int32), send_w[by_tok].astype(np.float32))


def _exchange(buf: torch.Tensor, send_counts, recv_counts, group) -> torch.Tensor:
    out = torch.empty((int(np.sum(recv_counts)),) + tuple(buf.shape[1:]), dtype=buf.dtype, device=buf.device)
    dist.all_to_all_single(out, buf.contiguous(), output_split_sizes=[int(c) for c in recv_counts],
                           input_split_sizes=[int(c) for c in send_counts], group=group)
    return out


def dispatch(x: torch.Tensor, plan: EPPlan, codec, group=None, four_over_six=True):
    """Sends this rank's routed rows of x [T, H] (bf16) in NVFP4.  Returns the
    rows received for the local experts, in local-expert order: (codes
    [R, H/2], scale rows [R, H/16], global scale [1]), where every rank used
    the same global scale (the all-reduced amax of all routed rows)."""
    rows = codec.index(plan.send_tokens, x.device)
    amax = codec.amax(x, rows)
    dist.all_reduce(amax, op=dist.ReduceOp.MAX, group=group)
    codes, sf_rows, gs = codec.quant_nvfp4_rows(x, rows, amax, four_over_six)
    rc = _exchange(codes, plan.send_counts, plan.recv_counts, group)
    rs = _exchange(sf_rows, plan.send_counts, plan.recv_counts, group)
    order = codec.index(plan.recv_order, x.device)
    return codec.gather_rows(rc, order), codec.gather_rows(rs, order), gs


def combine(y: torch.Tensor, plan: EPPlan, codec, rht_mask: int, group=None):
    """Sends the local experts' outputs y [R, H] (bf16, local-expert order)
    back in RHT + S2F6 and combines them per token.  Returns [T, H] bf16:
    each token's weighted sum of its experts' outputs."""
    back = np.empty_like(plan.recv_order)
    back[plan.recv_order] = np.arange(len(plan.recv_order), dtype=np.int32)
    y_arrival = codec.gather_rows(y, codec.index(back, y.device))
    codes, sf = codec.quant_s2f6(y_arrival, rht_mask)
    rc = _exchange(codes, plan.recv_counts, plan.send_counts, group)
    rs = _exchange(sf, plan.recv_counts, plan.send_counts, group)
    dev = y.device
    return codec.combine_s2f6(rc, rs, codec.index(plan.token_offsets, dev), codec.index(plan.token_rows, dev),
                              torch.from_numpy(plan.token_weights).to(dev), rht_mask)


class GpuCodec:
    """The exchange's device work in libbsq kernels."""

    def __init__(self):
        from . import api, bsq
        self.api, self.bsq = api, bsq

    @staticmethod
    def index(a: np.ndarray, device):
        return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(device)

    def amax(self, x, rows):
        return self.api.amax(x, row_index=rows)

    def quant_nvfp4_rows(self, x, rows, amax, four_over_six):
        R, H = rows.shape[0], x.shape[1]
        codes, sf, gs = self.api.quant_nvfp4(x, four_over_six=four_over_six, row_index=rows, amax_in=amax)
        sf_rows = torch.empty(R, H // 16, dtype=torch.uint8, device=x.device)
        self.bsq.bsq_sf_to_rows(sf, R, H // 16, sf_rows)
        return codes, sf_rows, gs

    def gather_rows(self, src, index):
        out = torch.empty((index.shape[0],) + tuple(src.shape[1:]), dtype=src.dtype, device=src.device)
        row_bytes = src[0].numel() * src.element_size() if src.shape[0] else 0
        self.bsq.bsq_gather_rows(src, row_bytes, index, index.shape[0], out)
        return out

    def quant_s2f6(self, y, rht_mask):
        return self.api.quant_s2f6(y, rht_mask=rht_mask)

    def combine_s2f6(self, codes, sf, token_offsets, rows, weights, rht_mask):
        return self.api.combine_s2f6(codes, sf, token_offsets, rows, weights, rht_mask)
