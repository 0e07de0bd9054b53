"""Seeded synthetic inputs for the five workloads (no quantization arithmetic).

This module only draws random tensors (torch CPU generator, so every machine
gets the same bits) and derives the MoE routing structure; the tests, the
bench and the smoke check pass its outputs to both the CUDA library and the
CPU oracle.  It holds none of the method's arithmetic.

Workloads (sizes as the pages' recipes give them):
  * ``nvfp4_linear_small`` -- A 128x256 N(0,1) with 1 % of columns x50, W
    256x256 N(0, 0.02); seed 0.
  * ``mxfp8_requant``     -- X 4096x4096 Student-t (nu = 3); seed 1.
  * ``nvfp4_linear_rht``  -- A 8192x4096 N(0,1) with 0.5 % of channels x100,
    W 14336x4096 N(0, 0.02); RHT sign seed 2.
  * ``moe_forward``       -- 16384 tokens, hidden 4096, 64 experts of ffn
    1536, top-8 routing from N(0,1) logits; seed 3.
  * ``mxfp8_backward``    -- dY 8192x14336 N(0, 1e-3), W 14336x4096
    N(0, 0.02), X 8192x4096 N(0,1); rollout A 64x4096 N(0,1); seed 4.

Draw order inside each generator is fixed (documented inline) so that a
change of order is a change of inputs.  Every generator takes size overrides
so that tests can draw the same recipe at oracle-friendly sizes.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return g


def _bf16(t: torch.Tensor) -> torch.Tensor:
    return t.to(torch.bfloat16).contiguous()


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> numpy uint16 bit patterns (same shape)."""
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def _outlier_columns(g, K: int, frac: float) -> torch.Tensor:
    count = int(round(frac * K))
    return torch.randperm(K, generator=g)[:count]


def nvfp4_linear_small(M=128, N=256, K=256, seed=0):
    """A [M,K] N(0,1) with round(1% K) columns scaled x50; W [N,K] N(0,0.02).
    Draw order: A, outlier columns, W."""
    g = _gen(seed)
    A = torch.randn(M, K, generator=g)
    cols = _outlier_columns(g, K, 0.01)
    A[:, cols] *= 50.0
    W = torch.randn(N, K, generator=g) * 0.02
    return _bf16(A), _bf16(W)


def student_t(shape, nu: int, g) -> torch.Tensor:
    """Student-t(nu) = Z / sqrt(chi2_nu / nu), chi2_nu a sum of nu squared normals."""
    z = torch.randn(*shape, generator=g)
    chi2 = torch.zeros(*shape)
    for _ in range(nu):
        chi2 += torch.randn(*shape, generator=g) ** 2
    return z / torch.sqrt(chi2 / nu)


def mxfp8_requant(M=4096, K=4096, seed=1):
    """X [M,K] Student-t(3).  Draw order: Z, then three chi components."""
    return _bf16(student_t((M, K), 3, _gen(seed)))


def nvfp4_linear_rht(M=8192, N=14336, K=4096, seed=2):
    """A [M,K] N(0,1) with round(0.5% K) channels x100; W [N,K] N(0,0.02).
    Returns (A, W, rht_seed).  Draw order: A, outlier columns, W."""
    g = _gen(seed)
    A = torch.randn(M, K, generator=g)
    cols = _outlier_columns(g, K, 0.005)
    A[:, cols] *= 100.0
    W = torch.randn(N, K, generator=g) * 0.02
    return _bf16(A), _bf16(W), seed


@dataclass
class MoeInputs:
    X: torch.Tensor            # [T, H] bf16 tokens
    W_up: torch.Tensor         # [E, F, H] bf16
    W_dn: torch.Tensor         # [E, H, F] bf16
    row_index: np.ndarray      # [T*topk] int32: token of each routed row, grouped by expert
    row_offsets: np.ndarray    # [E+1] int32: routed-row range of each expert
    sf_row_offsets: np.ndarray  # [E+1] int32: each expert's first scale-factor row (128-aligned)


def route_topk(logits: torch.Tensor, topk: int):
    """Top-k experts per token by (-logit, expert id) -- softmax is monotone, so
    the top-k of the softmax are the top-k logits.  Rows are grouped by expert
    (ascending), tokens ascending inside an expert."""
    T, E = logits.shape
    lg = logits.numpy().astype(np.float64)
    # lexsort: last key primary -> sort by -logit, ties by expert id
    order = np.lexsort((np.broadcast_to(np.arange(E), (T, E)), -lg), axis=1)[:, :topk]
    expert = order.reshape(-1)
    token = np.repeat(np.arange(T), topk)
    perm = np.lexsort((token, expert))
    row_index = token[perm].astype(np.int32)
    counts = np.bincount(expert, minlength=E)
    offs = np.zeros(E + 1, np.int32)
    offs[1:] = np.cumsum(counts)
    sf = np.zeros(E + 1, np.int32)
    sf[1:] = np.cumsum((counts + 127) // 128 * 128)
    return row_index, offs, sf


def moe_forward(T=16384, H=4096, E=64, F=1536, topk=8, seed=3, weights=True):
    """Draw order: logits [T,E], X [T,H], W_up [E,F,H], W_dn [E,H,F]."""
    g = _gen(seed)
    logits = torch.randn(T, E, generator=g)
    X = torch.randn(T, H, generator=g)
    if weights:
        W_up = torch.randn(E, F, H, generator=g) * 0.02
        W_dn = torch.randn(E, H, F, generator=g) * 0.02
    else:
        W_up = torch.zeros(0)
        W_dn = torch.zeros(0)
    ri, offs, sf = route_topk(logits, topk)
    return MoeInputs(_bf16(X), _bf16(W_up), _bf16(W_dn), ri, offs, sf)


def mxfp8_backward(M=8192, N=14336, K=4096, rollout_M=64, seed=4):
    """dY [M,N] N(0,1e-3), W [N,K] N(0,0.02), X [M,K] N(0,1), rollout A
    [rollout_M,K] N(0,1).  Draw order as listed."""
    g = _gen(seed)
    dY = torch.randn(M, N, generator=g) * 1e-3
    W = torch.randn(N, K, generator=g) * 0.02
    X = torch.randn(M, K, generator=g)
    A_roll = torch.randn(rollout_M, K, generator=g)
    return _bf16(dY), _bf16(W), _bf16(X), _bf16(A_roll)


def sample_points(M: int, N: int, n: int, seed: int = 1234):
    """Sampled (m, n) output positions: the four corners, the last row and
    column (ragged tails) and n uniform points."""
    rng = np.random.default_rng(seed)
    pm = list(rng.integers(0, M, n))
    pn = list(rng.integers(0, N, n))
    for m, nn in [(0, 0), (0, N - 1), (M - 1, 0), (M - 1, N - 1)]:
        pm.append(m)
        pn.append(nn)
    for j in range(0, N, max(1, N // 64)):
        pm.append(M - 1)
        pn.append(j)
    for i in range(0, M, max(1, M // 64)):
        pm.append(i)
        pn.append(N - 1)
    return np.array(pm, np.int64), np.array(pn, np.int64)


def ceil_div(a: int, b: int) -> int:
    return -(-a // b)


def round_up(a: int, b: int) -> int:
    return ceil_div(a, b) * b

