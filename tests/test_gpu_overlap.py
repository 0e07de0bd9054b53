"""Programmatic dependent launch (BSQ_KNOB_LAUNCH_OVERLAP) changes when a
kernel is scheduled, never what it reads: every kernel launched that way
waits for the previous kernel before touching memory.  A chain in which
each launch consumes the one before it -- RHT + amax + 1x16 NVFP4 quantize
of A, 16x16 quantize of W, the NVFP4 GEMM, then the amax + 1x16 quantize of
the GEMM's own bf16 output and a second GEMM on it -- runs back to back
with overlap on and with plain launches; every output is byte-identical.
The skinny split-K GEMM is chained the same way."""
import pytest
import torch

from fp8_math_b200 import api, bsq
from fp8_math_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _chain(A, Wd, mask, M, N, K):
    qa = api.quant_nvfp4(A, rht_mask=mask)
    qw = api.quant_nvfp4(Wd, block_2d=True, rht_mask=mask)
    C = api.gemm(0, qa[0], qa[1], qw[0], qw[1], M, N, K, gsA=qa[2], gsB=qw[2])
    qc = api.quant_nvfp4(C)                       # reads the GEMM's output
    qw2 = api.quant_nvfp4(Wd[:, :N].contiguous(), block_2d=True)
    D = api.gemm(0, qc[0], qc[1], qw2[0], qw2[1], M, Wd.shape[0], N, gsA=qc[2], gsB=qw2[2])
    return [*qa, *qw, C, *qc, D]


@pytest.mark.parametrize("M,N,K", [(512, 1024, 1024), (2048, 4096, 4096)])
def test_overlap_chain_matches_plain_launches(M, N, K):
    dev = torch.device("cuda")
    mask = bsq.bsq_rht_sign_mask(3)
    A0, W0 = W.nvfp4_linear_small(M=M, N=N, K=K, seed=5)
    A, Wd = A0.to(dev), W0.to(dev)
    outs = {}
    try:
        for overlap in (0, 1):
            assert bsq.bsq_debug_kernel_choice(bsq.BSQ_KNOB_LAUNCH_OVERLAP, overlap) == bsq.BSQ_OK
            for _ in range(3):                    # back to back: the later launches overlap the earlier ones
                got = _chain(A, Wd, mask, M, N, K)
            torch.cuda.synchronize()
            outs[overlap] = [t.clone() for t in got]
    finally:
        bsq.bsq_debug_kernel_choice(bsq.BSQ_KNOB_LAUNCH_OVERLAP, -1)
    for i, (x, y) in enumerate(zip(outs[0], outs[1])):
        assert torch.equal(x, y), f"output {i} differs with launch overlap"
    assert bsq.bsq_check() == bsq.BSQ_OK


@pytest.mark.parametrize("split", [1, 2, 4])
def test_overlap_skinny_chain(split):
    dev = torch.device("cuda")
    M, N, K = 64, 4096, 4096
    A0, W0 = W.nvfp4_linear_small(M=M, N=N, K=K, seed=9)
    A, Wd = A0.to(dev), W0.to(dev)
    outs = {}
    try:
        bsq.bsq_debug_kernel_choice(bsq.BSQ_KNOB_GEMM_SPLITK, split)
        for overlap in (0, 1):
            bsq.bsq_debug_kernel_choice(bsq.BSQ_KNOB_LAUNCH_OVERLAP, overlap)
            qw = api.quant_nvfp4(Wd, block_2d=True)
            for _ in range(3):
                qa = api.quant_nvfp4(A)
                C = api.gemm(0, qa[0], qa[1], qw[0], qw[1], M, N, K, gsA=qa[2], gsB=qw[2])
                qc = api.quant_nvfp4(C)
                D = api.gemm(0, qc[0], qc[1], qw[0], qw[1], M, N, N, gsA=qc[2], gsB=qw[2])
            torch.cuda.synchronize()
            outs[overlap] = [t.clone() for t in (*qa, C, *qc, D)]
    finally:
        bsq.bsq_debug_kernel_choice(bsq.BSQ_KNOB_LAUNCH_OVERLAP, -1)
        bsq.bsq_debug_kernel_choice(bsq.BSQ_KNOB_GEMM_SPLITK, -1)
    for i, (x, y) in enumerate(zip(outs[0], outs[1])):
        assert torch.equal(x, y), f"output {i} differs with launch overlap (split {split})"
    assert bsq.bsq_check() == bsq.BSQ_OK
