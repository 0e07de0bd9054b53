"""The linear step captured once in a CUDA graph and replayed on new inputs:
RHT + amax + 1x16 NVFP4 quantize of A, RHT + amax + 16x16 quantize of W,
NVFP4 GEMM with bf16 output.  Every replay's codes, scales, global scales
and GEMM output equal, byte for byte, the same calls made eagerly on the
same inputs (which the parity tests check against the oracle)."""
import pytest
import torch

from fp8_math_b200 import api, bsq
from fp8_math_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("M,N,K", [(128, 256, 256), (512, 1024, 1024), (2048, 4096, 2048)])
def test_linear_step_graph_replay_matches_eager(M, N, K):
    dev = torch.device("cuda")
    mask = bsq.bsq_rht_sign_mask(2)
    A0, W0 = W.nvfp4_linear_small(M=M, N=N, K=K, seed=11)
    A, Wd = A0.to(dev), W0.to(dev)
    qa = api.quant_nvfp4(A, rht_mask=mask)
    qw = api.quant_nvfp4(Wd, block_2d=True, rht_mask=mask)
    C = torch.empty(M, N, dtype=torch.bfloat16, device=dev)

    def step():
        api.quant_nvfp4(A, rht_mask=mask, out=qa)
        api.quant_nvfp4(Wd, block_2d=True, rht_mask=mask, out=qw)
        api.gemm(0, qa[0], qa[1], qw[0], qw[1], M, N, K, gsA=qa[2], gsB=qw[2], out=C)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step()  # every call once outside capture
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    outs = (*qa, *qw, C)
    for seed in (21, 22, 23):
        A1, W1 = W.nvfp4_linear_small(M=M, N=N, K=K, seed=seed)
        A.copy_(A1.to(dev))
        Wd.copy_(W1.to(dev))
        g.replay()
        torch.cuda.synchronize()
        got = [t.clone() for t in outs]
        step()
        torch.cuda.synchronize()
        for i, (x, y) in enumerate(zip(got, outs)):
            assert torch.equal(x, y), f"output {i} differs after replay (seed {seed})"
    assert bsq.bsq_check() == bsq.BSQ_OK
