"""bsq_global_scale_noalloc: the NVFP4 global scale for callers that may not
call cudaMalloc (their device memory all belongs to a framework's pool
allocator, or they run on a latency-critical path where an allocation can
synchronize the device).  Its scratch is a file-scope device array shared by
every call on a device, so these tests call it several times in a row --
each call finds the partial maxima the previous one left behind -- and check
it against the allocating entry point bsq_quant_nvfp4 and against the
oracle's s_g = amax / 2688.  Collected last on purpose: a failure here
stops a -x run only after every other test has run."""
import numpy as np
import pytest
import torch

from fp8_math_b200 import api, bsq
from fp8_math_b200 import workloads as W
from gpu_util import bits, dev

pytestmark = pytest.mark.gpu


def _expect(ora, x, mask):
    amax = ora.amax(bits(x), rht_mask=mask)
    return np.float32(1.0) if amax == 0 else np.float32(np.float32(amax) / np.float32(2688.0))


def test_global_scale_noalloc_matches_quantize_entry_point(ora):
    A, Wt, seed = W.nvfp4_linear_rht(M=512, N=272, K=1024)
    mask = bsq.bsq_rht_sign_mask(seed)
    big = W.nvfp4_linear_rht(M=2048, N=16, K=4096)[0]       # 128 CTAs, then fewer again
    for x, rht in [(A, False), (Wt, True), (big, True), (A * 3, True), (Wt[:16], False)]:
        xd = dev(x)
        M, K = x.shape
        m = mask if rht else None
        _, _, gs_ref = api.quant_nvfp4(xd, rht_mask=m)
        gs = torch.full((1,), -1.0, device=xd.device)
        bsq.bsq_global_scale_noalloc(xd, M, K, K, rht, mask if rht else 0, gs)
        assert bsq.bsq_check() == bsq.BSQ_OK
        assert gs.item() == gs_ref.item()
        assert np.float32(gs.item()) == _expect(ora, x, m)


def test_global_scale_noalloc_strided_rows(ora):
    """A row stride larger than K (a column slice of a wider tensor)."""
    A = W.nvfp4_linear_rht(M=300, N=16, K=2048)[0]
    view = dev(A)[:, 512:1536]
    gs = torch.full((1,), -1.0, device=view.device)
    for _ in range(2):
        bsq.bsq_global_scale_noalloc(view, 300, 1024, 2048, False, 0, gs)
        assert bsq.bsq_check() == bsq.BSQ_OK
        assert np.float32(gs.item()) == _expect(ora, A[:, 512:1536].contiguous(), None)


def test_global_scale_noalloc_empty_invalid_and_oversize():
    gs = torch.full((1,), -1.0, device="cuda")
    x = torch.zeros(1, 64, dtype=torch.bfloat16, device="cuda")
    bsq.bsq_global_scale_noalloc(x, 0, 64, 64, False, 0, gs)   # M = 0: amax 0, s_g = 1
    assert gs.item() == 1.0
    with pytest.raises(bsq.BsqError):
        bsq.bsq_global_scale_noalloc(x, 4, 40, 40, False, 0, gs)   # K % 16 != 0
    # more than 4095 partial maxima: refused before any launch (x is never read)
    with pytest.raises(bsq.BsqError) as e:
        bsq.bsq_global_scale_noalloc(x, 65521, 4096, 4096, False, 0, gs)
    assert e.value.status == bsq.BSQ_ERR_UNSUPPORTED
    assert gs.item() == 1.0
