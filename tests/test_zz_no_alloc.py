"""bsq_global_scale_noalloc (scratch in a file-scope device array, no
allocation) against the allocating entry point bsq_quant_nvfp4, two calls in
a row so that the second call finds the scratch the first one left behind,
and against the oracle's s_g = amax / 2688.  Collected last on purpose."""
import numpy as np
import pytest
import torch

from fp8_math_b200 import api, bsq
from fp8_math_b200 import workloads as W
from gpu_util import bits, dev

pytestmark = pytest.mark.gpu


def test_global_scale_noalloc_matches_quantize_entry_point(ora):
    A, Wt, seed = W.nvfp4_linear_rht(M=512, N=272, K=1024)
    mask = bsq.bsq_rht_sign_mask(seed)
    for x, rht in [(A, False), (Wt, True), (A * 3, True)]:   # two (and a third) calls in a row
        xd = dev(x)
        M, K = x.shape
        _, _, gs_ref = api.quant_nvfp4(xd, rht_mask=mask if rht else None)
        gs = torch.full((1,), -1.0, device=xd.device)
        bsq.bsq_global_scale_noalloc(xd, M, K, K, rht, mask if rht else 0, gs)
        assert bsq.bsq_check() == bsq.BSQ_OK
        assert gs.item() == gs_ref.item()
        amax = ora.amax(bits(x), rht_mask=mask if rht else None)
        expect = np.float32(1.0) if amax == 0 else np.float32(np.float32(amax) / np.float32(2688.0))
        assert np.float32(gs.item()) == expect


def test_global_scale_noalloc_empty_and_invalid():
    gs = torch.full((1,), -1.0, device="cuda")
    x = torch.zeros(1, 64, dtype=torch.bfloat16, device="cuda")
    bsq.bsq_global_scale_noalloc(x, 0, 64, 64, False, 0, gs)   # M = 0: amax 0, s_g = 1
    assert gs.item() == 1.0
    with pytest.raises(bsq.BsqError):
        bsq.bsq_global_scale_noalloc(x, 4, 40, 40, False, 0, gs)   # K % 16 != 0
