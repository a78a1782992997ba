"""The no-allocation variant of the fused layer.

Some callers cannot allocate device memory: a plugin hosted by a runtime that
owns all device memory and hands out no allocator, or a latency-critical path
where cudaMalloc, which may synchronize the device, is not acceptable.  For them
nvfp4_linear_fused_noalloc keeps its scratch in a static device array of the
library instead of a caller workspace.  This test calls it through the C ABI
twice in a row (the second call reuses the scratch the first one left behind)
and checks each result against the workspace entry point nvfp4_linear_fused on
the same inputs, and the fp32 result against the CPU oracle as well.  It runs last so that a failure here leaves every other test
already run; it passes alone in a fresh process as well as after the others.
"""
import numpy as np
import pytest

import oracle
from nvfp4_w4a4_block_b200 import workloads as W

from _helpers import assert_gemm_close, to_cuda_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nv():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import nvfp4_w4a4_block_b200 as nv
    nv.lib()
    return nv


def test_noalloc_matches_workspace_entry_on_two_calls_in_a_row(nv):
    import torch
    cases = [(32, 512, 1024, [256, 256]),      # decode-sized: swapped decode kernel
             (200, 384, 640, [128, 256])]      # more tokens: CTA-pair kernel
    for seed, (m, n, k, segs) in enumerate(cases):
        xb, wb, off = W.random_case(40 + seed, m, n, k, seg_rows=segs)
        x = to_cuda_bf16(xb)
        pw = nv.pack_weight(to_cuda_bf16(wb), off)
        expect = oracle.linear_reference(xb, wb, off)["y"]
        for flags in (nv.FLAG_F32_OUT, 0):
            ref = nv.linear_fused(x, pw, flags=flags)
            got = nv.linear_fused_noalloc(x, pw, flags=flags)
            torch.cuda.synchronize()
            assert nv.get_device_error() == nv.OK
            r = ref.float().cpu().numpy().astype(np.float64)
            g = got.float().cpu().numpy().astype(np.float64)
            assert_gemm_close(g, r, bf16=(flags == 0))
            assert torch.equal(got, ref)          # same kernels, same inputs: identical bits
            assert_gemm_close(g, expect, bf16=(flags == 0))


def test_noalloc_rejects_problems_beyond_its_scratch(nv):
    import torch
    k = 5120
    m = 2896                                              # one token beyond the limit at K = 5120
    pw = nv.pack_weight(to_cuda_bf16(W.random_case(50, 1, 64, k)[1]))
    x = torch.zeros((m, k), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(nv.NVFP4Error) as err:
        nv.linear_fused_noalloc(x, pw)
    assert err.value.status == nv.ERR_SCRATCH_LIMIT
    # the largest problem that fits, and a small one, still work afterwards
    for rows in (m - 1, 8):
        y = nv.linear_fused_noalloc(x[:rows], pw)
        torch.cuda.synchronize()
        assert nv.get_device_error() == nv.OK
        assert y.shape == (rows, 64) and not (y.float() != 0).any()      # zero activations give zeros
