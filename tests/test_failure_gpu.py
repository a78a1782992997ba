"""Failure detection on the GPU without a fault: the GEMM's pipeline waits are
bounded, and a wait that runs out is reported through the device error word
while the context stays usable.  The stall comes from a testing flag with which
the producer withholds one K stage (nothing is in flight for it), so the MMA
issuer's bounded wait runs out; every other role then gives up on its own
bounded waits, drains what it issued and frees its tensor memory."""
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


@pytest.mark.parametrize("m", [8, 40, 300], ids=["decode_T8", "decode_T64", "pair"])
def test_gemm_wait_timeout_is_reported_and_the_context_stays_usable(nv, m):
    import torch
    n, k = 392, 1344
    xb, wb, off = W.random_case(70 + m, m, n, k, seg_rows=[128, 264])
    x = to_cuda_bf16(xb)
    pw = nv.pack_weight(to_cuda_bf16(wb), off)
    qx, sfx, sx = nv.quantize_act(x)
    torch.cuda.synchronize()
    assert nv.get_device_error() == nv.OK
    nv.set_wait_timeout_ns(2_000_000)                  # 2 ms per wait
    try:
        nv.gemm(qx, sfx, sx, m, pw, flags=nv.FLAG_F32_OUT | nv.FLAG_TEST_STALL)
        assert nv.get_device_error() == nv.ERR_TIMEOUT
        assert nv.get_device_error() == nv.OK          # read and cleared
    finally:
        nv.set_wait_timeout_ns(2_000_000_000)
    # The same context computes the right answer afterwards.
    y = nv.gemm(qx, sfx, sx, m, pw, flags=nv.FLAG_F32_OUT)
    torch.cuda.synchronize()
    assert nv.get_device_error() == nv.OK
    ref = oracle.linear_reference(xb, wb, off)
    assert_gemm_close(y.cpu().numpy(), ref["y"], bf16=False)


def test_pair_gemm_late_stall_drains_and_the_context_stays_usable(nv):
    """The CTA-pair kernel withholds the last K stage of each pair's second
    output tile, after the first tile was stored: the MMA issuer's wait runs
    out, the pair accounts for the copies of every ring slot and waits for
    those in flight before it releases its memory, and the same context then
    computes the right answer.  600 x 7680 gives 90 output tiles over the 74
    pairs, so some pairs have a second tile."""
    import torch
    m, n, k = 600, 7680, 1344
    xb, wb, off = W.random_case(77, m, n, k, seg_rows=[3840, 3840])
    x = to_cuda_bf16(xb)
    pw = nv.pack_weight(to_cuda_bf16(wb), off)
    qx, sfx, sx = nv.quantize_act(x)
    torch.cuda.synchronize()
    assert nv.get_device_error() == nv.OK
    nv.set_wait_timeout_ns(2_000_000)
    try:
        for _ in range(2):                              # twice: the abort path leaves nothing behind
            nv.gemm(qx, sfx, sx, m, pw, flags=nv.FLAG_F32_OUT | nv.FLAG_TEST_STALL_LATE)
            assert nv.get_device_error() == nv.ERR_TIMEOUT
            assert nv.get_device_error() == nv.OK
    finally:
        nv.set_wait_timeout_ns(2_000_000_000)
    y = nv.gemm(qx, sfx, sx, m, pw, flags=nv.FLAG_F32_OUT)
    torch.cuda.synchronize()
    assert nv.get_device_error() == nv.OK
    ref = oracle.linear_reference(xb, wb, off)
    assert_gemm_close(y.cpu().numpy(), ref["y"], bf16=False)


@pytest.mark.parametrize("m", [8, 40], ids=["decode_T8", "decode_T64"])
def test_decode_gemm_late_stall_is_reported(nv, m):
    """The decode kernel withholding its last K stage: reported as a timeout,
    and the next call is correct."""
    import torch
    n, k = 392, 1344
    xb, wb, off = W.random_case(78 + m, m, n, k, seg_rows=[128, 264])
    x = to_cuda_bf16(xb)
    pw = nv.pack_weight(to_cuda_bf16(wb), off)
    qx, sfx, sx = nv.quantize_act(x)
    torch.cuda.synchronize()
    nv.set_wait_timeout_ns(2_000_000)
    try:
        nv.gemm(qx, sfx, sx, m, pw, flags=nv.FLAG_F32_OUT | nv.FLAG_TEST_STALL_LATE)
        assert nv.get_device_error() == nv.ERR_TIMEOUT
    finally:
        nv.set_wait_timeout_ns(2_000_000_000)
    y = nv.gemm(qx, sfx, sx, m, pw, flags=nv.FLAG_F32_OUT)
    torch.cuda.synchronize()
    assert nv.get_device_error() == nv.OK
    ref = oracle.linear_reference(xb, wb, off)
    assert_gemm_close(y.cpu().numpy(), ref["y"], bf16=False)



@pytest.mark.parametrize("late", [False, True], ids=["second_stage", "last_stage"])
def test_split_k_decode_stall_is_reported_and_the_context_stays_usable(nv, late):
    """The split-K decode GEMM (8 tokens, N = 512: one cluster of four CTAs,
    each on a quarter of K) withholds a stage in every CTA: the waits run out,
    the three CTAs still push their (zero) partial sums so that CTA 0's slot
    barrier completes, and the same context then computes the right answer."""
    import torch
    m, n, k = 8, 512, 2048
    xb, wb, off = W.random_case(81, m, n, k)
    x = to_cuda_bf16(xb)
    pw = nv.pack_weight(to_cuda_bf16(wb), off)
    qx, sfx, sx = nv.quantize_act(x)
    torch.cuda.synchronize()
    assert nv.get_device_error() == nv.OK
    stall = nv.FLAG_TEST_STALL_LATE if late else nv.FLAG_TEST_STALL
    nv.set_wait_timeout_ns(2_000_000)
    try:
        for _ in range(2):
            nv.gemm(qx, sfx, sx, m, pw, flags=nv.FLAG_F32_OUT | stall)
            assert nv.get_device_error() == nv.ERR_TIMEOUT
            assert nv.get_device_error() == nv.OK
    finally:
        nv.set_wait_timeout_ns(2_000_000_000)
    y = nv.gemm(qx, sfx, sx, m, pw, flags=nv.FLAG_F32_OUT)
    torch.cuda.synchronize()
    assert nv.get_device_error() == nv.OK
    ref = oracle.linear_reference(xb, wb, off)
    assert_gemm_close(y.cpu().numpy(), ref["y"], bf16=False)
