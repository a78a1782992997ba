"""The dense FP4 tensor-core probe (a measurement helper, not a step of the
layer): it runs the GEMM's own block-scaled pair MMA from shared-memory
operands on every SM, reports its flop count, finishes without a device error,
and its rate is a tensor-core rate -- above what the prefill GEMM reaches on a
whole problem, and within the part's nominal dense FP4 figure times the ratio of
the highest SM clock to the clock that figure assumes."""
import pytest

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nv():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import nvfp4_w4a4_block_b200 as nv
    nv.lib()
    return nv


@pytest.mark.parametrize("copies", [False, True], ids=["mma_only", "with_scale_copies"])
def test_probe_runs_and_reports_a_tensor_core_rate(nv, copies):
    import torch
    pairs = torch.cuda.get_device_properties(0).multi_processor_count // 2
    nv.mma_peak_probe(1000, with_scale_copies=copies)
    s = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s)
    flops = nv.mma_peak_probe(20000, with_scale_copies=copies)
    e1.record(s)
    torch.cuda.synchronize()
    assert nv.get_device_error() == nv.OK
    assert flops == 2.0 * 256 * 256 * 64 * 4 * 20000 * pairs
    tflops = flops / (e0.elapsed_time(e1) * 1e-3) / 1e12
    assert 2000.0 < tflops < 15000.0, tflops


def test_probe_rejects_bad_arguments(nv):
    import torch
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    for pairs, iters in ((0, 10), (1, 0), (sms // 2 + 1, 10)):
        with pytest.raises(nv.NVFP4Error):
            nv.mma_peak_probe(iters, pairs=pairs)
