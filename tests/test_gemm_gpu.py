"""GPU parity of the block-scaled FP4 GEMM and of the whole linear layer
against the CPU oracle (fp64 GEMM on the identical dequantized operands).

The operands the GPU quantized are first asserted bit-exact with the oracle's,
so any GEMM error is the kernel's.  Tolerance (tests/_helpers.py): fp32
output within 1e-3 of max(|R|, row RMS); bf16 output additionally within its
own rounding (2^-8 relative), and equal to the RNE rounding of the same
kernel's fp32 output.
"""
import numpy as np
import pytest

import oracle
from nvfp4_w4a4_block_b200 import workloads as W

from _helpers import assert_gemm_close, bf16_rne_from_f32, to_cuda_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nv():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import nvfp4_w4a4_block_b200 as nv
    nv.lib()
    return nv


def _bf16_to_f64(t):
    import torch
    return t.float().cpu().numpy().astype(np.float64)


def _layer(nv, xb, wb, seg_offsets, act_static=None, flags=0):
    """Run the whole layer on the GPU; return (y_gpu, oracle dict, packed weight).
    Both operands' codes, scale bytes and global scales are first asserted equal
    to the oracle's, so any output error is the GEMM's."""
    import torch
    x = to_cuda_bf16(xb)
    pw = nv.pack_weight(to_cuda_bf16(wb), seg_offsets)
    g = None if act_static is None else torch.tensor([act_static], dtype=torch.float32, device="cuda")
    y = nv.linear_fused(x, pw, act_gscale=g, flags=flags)
    qx, sfx, sx = nv.quantize_act(x, gscale=g)
    torch.cuda.synchronize()
    assert nv.get_device_error() == nv.OK
    ref = oracle.linear_reference(xb, wb, seg_offsets, act_scale=act_static)
    k = xb.shape[1]
    assert pw.gscale.cpu().numpy().tobytes() == ref["s_w"].tobytes()
    assert np.array_equal(pw.q.cpu().numpy(), ref["qw"]), "weight codes differ"
    assert np.array_equal(pw.sf.cpu().numpy(), oracle.sf_to_physical(ref["sfw"], k)), "weight scales differ"
    assert np.float32(sx.item()).tobytes() == np.float32(ref["s_x"]).tobytes()
    assert np.array_equal(qx.cpu().numpy(), ref["qx"]), "activation codes differ"
    assert np.array_equal(sfx.cpu().numpy(), oracle.sf_to_physical(ref["sfx"], k)), "activation scales differ"
    return y, ref, pw


@pytest.mark.parametrize("m,n,k,segs", [
    (16, 128, 256, None),          # tiny workload shape
    (1, 8, 64, None),              # smallest: one row, one column group, one K atom
    (3, 96, 64, None),
    (128, 256, 256, None),         # exactly one tile, one stage
    (300, 600, 1088, None),        # ragged M, N and K-stage tails, several tiles
    (257, 520, 320, [0, 256, 520]),
    (64, 1040, 2048, [0, 512, 768, 1024, 1040]),
    (130, 264, 5120, [0, 136, 264]),
    (8300, 600, 256, [0, 264, 600]),  # 33 M tiles: tile groups of 16, 16 and a ragged 1
])
def test_gemm_parity_random(nv, m, n, k, segs):
    import torch
    seg_rows = None if segs is None else [segs[i + 1] - segs[i] for i in range(len(segs) - 1)]
    xb, wb, off = W.random_case(7, m, n, k, seg_rows=seg_rows)
    y32, ref, pw = _layer(nv, xb, wb, off, flags=nv.FLAG_F32_OUT)
    assert_gemm_close(y32.cpu().numpy(), ref["y"], bf16=False)
    ybf = nv.linear_fused(to_cuda_bf16(xb), pw)
    torch.cuda.synchronize()
    assert_gemm_close(_bf16_to_f64(ybf), ref["y"], bf16=True)
    # the bf16 output is exactly the RNE rounding of the fp32 result
    assert np.array_equal(ybf.view(torch.int16).cpu().numpy().view(np.uint16), bf16_rne_from_f32(y32.cpu().numpy()))


@pytest.mark.parametrize("m", [8, 40, 200], ids=["decode_T8", "decode_T64", "pair"])
def test_gemm_eight_modules_some_eight_columns_wide(nv, m):
    """The largest number of fused modules (eight, each with its own weight
    global scale, spread 1x-8x), four of them only 8 columns wide -- the finest
    boundary granularity -- on each GEMM kernel: every output column is scaled by
    the scale of its own module."""
    import torch
    widths = [8, 8, 120, 8, 120, 8, 120, 8]
    xb, wb, off = W.random_case(71, m, sum(widths), 1088, seg_rows=widths)
    assert len(off) - 1 == 8
    y32, ref, pw = _layer(nv, xb, wb, off, flags=nv.FLAG_F32_OUT)
    assert_gemm_close(y32.cpu().numpy(), ref["y"], bf16=False)
    g = pw.gscale.cpu().numpy()
    assert g.max() / g.min() > 4.0                      # a column scaled by another module's scale shows
    ybf = nv.linear_fused(to_cuda_bf16(xb), pw)
    torch.cuda.synchronize()
    assert np.array_equal(ybf.view(torch.int16).cpu().numpy().view(np.uint16), bf16_rne_from_f32(y32.cpu().numpy()))


@pytest.mark.parametrize("m", [1, 7, 8, 9, 16, 17, 31, 32, 33, 63, 64, 65, 100, 128, 129])
def test_gemm_token_buckets(nv, m):
    """Every token-count bucket of the swapped decode kernel (8/16/32/64/128) and
    the switch to the tile kernel above 128, with ragged N (200 = 128 + 72) and a
    partial last K stage (320 = 256 + 64), two segments."""
    import torch
    xb, wb, off = W.random_case(20 + m, m, 200, 320, seg_rows=[64, 136])
    y32, ref, pw = _layer(nv, xb, wb, off, flags=nv.FLAG_F32_OUT)
    assert_gemm_close(y32.cpu().numpy(), ref["y"], bf16=False)
    ybf = nv.linear_fused(to_cuda_bf16(xb), pw)
    torch.cuda.synchronize()
    assert np.array_equal(ybf.view(torch.int16).cpu().numpy().view(np.uint16), bf16_rne_from_f32(y32.cpu().numpy()))


def test_gemm_exact_on_representable_operands(nv):
    """E2M1 grid values x power-of-two block magnitudes under power-of-two global
    scales quantize losslessly, so the layer must reproduce X.W^T (fp64 via
    NumPy) to fp32 accumulation accuracy."""
    import torch
    rng = np.random.default_rng(12)
    grid = np.array([0, .5, 1, 1.5, 2, 3, 4, 6, -.5, -1, -1.5, -2, -3, -4, -6])
    m, n, k = 200, 264, 512

    def rep(rows):
        v = rng.choice(grid, size=(rows, k))
        v[:, ::16] = 6.0
        return v * np.repeat(2.0 ** rng.integers(-3, 3, size=(rows, k // 16)), 16, axis=1)

    x, w = rep(m), rep(n)
    xb, wb = W.f32_to_bf16_bits(x), W.f32_to_bf16_bits(w)
    pw = nv.pack_weight(to_cuda_bf16(wb), gscale=torch.tensor([2.0 ** -5], device="cuda"))
    y = nv.linear(to_cuda_bf16(xb), pw, act_gscale=torch.tensor([2.0 ** -6], device="cuda"),
                  flags=nv.FLAG_F32_OUT)
    torch.cuda.synchronize()
    exact = x @ w.T
    err = np.abs(y.cpu().numpy().astype(np.float64) - exact)
    assert (err <= 1e-6 * np.maximum(np.abs(exact), 1.0)).all()


def test_fused_segments_match_separate_modules_and_collapsed_mode_fails(nv):
    """Per-segment epilogue == separate per-module GEMMs; the collapsed-max mode
    (the serving mismatch of "Why Gated DeltaNet Survives 4-Bit Quantization",
    §6 "Per-module calibration vs. fused-GEMM scaling") mis-scales the smaller-scale module
    by the scale ratio."""
    import torch
    m, k = 96, 512
    xb, wb, off = W.random_case(9, m, 512, k, seg_rows=[256, 256])
    wf = W.bf16_bits_to_f32(wb).copy()
    wf[256:] *= 2.75 / 2.0                          # segment scales differ ~2.75x
    wb = W.f32_to_bf16_bits(wf)
    x = to_cuda_bf16(xb)
    pw = nv.pack_weight(to_cuda_bf16(wb), off)
    fused = nv.linear_fused(x, pw, flags=nv.FLAG_F32_OUT)
    for i in range(2):
        pwi = nv.pack_weight(to_cuda_bf16(np.ascontiguousarray(wb[off[i]:off[i + 1]])))
        yi = nv.linear(x, pwi, flags=nv.FLAG_F32_OUT)
        torch.cuda.synchronize()
        assert torch.equal(yi, fused[:, off[i]:off[i + 1]])
    bad = nv.linear_fused(x, pw, flags=nv.FLAG_F32_OUT | nv.FLAG_COLLAPSED_MAX_SCALE)
    torch.cuda.synchronize()
    s_w = pw.gscale.cpu().numpy()
    ratio = s_w.max() / s_w.min()
    assert ratio > 2.5
    small = int(np.argmin(s_w))
    sl = slice(off[small], off[small + 1])
    e = (torch.linalg.norm(bad[:, sl] - fused[:, sl]) / torch.linalg.norm(fused[:, sl])).item()
    assert abs(e - (ratio - 1)) < 1e-3
    ref = oracle.linear_reference(xb, wb, off)
    assert_gemm_close(fused.cpu().numpy(), ref["y"], bf16=False)


def test_gemm_entry_on_prequantized_operands(nv):
    import torch
    xb, wb, off = W.random_case(10, 200, 384, 768)
    x = to_cuda_bf16(xb)
    qx, sfx, sx = nv.quantize_act(x)
    pw = nv.pack_weight(to_cuda_bf16(wb))
    y = nv.gemm(qx, sfx, sx, 200, pw, flags=nv.FLAG_F32_OUT)
    y2 = nv.linear(x, pw, flags=nv.FLAG_F32_OUT)
    torch.cuda.synchronize()
    assert torch.equal(y, y2)


@pytest.mark.parametrize("m", [1, 5, 8, 16, 31, 32, 64])
@pytest.mark.parametrize("static", [None, 0.003])
def test_layer_equals_quantize_then_gemm(nv, m, static):
    """The whole layer (nvfp4_linear_fused, which chains the quantizer and the
    GEMM with programmatic dependent launch) is bit-identical to quantizing
    first (nvfp4_quantize_act) and running the GEMM on those codes (nvfp4_gemm)."""
    import torch
    xb, wb, off = W.random_case(60 + m, m, 392, 1344, seg_rows=[128, 264])
    x = to_cuda_bf16(xb)
    pw = nv.pack_weight(to_cuda_bf16(wb), off)
    g = None if static is None else torch.tensor([static], dtype=torch.float32, device="cuda")
    for flags in (nv.FLAG_F32_OUT, 0):
        fused = nv.linear_fused(x, pw, act_gscale=g, flags=flags)
        qx, sfx, sx = nv.quantize_act(x, gscale=g)
        split = nv.gemm(qx, sfx, sx, m, pw, flags=flags)
        torch.cuda.synchronize()
        assert nv.get_device_error() == nv.OK
        assert torch.equal(fused, split)


@pytest.mark.parametrize("m", [8, 40, 300])
def test_strided_output_rows_leave_the_gap_untouched(nv, m):
    """Y with a row stride beyond N (the bf16 tile stores go through TMA with
    the caller's stride): the N columns match the contiguous result bit for bit
    and the padding columns keep their contents."""
    import torch
    n, k = 328, 640
    xb, wb, off = W.random_case(12, m, n, k, seg_rows=[136, 192])
    x = to_cuda_bf16(xb)
    pw = nv.pack_weight(to_cuda_bf16(wb), off)
    ref = nv.linear_fused(x, pw)
    big = torch.full((m, n + 72), 3.0, dtype=torch.bfloat16, device="cuda")
    nv.linear_fused(x, pw, out=big[:, :n])
    torch.cuda.synchronize()
    assert torch.equal(big[:, :n], ref)
    assert (big[:, n:] == 3.0).all()


def test_static_activation_scale(nv):
    xb, wb, off = W.random_case(11, 140, 256, 640)
    y, ref, _ = _layer(nv, xb, wb, off, act_static=0.004, flags=nv.FLAG_F32_OUT)
    assert_gemm_close(y.cpu().numpy(), ref["y"], bf16=False)


def test_zero_rows_is_a_noop(nv):
    import torch
    pw = nv.pack_weight(to_cuda_bf16(W.random_case(0, 1, 64, 128)[1]))
    x = torch.empty((0, 128), dtype=torch.bfloat16, device="cuda")
    y = nv.linear(x, pw)
    assert y.shape == (0, 64)


# ----------------------------------------------------------------- workloads

def _rows_sample(m, seed, n_rand):
    rng = np.random.default_rng(seed)
    return np.unique(np.concatenate([np.arange(min(m, 64)), rng.integers(0, m, n_rand),
                                     np.arange(max(0, m - 32), m)]))


def _workload_layer(nv, wl, xb, rows=None):
    """The whole layer on one workload, checked the way the tolerance reading
    asks for it:
      * codes and scale bytes of both operands equal the oracle's (weights in
        full; activations in full, or on the sampled rows when `rows` is given,
        the global scale always from the whole tensor);
      * the fp32 output is within 1e-3 of max(|R|, row RMS) of the fp64 oracle;
      * the bf16 output is within that plus its own rounding, and equals the
        round-to-nearest-even bf16 of the same kernel's fp32 output bit for bit.
    """
    import torch
    wb = wl.w()
    x = to_cuda_bf16(xb)
    pw = nv.pack_weight(to_cuda_bf16(wb), wl.seg_offsets)
    qx, sfx, sx = nv.quantize_act(x)
    y32 = nv.linear_fused(x, pw, flags=nv.FLAG_F32_OUT)
    ybf = nv.linear_fused(x, pw)
    torch.cuda.synchronize()
    assert nv.get_device_error() == nv.OK
    ref = oracle.linear_reference(xb, wb, wl.seg_offsets, rows=rows)
    # operands: bit-exact
    assert pw.gscale.cpu().numpy().tobytes() == ref["s_w"].tobytes()
    assert np.array_equal(pw.q.cpu().numpy(), ref["qw"]), "weight codes differ"
    assert np.array_equal(pw.sf.cpu().numpy(), oracle.sf_to_physical(ref["sfw"], wl.k)), "weight scales differ"
    assert np.float32(sx.item()).tobytes() == np.float32(ref["s_x"]).tobytes()
    if rows is None:
        assert np.array_equal(qx.cpu().numpy(), ref["qx"]), "activation codes differ"
        assert np.array_equal(sfx.cpu().numpy(), oracle.sf_to_physical(ref["sfx"], wl.k)), "activation scales differ"
        y32h, ybfh = y32.cpu().numpy(), ybf.view(torch.int16).cpu().numpy().view(np.uint16)
    else:
        sel = torch.as_tensor(np.asarray(rows), device="cuda")
        assert np.array_equal(qx[sel].cpu().numpy(), ref["qx"]), "activation codes differ"
        sf_h = sfx.cpu().numpy()
        offs = np.array([[oracle.sf_offset(int(r), c, wl.k) for c in range(wl.k // 16)] for r in rows])
        assert np.array_equal(sf_h[offs], ref["sfx"]), "activation scales differ"
        y32h, ybfh = y32[sel].cpu().numpy(), ybf[sel].view(torch.int16).cpu().numpy().view(np.uint16)
    # GEMM: fp32 within 1e-3, bf16 within 1e-3 + its rounding and equal to RNE(fp32)
    assert_gemm_close(y32h, ref["y"], bf16=False)
    assert_gemm_close(W.bf16_bits_to_f32(ybfh), ref["y"], bf16=True)
    assert np.array_equal(ybfh, bf16_rne_from_f32(y32h))


def test_tiny_workload_full(nv):
    _workload_layer(nv, W.TINY, W.TINY.x())


@pytest.mark.parametrize("m", W.DECODE_M)
def test_decode_workload_full(nv, m):
    _workload_layer(nv, W.DECODE, W.DECODE.x(m))


def test_fused_qkvg_workload_full(nv):
    """4096 x 5120 -> 6144 + 2048 + 2048 + 96, four modules with their own
    weight global scales: every output element against the oracle."""
    _workload_layer(nv, W.FUSED_QKVG, W.FUSED_QKVG.x())


def test_prefill_workload_sampled_rows(nv):
    wl = W.PREFILL
    _workload_layer(nv, wl, wl.x(), rows=_rows_sample(wl.m, wl.cfg_id, 64))


def test_long_prefill_workload_sampled_rows(nv):
    wl = W.LONG_DOWN
    _workload_layer(nv, wl, wl.x(), rows=_rows_sample(wl.m, wl.cfg_id, 32)[::2])


@pytest.mark.parametrize("m", [8, 40, 200], ids=["decode_T8", "decode_T64", "pair"])
def test_inputs_rewritten_just_before_a_call_are_the_ones_it_reads(nv, m):
    """Every GEMM is launched with programmatic stream serialization, so it may
    start while the kernel before it still runs; the library's quantizers let
    their dependents start early too.  Packed weights and activation codes
    rewritten in place by the immediately preceding call (nothing in between on
    the stream) must still be the ones the layer reads: the results equal those
    computed from freshly allocated operands."""
    import ctypes
    import torch
    n, k = 392, 1344
    xb1, wb1, off = W.random_case(80 + m, m, n, k, seg_rows=[128, 264])
    xb2, wb2, _ = W.random_case(90 + m, m, n, k, seg_rows=[128, 264])
    x1, x2 = to_cuda_bf16(xb1), to_cuda_bf16(xb2)
    w2 = to_cuda_bf16(wb2)
    ref_pw = nv.pack_weight(w2, off)
    expect_layer = nv.linear_fused(x1, ref_pw, flags=nv.FLAG_F32_OUT)
    qx2, sfx2, sx2 = nv.quantize_act(x2)
    expect_gemm = nv.gemm(qx2, sfx2, sx2, m, ref_pw, flags=nv.FLAG_F32_OUT)
    torch.cuda.synchronize()

    pw = nv.pack_weight(to_cuda_bf16(wb1), off)            # buffers that will be overwritten
    qx, sfx, sx = nv.quantize_act(x1)
    nv.linear_fused(x1, pw, flags=nv.FLAG_F32_OUT)          # warm, with the first weight
    torch.cuda.synchronize()
    L = nv.lib()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    segs = (ctypes.c_int64 * len(off))(*off)
    ws = torch.empty(nv.workspace_bytes(n, 0, k), dtype=torch.uint8, device="cuda")
    ws_layer = torch.empty(nv.workspace_bytes(m, n, k), dtype=torch.uint8, device="cuda")
    torch.cuda.synchronize()
    # repack in place, then the layer right behind it
    st = L.nvfp4_pack_weight(w2.data_ptr(), n, k, k, segs, len(off) - 1, None, pw.gscale.data_ptr(), pw.q.data_ptr(),
                             pw.sf.data_ptr(), ws.data_ptr(), ws.numel(), stream)
    assert st == nv.OK
    y_layer = nv.linear_fused(x1, pw, flags=nv.FLAG_F32_OUT, ws=ws_layer)
    # re-quantize the activations in place, then the GEMM right behind it
    nv.quantize_act(x2, q=qx, sf=sfx, gscale_out=sx)
    y_gemm = nv.gemm(qx, sfx, sx, m, pw, flags=nv.FLAG_F32_OUT)
    torch.cuda.synchronize()
    assert nv.get_device_error() == nv.OK
    assert torch.equal(y_layer, expect_layer)
    assert torch.equal(y_gemm, expect_gemm)


@pytest.mark.parametrize("m", [1, 32, 200], ids=["decode_T8", "decode_T32", "pair"])
def test_layer_and_gemm_replay_from_a_cuda_graph(nv, m):
    """The quantizer -> GEMM chain (with its programmatic launch edges) and the
    stand-alone GEMM captured into one CUDA graph and replayed give the eager
    results bit for bit, also when the inputs change between replays."""
    import torch
    n, k = 520, 1088
    xb, wb, off = W.random_case(95 + m, m, n, k, seg_rows=[264, 256])
    pw = nv.pack_weight(to_cuda_bf16(wb), off)
    x = to_cuda_bf16(xb)
    qx, sfx, sx = nv.quantize_act(x)
    ws = torch.empty(nv.workspace_bytes(m, n, k), dtype=torch.uint8, device="cuda")
    y_layer = torch.empty((m, n), dtype=torch.bfloat16, device="cuda")
    y_gemm = torch.empty((m, n), dtype=torch.float32, device="cuda")

    def step():
        nv.linear_fused(x, pw, out=y_layer, ws=ws)
        nv.gemm(qx, sfx, sx, m, pw, out=y_gemm, flags=nv.FLAG_F32_OUT)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step()                                           # first calls (per-device set-up) outside capture
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    for seed in (96, 97):
        xb2, _, _ = W.random_case(seed + m, m, n, k)
        x.copy_(to_cuda_bf16(xb2))
        q2, sf2, s2 = nv.quantize_act(x)
        qx.copy_(q2)
        sfx.copy_(sf2)
        sx.copy_(s2)
        g.replay()
        torch.cuda.synchronize()
        assert nv.get_device_error() == nv.OK
        assert torch.equal(y_layer, nv.linear_fused(x, pw))
        assert torch.equal(y_gemm, nv.gemm(qx, sfx, sx, m, pw, flags=nv.FLAG_F32_OUT))
    del g


@pytest.mark.parametrize("m", [8, 40, 200], ids=["decode_T8", "decode_T64", "pair"])
def test_static_weights_flag_changes_nothing_but_the_launch_order(nv, m):
    """With NVFP4_FLAG_STATIC_WEIGHTS the GEMM requests its first weight stages
    before it waits for the preceding kernel; back-to-back calls on packed
    (static) weights give the same bits as without the flag."""
    import torch
    xb, wb, off = W.random_case(98 + m, m, 520, 1344, seg_rows=[264, 256])
    pw = nv.pack_weight(to_cuda_bf16(wb), off)
    pw2 = nv.pack_weight(to_cuda_bf16(W.random_case(99 + m, m, 520, 1344, seg_rows=[264, 256])[1]), off)
    qx, sfx, sx = nv.quantize_act(to_cuda_bf16(xb))
    for flags in (0, nv.FLAG_F32_OUT):
        ref1 = nv.gemm(qx, sfx, sx, m, pw, flags=flags)
        ref2 = nv.gemm(qx, sfx, sx, m, pw2, flags=flags)
        got = [nv.gemm(qx, sfx, sx, m, p, flags=flags | nv.FLAG_STATIC_WEIGHTS) for p in (pw, pw2, pw, pw2)]
        torch.cuda.synchronize()
        assert nv.get_device_error() == nv.OK
        assert torch.equal(got[0], ref1) and torch.equal(got[2], ref1)
        assert torch.equal(got[1], ref2) and torch.equal(got[3], ref2)



# Up to 32 tokens on few weight tiles (N up to 74 x 128) with K of at least 8
# stages: the decode GEMM splits K over a cluster of four CTAs and reduces the
# partial sums in CTA 0.  The down-projection of the decode workloads' model
# (5120 x 17408), a ragged N with three modules, a partial last K stage.
SPLIT_K_CASES = [
    (1, 512, 2048, None),
    (8, 1000, 5120, [264, 256, 480]),
    (16, 5120, 17408, None),
    (3, 2048, 2112, [1024, 1024]),
    (12, 9472, 2048, None),
    (32, 5120, 17408, None),
    (24, 1000, 2112, [264, 256, 480]),
]


@pytest.mark.parametrize("m,n,k,segs", SPLIT_K_CASES)
def test_split_k_decode_gemm(nv, m, n, k, segs):
    import torch
    xb, wb, off = W.random_case(500 + m, m, n, k, seg_rows=segs)
    x = to_cuda_bf16(xb)
    pw = nv.pack_weight(to_cuda_bf16(wb), off)
    y32 = nv.linear_fused(x, pw, flags=nv.FLAG_F32_OUT)
    ybf = nv.linear_fused(x, pw)
    qx, sfx, sx = nv.quantize_act(x)
    g32 = nv.gemm(qx, sfx, sx, m, pw, flags=nv.FLAG_F32_OUT)
    gst = nv.gemm(qx, sfx, sx, m, pw, flags=nv.FLAG_F32_OUT | nv.FLAG_STATIC_WEIGHTS)
    torch.cuda.synchronize()
    assert nv.get_device_error() == nv.OK
    ref = oracle.linear_reference(xb, wb, off)
    assert_gemm_close(y32.cpu().numpy(), ref["y"], bf16=False)
    assert np.array_equal(ybf.view(torch.int16).cpu().numpy().view(np.uint16), bf16_rne_from_f32(y32.cpu().numpy()))
    assert torch.equal(y32, g32) and torch.equal(y32, gst)        # deterministic: the same sums in the same order
