"""GPU parity of the NVFP4 quantization kernels against the CPU oracle.

Codes, scale bytes (physical tensor-core layout, pads included) and the global
scale must match bit for bit; both sides take every rounding decision in fp32
with the same operation order.
"""
import os

import numpy as np
import pytest

import oracle
from nvfp4_w4a4_block_b200 import workloads as W

from _helpers import to_cuda_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nv():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import nvfp4_w4a4_block_b200 as nv
    nv.lib()
    return nv


def _run_quant(nv, bits, static=None):
    import torch
    x = to_cuda_bf16(bits)
    g = None if static is None else torch.tensor([static], dtype=torch.float32, device="cuda")
    q, sf, s = nv.quantize_act(x, gscale=g)
    torch.cuda.synchronize()
    assert nv.get_device_error() == nv.OK
    return q.cpu().numpy(), sf.cpu().numpy(), np.float32(s.item())


def _expect(bits, static=None):
    s = oracle.global_scale(oracle.amax(bits)) if static is None else np.float32(static)
    q, sf = oracle.quantize(bits, s)
    return q, oracle.sf_to_physical(sf, bits.shape[1]), s


def _compare(nv, bits, static=None):
    qg, sfg, sg = _run_quant(nv, bits, static)
    qo, sfo, so = _expect(bits, static)
    assert sg.tobytes() == np.float32(so).tobytes()
    assert sfg.shape == sfo.shape
    if not np.array_equal(sfg, sfo):
        bad = np.flatnonzero(sfg != sfo)
        raise AssertionError(f"{bad.size} scale bytes differ, first at {bad[0]}: gpu {sfg[bad[0]]:#x} "
                             f"oracle {sfo[bad[0]]:#x}")
    if not np.array_equal(qg, qo):
        bad = np.argwhere(qg != qo)
        r, c = bad[0]
        raise AssertionError(f"{len(bad)} code bytes differ, first at {r},{c}: gpu {qg[r, c]:#x} "
                             f"oracle {qo[r, c]:#x}")


@pytest.mark.parametrize("m,k", [(1, 64), (2, 128), (16, 256), (127, 320), (300, 1088), (129, 5120),
                                 (37, 17408), (1000, 64)])
def test_quantize_random_shapes_dynamic(nv, m, k):
    x, _, _ = W.random_case(3, m, 8, k)
    _compare(nv, x)


@pytest.mark.parametrize("m,k", [(1000, 1088), (2049, 1024), (130, 17408), (8192, 128)])
@pytest.mark.parametrize("static", [None, 0.002])
def test_quantize_tiled_path_shapes(nv, m, k, static):
    """Tensors above 2^20 elements take the tiled encoder (128-row x 64-column
    tiles, whole scale atoms); ragged row tiles leave zero pad scales."""
    x, _, _ = W.random_case(30, m, 8, k)
    _compare(nv, x, static)


def test_quantize_ties_on_the_tiled_path(nv):
    ties = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], np.float32)
    rows = []
    for j in range(-10, 6):
        blk = np.concatenate([[6.0], ties, -ties, [0.0]]).astype(np.float32) * np.float32(2.0 ** j)
        rows.append(np.tile(blk, 128))
    x = W.f32_to_bf16_bits(np.tile(np.stack(rows), (40, 1)))      # 640 x 2048 > 2^20
    assert x.size > (1 << 20)
    _compare(nv, x, 2.0 ** -8)
    _compare(nv, x)


@pytest.mark.parametrize("static", [2.0 ** -9, 1e-3, 0.37, 1e-6, 0.0])
def test_quantize_static_scale(nv, static):
    x, _, _ = W.random_case(4, 200, 8, 512)
    _compare(nv, x, static)


@pytest.mark.parametrize("bad", [-1.0, float("inf"), float("nan")], ids=["negative", "inf", "nan"])
@pytest.mark.parametrize("m,k", [(8, 5120), (300, 1088), (1000, 1088)], ids=["cluster", "per_unit", "tiled"])
def test_quantize_invalid_static_scale_is_reported(nv, m, k, bad):
    """A given global scale that is negative or not finite is reported as
    non-finite, and the tensor is encoded as with scale 0 (zero block scales,
    codes +-0 by sign), on each quantizer path."""
    import torch
    x, _, _ = W.random_case(35, m, 8, k)
    g = torch.tensor([bad], dtype=torch.float32, device="cuda")
    q, sf, s = nv.quantize_act(to_cuda_bf16(x), gscale=g)
    torch.cuda.synchronize()
    assert nv.get_device_error() == nv.ERR_NONFINITE
    assert nv.get_device_error() == nv.OK
    qo, sfo, _ = _expect(x, 0.0)
    assert s.item() == 0.0
    assert np.array_equal(sf.cpu().numpy(), sfo)
    assert np.array_equal(q.cpu().numpy(), qo)


def test_quantize_every_bf16_value_on_identity_scale(nv):
    """Global scale 2^-8 and a 6.0 in every block make the element divisor exactly
    1, so each bf16 value in [-6, 6] is encoded as itself: every tie, every
    sub-grid value, both zeros."""
    bits = np.arange(0, 1 << 16, dtype=np.uint32).astype(np.uint16)
    vals = W.bf16_bits_to_f32(bits)
    keep = bits[np.isfinite(vals) & (np.abs(vals) <= 6.0)]
    per_block = 15
    nblk = (keep.size + per_block - 1) // per_block
    pad = nblk * per_block - keep.size
    body = np.concatenate([keep, np.zeros(pad, np.uint16)]).reshape(nblk, per_block)
    six = W.f32_to_bf16_bits(np.full((nblk, 1), 6.0, np.float32))
    blocks = np.concatenate([six, body], axis=1)                      # [nblk, 16]
    k = 1024
    rows = (nblk * 16 + k - 1) // k
    flat = np.concatenate([blocks.reshape(-1), np.tile(six.reshape(-1)[:1], rows * k - nblk * 16)])
    _compare(nv, flat.reshape(rows, k), 2.0 ** -8)


def test_quantize_ties_under_power_of_two_block_scales(nv):
    """Exact ties (0.25, 0.75, ... 5 times the divisor) at many block magnitudes."""
    ties = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], np.float32)
    rows = []
    for j in range(-10, 6):
        blk = np.concatenate([[6.0], ties, -ties, [0.0]]).astype(np.float32) * np.float32(2.0 ** j)
        rows.append(np.tile(blk, 4))
    x = W.f32_to_bf16_bits(np.stack(rows))
    _compare(nv, x, 2.0 ** -8)
    _compare(nv, x)


def test_quantize_zero_and_negative_zero(nv):
    x = np.zeros((3, 64), np.uint16)
    x[1, ::2] = 0x8000                                  # -0.0
    _compare(nv, x)
    _compare(nv, x, 0.5)


@pytest.mark.parametrize("m,k,pad", [(64, 256, 128), (8, 5120, 64), (129, 5120, 192), (1000, 1088, 64)],
                         ids=["cluster_small", "cluster_decode", "per_unit", "tiled"])
@pytest.mark.parametrize("static", [None, 0.004])
def test_quantize_strided_rows(nv, m, k, pad, static):
    """Rows of X further apart than K (a view into a wider buffer, whose extra
    columns hold large values that must not leak into the amax) on each
    quantizer path."""
    import torch
    xb, _, _ = W.random_case(5, m, 8, k)
    big = np.full((m, k + pad), W.f32_to_bf16_bits(np.array([1000.0], np.float32))[0], np.uint16)
    big[:, :k] = xb
    xt = to_cuda_bf16(big)[:, :k]
    g = None if static is None else torch.tensor([static], dtype=torch.float32, device="cuda")
    q, sf, s = nv.quantize_act(xt, gscale=g)
    torch.cuda.synchronize()
    assert nv.get_device_error() == nv.OK
    qo, sfo, so = _expect(xb, static)
    assert s.item() == float(so)
    assert np.array_equal(q.cpu().numpy(), qo)
    assert np.array_equal(sf.cpu().numpy(), sfo)


def test_quantize_nonfinite_sets_device_error(nv):
    import torch
    x = np.zeros((4, 64), np.uint16)
    x[2, 5] = 0x7F80                                     # +inf
    xt = to_cuda_bf16(x)
    nv.quantize_act(xt)
    assert nv.get_device_error() == nv.ERR_NONFINITE
    assert nv.get_device_error() == nv.OK               # cleared
    nv.quantize_act(to_cuda_bf16(np.ones((4, 64), np.uint16)))
    torch.cuda.synchronize()
    assert nv.get_device_error() == nv.OK


# (m, k, launches of a dynamic-scale quantization): one cluster launch up to
# 327680 elements (5 units per thread) and up to 786432 (its 12-unit instance);
# above that the amax pass and the per-unit encoder (two launches).
ONE_LAUNCH_LIMIT_CASES = [
    (1, 5120, 1), (4, 5120, 1), (8, 5120, 1), (9, 5120, 1), (1, 40960, 1), (1, 41024, 1), (2, 20480, 1),
    (32, 5120, 1), (38, 5120, 1), (39, 5120, 1), (64, 5120, 1), (18, 17408, 1), (19, 17408, 1),
    (1, 196608, 1), (1, 327680, 1), (1, 327744, 1),
    (65, 5120, 1), (100, 5120, 1), (128, 5120, 1), (153, 5120, 1), (154, 5120, 2),
    (45, 17408, 1), (46, 17408, 2), (1, 786432, 1), (1, 786496, 2),
]


@pytest.mark.parametrize("m,k,launches", ONE_LAUNCH_LIMIT_CASES)
def test_quantize_decode_sizes_around_the_one_launch_limit(nv, m, k, launches):
    """Dynamic-scale activations are quantized in one cluster launch (the whole
    tensor held in registers) up to 327680 elements with 5 units per thread and
    up to 786432 with 12; just above that the amax pass and the per-unit encoder
    take over.  Both sides of each limit, and shapes whose pad rows fill most of
    the scale block."""
    import torch
    x, _, _ = W.random_case(33, m, 8, k)
    xt = to_cuda_bf16(x)
    torch.cuda.synchronize()
    c0 = nv.launch_count()
    nv.quantize_act(xt)
    torch.cuda.synchronize()
    assert nv.launch_count() - c0 == launches
    _compare(nv, x)


def test_fallback_without_the_cluster_quantizer_gives_the_same_bytes(nv):
    """With the one-launch cluster quantizer switched off (what a device that
    cannot hold a 16-CTA cluster gets), decode-sized activations take the amax
    pass and the per-unit encoder: the same codes, scales and global scale, and
    the same decode layer output.  Runs in a child process, since the choice is
    made once per device."""
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    code = r"""
import sys, numpy as np, torch
sys.path.insert(0, %r); sys.path.insert(0, %r)
import oracle, nvfp4_w4a4_block_b200 as nv
from nvfp4_w4a4_block_b200 import workloads as W
from _helpers import to_cuda_bf16, assert_gemm_close
nv.lib()
for m, k, static in [(1, 5120, None), (8, 5120, None), (32, 5120, 0.004), (64, 5120, None)]:
    x, w, off = W.random_case(36, m, 264, k, seg_rows=[136, 128])
    g = None if static is None else torch.tensor([static], dtype=torch.float32, device="cuda")
    xt = to_cuda_bf16(x)
    c0 = nv.launch_count()
    q, sf, s = nv.quantize_act(xt, gscale=g)
    assert nv.launch_count() - c0 == (1 if static is not None else 2)   # encoder (+ amax pass): no cluster
    torch.cuda.synchronize()
    assert nv.get_device_error() == nv.OK
    so = oracle.global_scale(oracle.amax(x)) if static is None else np.float32(static)
    qo, sfo = oracle.quantize(x, so)
    assert np.float32(s.item()).tobytes() == np.float32(so).tobytes()
    assert np.array_equal(q.cpu().numpy(), qo)
    assert np.array_equal(sf.cpu().numpy(), oracle.sf_to_physical(sfo, k))
    pw = nv.pack_weight(to_cuda_bf16(w), off)
    y = nv.linear_fused(to_cuda_bf16(x), pw, act_gscale=g, flags=nv.FLAG_F32_OUT)
    torch.cuda.synchronize()
    ref = oracle.linear_reference(x, w, off, act_scale=static)
    assert_gemm_close(y.cpu().numpy(), ref["y"], bf16=False)
print("ok")
""" % (root, os.path.join(root, "tests"))
    env = dict(os.environ, NVFP4_NO_CLUSTER_QUANTIZER="1")
    r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout + r.stderr
    assert r.stdout.split()[0] == "ok"


@pytest.mark.parametrize("m,k", [(1, 5120), (8, 5120), (38, 5120), (64, 5120)])
def test_quantize_nonfinite_in_the_one_launch_path(nv, m, k):
    import torch
    x, _, _ = W.random_case(34, m, 8, k)
    x = x.copy()
    x[m - 1, k - 3] = 0xFF80                             # -inf in the last unit
    nv.quantize_act(to_cuda_bf16(x))
    assert nv.get_device_error() == nv.ERR_NONFINITE
    nv.quantize_act(to_cuda_bf16(np.ones((m, k), np.uint16)))
    torch.cuda.synchronize()
    assert nv.get_device_error() == nv.OK


@pytest.mark.parametrize("wl", [W.TINY, W.PREFILL, W.FUSED_QKVG], ids=lambda w: w.name)
def test_quantize_workload_activations(nv, wl):
    _compare(nv, wl.x())


@pytest.mark.parametrize("m", W.DECODE_M)
def test_quantize_decode_activations_every_token_count(nv, m):
    """The decode activations at M = 1, 8 and 32 (the first rows of one draw):
    each token count has its own dynamic global scale, so each is compared."""
    _compare(nv, W.DECODE.x(m))


def test_quantize_long_prefill_activations_sampled_rows(nv):
    """32768 x 17408 (the standalone-quantize workload): the global scale comes
    from the whole tensor; codes and scales are compared on sampled rows."""
    import torch
    wl = W.LONG_DOWN
    xb = wl.x()
    x = to_cuda_bf16(xb)
    q, sf, s = nv.quantize_act(x)
    torch.cuda.synchronize()
    s_ref = oracle.global_scale(oracle.amax(xb))
    assert np.float32(s.item()).tobytes() == s_ref.tobytes()
    rows = np.unique(np.concatenate([np.arange(0, 128), np.random.default_rng(0).integers(0, wl.m, 128),
                                     np.arange(wl.m - 64, wl.m)]))
    qo, sfo = oracle.quantize(np.ascontiguousarray(xb[rows]), s_ref)
    qg = q[torch.as_tensor(rows, device="cuda")].cpu().numpy()
    assert np.array_equal(qg, qo)
    sf_h = sf.cpu().numpy()
    offs = np.array([[oracle.sf_offset(int(r), c, wl.k) for c in range(wl.k // 16)] for r in rows])
    assert np.array_equal(sf_h[offs], sfo)


@pytest.mark.parametrize("wl", [W.TINY, W.DECODE, W.PREFILL, W.FUSED_QKVG, W.LONG_DOWN], ids=lambda w: w.name)
def test_pack_weight_per_segment_scales(nv, wl):
    """Every workload's packed weight, in full: per-segment global scales, codes
    and scale bytes (pads included) equal to the oracle's."""
    import torch
    wb = wl.w()
    pw = nv.pack_weight(to_cuda_bf16(wb), wl.seg_offsets)
    torch.cuda.synchronize()
    s_ref = oracle.segment_scales(wb, wl.seg_offsets)
    assert pw.gscale.cpu().numpy().tobytes() == s_ref.tobytes()
    qo, sfo = oracle.quantize(wb, oracle.row_scales_from_segments(wl.seg_offsets, s_ref))
    assert np.array_equal(pw.q.cpu().numpy(), qo)
    assert np.array_equal(pw.sf.cpu().numpy(), oracle.sf_to_physical(sfo, wl.k))
