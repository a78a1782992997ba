"""Pins for the oracle's three off-path steps: dequantization to bf16 (the model
card's expansion of a packed checkpoint to BF16), harmonization of a fused
group (the checkpoint-side repair of "Why Gated DeltaNet Survives 4-Bit
Quantization", §6), and checkpoint import of a linear-layout block-scale matrix.

Each oracle function is checked against something other than itself: brute
force over every bf16 value, torch's fp32->bf16 cast, exact rational
arithmetic, the E4M3 half-ulp bound the paper quotes (<= 6.2%), exactness of
power-of-two folds, and the paper's qualitative before/after of the fused-GEMM
probe.
"""
import json
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

from nvfp4_w4a4_block_b200 import workloads as W

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "pages_values.json")))


def _bf16(a):
    return W.f32_to_bf16_bits(np.asarray(a, dtype=np.float32))


def _all_bf16_magnitudes():
    """Every finite non-negative bf16 value, ascending, with its bit pattern."""
    bits = np.arange(0, 0x7F80, dtype=np.uint32)
    vals = (bits << 16).view(np.float32).astype(np.float64)
    return bits.astype(np.uint16), vals


def _brute_bf16(v: float, bits, vals) -> int:
    """Nearest bf16 by search over the whole table; ties to the even pattern."""
    sign = 0x8000 if np.signbit(v) else 0
    a = abs(v)
    top = vals[-1]
    half_ulp_top = (vals[-1] - vals[-2]) / 2
    if a >= top + half_ulp_top:
        return sign | 0x7F80
    i = int(np.searchsorted(vals, a))
    cands = [j for j in (i - 1, i) if 0 <= j < len(vals)]
    best = min(cands, key=lambda j: (abs(vals[j] - a), int(bits[j]) & 1))
    return sign | int(bits[best])


# ---------------------------------------------------------------------------
# bf16 rounding of an exact value
# ---------------------------------------------------------------------------

def test_bf16_rounding_matches_brute_force_search(oracle_mod):
    bits, vals = _all_bf16_magnitudes()
    rng = np.random.default_rng(5)
    xs = list(np.ldexp(rng.uniform(0.5, 1.0, 3000), rng.integers(-140, 129, 3000)))
    # exact midpoints between neighbours (ties), and points just either side of them
    idx = rng.integers(1, len(vals) - 1, 600)
    mids = (vals[idx] + vals[idx + 1]) / 2
    xs += list(mids) + list(np.nextafter(mids, 0)) + list(np.nextafter(mids, np.inf))
    xs += [0.0, -0.0, vals[1] / 2, vals[1] * 1.5, vals[-1], vals[-1] * (1 + 2 ** -9), 1e39]
    for i, x in enumerate(xs):
        x = float(x) * (-1.0 if i % 3 == 0 else 1.0)
        assert oracle_mod.bf16_from_f64(x) == _brute_bf16(x, bits, vals), x


def test_bf16_rounding_agrees_with_torch_cast_of_fp32(oracle_mod):
    rng = np.random.default_rng(6)
    x32 = (rng.standard_normal(20000) * np.exp(rng.uniform(-30, 30, 20000))).astype(np.float32)
    ref = torch.from_numpy(x32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([oracle_mod.bf16_from_f64(float(v)) for v in x32], dtype=np.uint16)
    assert np.array_equal(got, ref)


# ---------------------------------------------------------------------------
# Dequantization to bf16 (expansion of a packed tensor)
# ---------------------------------------------------------------------------

def test_dequantize_bf16_values_are_exact_products_rounded_once(oracle_mod):
    """Element (r, j) is the bf16 nearest to code value x block scale x global
    scale, the product taken in exact rational arithmetic."""
    bits, vals = _all_bf16_magnitudes()
    rng = np.random.default_rng(7)
    rows, k = 5, 64
    q = rng.integers(0, 256, (rows, k // 2), dtype=np.uint8)
    sf = rng.integers(0, 0x7F, (rows, k // 16), dtype=np.uint8)
    s = np.array([0.013, 1.7e-3, 3.1, 1.0, 2.0 ** -20], dtype=np.float32)
    out = oracle_mod.dequantize_bf16(q, sf, s)
    e2m1 = GOLDEN["e2m1_magnitudes"]["value"]
    for r in range(rows):
        for j in range(k):
            code = (q[r, j // 2] >> (4 * (j & 1))) & 15
            mag = Fraction(e2m1[code & 7]) * (-1 if code & 8 else 1)
            sc = Fraction(oracle_mod.e4m3_value(int(sf[r, j // 16])))
            exact = mag * sc * Fraction(float(s[r]))
            want = _brute_bf16(float(exact), bits, vals) if exact != 0 else (0x8000 if code & 8 else 0)
            # float(exact) is exact: at most 2 + 4 + 24 significant bits
            assert Fraction(float(exact)) == exact
            assert out[r, j] == want, (r, j)


def test_dequantize_bf16_inverts_quantize_on_representable_inputs(oracle_mod):
    """Grid values under power-of-two block and global scales come back bit for bit."""
    rng = np.random.default_rng(8)
    rows, k = 6, 128
    grid = np.array(GOLDEN["e2m1_magnitudes"]["value"])
    vals = rng.choice(np.concatenate([grid, -grid]), size=(rows, k))
    for r in range(rows):
        for b in range(k // 16):
            vals[r, b * 16 + rng.integers(16)] = 6.0 * rng.choice([1, -1])
    x = vals * np.repeat(2.0 ** rng.integers(-6, 2, size=(rows, k // 16)), 16, axis=1)
    xb = _bf16(x)
    q, sf = oracle_mod.quantize(xb, np.float32(2.0 ** -7))
    out = oracle_mod.dequantize_bf16(q, sf, np.float32(2.0 ** -7))
    nz = W.bf16_bits_to_f32(xb) != 0
    assert np.array_equal(out[nz], xb[nz])
    assert (W.bf16_bits_to_f32(out[~nz]) == 0).all()


def test_dequantize_bf16_roundtrip_error_is_in_the_pages_range(oracle_mod):
    """Quantize then expand N(0, 0.02) weights: relative error 4-10% (model card)."""
    lo, hi = GOLDEN["roundtrip_relative_error"]["range"]
    w = W.weights(9, [256], 512, [0.02])
    s = oracle_mod.global_scale(oracle_mod.amax(w))
    q, sf = oracle_mod.quantize(w, s)
    back = W.bf16_bits_to_f32(oracle_mod.dequantize_bf16(q, sf, s)).astype(np.float64)
    ref = W.bf16_bits_to_f32(w).astype(np.float64)
    rel = np.linalg.norm(back - ref) / np.linalg.norm(ref)
    assert lo <= rel <= hi


# ---------------------------------------------------------------------------
# Harmonization of a fused group
# ---------------------------------------------------------------------------

def _fused_weight(seed, seg_rows, k, sigmas):
    w = W.weights(seed, seg_rows, k, sigmas)
    off = [int(v) for v in np.concatenate([[0], np.cumsum(seg_rows)])]
    return w, off


def test_harmonize_keeps_the_largest_module_and_bounds_rerounding(oracle_mod):
    """The module with the largest scale is untouched; every other block scale
    is re-rounded by at most E4M3's half ulp (2^-4 relative, the paper's
    <= 6.2%) wherever the folded value is a normal E4M3 number."""
    bound = GOLDEN["e4m3_rerounding_bound"]["value"]
    w, off = _fused_weight(11, [64, 32, 40, 8], 256, [0.02, 0.02 * 1.82, 0.02 * 2.75, 0.02 * 0.5])
    s = oracle_mod.segment_scales(w, off)
    q, sf = oracle_mod.quantize(w, oracle_mod.row_scales_from_segments(off, s))
    new, shared = oracle_mod.harmonize(sf, off, s)
    assert shared == s.max()
    top = int(np.argmax(s))
    assert np.array_equal(new[off[top]:off[top + 1]], sf[off[top]:off[top + 1]])
    for i in range(len(s)):
        ratio = np.float32(s[i]) / np.float32(shared)
        old_v = np.vectorize(oracle_mod.e4m3_value)(sf[off[i]:off[i + 1]])
        new_v = np.vectorize(oracle_mod.e4m3_value)(new[off[i]:off[i + 1]])
        target = old_v * float(ratio)
        normal = target >= 2.0 ** -6
        rel = np.abs(new_v[normal] - target[normal]) / target[normal]
        assert rel.max() <= 2.0 ** -4 and rel.max() <= bound + 5e-4
        assert (new_v <= 448.0).all()
        # subnormal range: within half of the subnormal step 2^-9
        assert (np.abs(new_v[~normal] - target[~normal]) <= 2.0 ** -10 + 1e-12).all()


def test_harmonize_power_of_two_ratios_are_lossless(oracle_mod):
    """When every module scale is the largest divided by a power of two, folding
    is exact: the expanded weights under the shared scale equal the expanded
    weights under the per-module scales (normal-range blocks)."""
    w = W.weights(12, [32, 32, 32], 128, [0.02, 0.02, 0.02])
    off = [0, 32, 64, 96]
    s = np.array([2.0 ** -9, 2.0 ** -10, 2.0 ** -12], np.float32)
    q, sf = oracle_mod.quantize(w, oracle_mod.row_scales_from_segments(off, s))
    new, shared = oracle_mod.harmonize(sf, off, s)
    assert shared == np.float32(2.0 ** -9)
    before = oracle_mod.dequantize(q, sf, oracle_mod.row_scales_from_segments(off, s))
    after = oracle_mod.dequantize(q, new, shared)
    folded_ok = np.repeat(np.vectorize(oracle_mod.e4m3_value)(sf) *
                          np.repeat(s / shared, [32, 32, 32])[:, None] >= 2.0 ** -6, 16, axis=1)
    assert folded_ok.mean() > 0.9
    assert np.array_equal(before[folded_ok], after[folded_ok])


def test_harmonize_rejects_non_finite_or_negative_scales(oracle_mod):
    sf = np.full((16, 4), 0x38, np.uint8)
    for bad in ([1.0, float("nan")], [1.0, float("inf")], [1.0, -0.5]):
        new, shared = oracle_mod.harmonize(sf, [0, 8, 16], bad)
        assert np.isnan(shared) and np.array_equal(new, sf)
    new, shared = oracle_mod.harmonize(sf, [0, 8, 16], [0.0, 0.0])
    assert shared == 0.0 and np.array_equal(new, sf)


def test_harmonize_keeps_nan_scale_bytes(oracle_mod):
    """A NaN block-scale byte (E4M3 0x7F, or 0xFF with the sign bit set), which
    only a corrupt checkpoint could hold, stays as it is: NaN times any module
    ratio is NaN under IEEE rules (checked here with NumPy's float32 product),
    and E4M3's one NaN code per sign encodes it.  Every other byte folds exactly
    as it does without the NaN bytes present."""
    w, off = _fused_weight(13, [32, 48], 128, [0.02, 0.02 * 2.75])
    s = oracle_mod.segment_scales(w, off)
    q, sf = oracle_mod.quantize(w, oracle_mod.row_scales_from_segments(off, s))
    planted = [(3, 5, 0x7F), (off[1] + 2, 0, 0xFF), (off[1] + 40, 7, 0x7F)]
    sf_nan = sf.copy()
    for r, c, b in planted:
        sf_nan[r, c] = b
    new, shared = oracle_mod.harmonize(sf, off, s)
    new_nan, shared_nan = oracle_mod.harmonize(sf_nan, off, s)
    assert shared_nan == shared
    keep = np.ones(sf.shape, bool)
    for r, c, b in planted:
        seg = int(np.searchsorted(off, r, side="right")) - 1
        ratio = np.float32(s[seg]) / np.float32(shared)
        assert np.isnan(np.float32(oracle_mod.e4m3_value(b)) * ratio)
        assert new_nan[r, c] == b
        keep[r, c] = False
    assert np.array_equal(new_nan[keep], new[keep])


def test_harmonized_gemm_repairs_the_collapsed_mismatch(oracle_mod):
    """The paper's GEMM-level probe: serving a fused group with the largest
    module scale and unchanged block scales is off by the scale ratio
    (0.35 / 0.57 in the paper); after folding the ratios into the block scales
    the one-scale GEMM is back within the re-rounding error of the per-module
    result, and exact on the module that owns the largest scale."""
    probe = GOLDEN["fused_mismatch_probe"]
    x, _, _ = W.random_case(13, 16, 64, 256)
    r1, r2 = probe["paired_scale_ratios"]
    w = W.weights(13, [64, 64, 64], 256, [0.02, 0.02 * r1, 0.02 * r2])
    off = [0, 64, 128, 192]
    good = oracle_mod.linear_reference(x, w, off)
    s_w = good["s_w"]
    rows = np.arange(16)
    ref = good["y"]
    collapsed = oracle_mod.linear_rows(good["qx"], good["sfx"], good["s_x"], rows, good["qw"], good["sfw"],
                                       np.full(192, s_w.max(), np.float32))
    new, shared = oracle_mod.harmonize(good["sfw"], off, s_w)
    repaired = oracle_mod.linear_rows(good["qx"], good["sfx"], good["s_x"], rows, good["qw"], new,
                                      np.full(192, shared, np.float32))

    def err(y, i):
        a, b = off[i], off[i + 1]
        return np.linalg.norm(y[:, a:b] - ref[:, a:b]) / np.linalg.norm(ref[:, a:b])

    top = int(np.argmax(s_w))
    for i in range(3):
        if i == top:
            assert err(collapsed, i) == 0.0 and err(repaired, i) == 0.0
        else:
            assert err(collapsed, i) > min(probe["mismatched"])
            assert err(repaired, i) < 2.0 ** -4


# ---------------------------------------------------------------------------
# Checkpoint import
# ---------------------------------------------------------------------------

def test_import_of_a_linear_scale_matrix_is_the_tensor_core_scatter(oracle_mod):
    """A checkpoint's [rows, K/16] block-scale matrix lands where the physical
    layout puts logical (r, c): checked byte by byte against the layout rule
    written out, pads zero."""
    rows, k = 200, 320
    rng = np.random.default_rng(14)
    lin = rng.integers(1, 0x7F, (rows, k // 16), dtype=np.uint8)
    phys = oracle_mod.import_scales(lin, k)
    cols_pad = (k // 16 + 3) // 4 * 4
    assert phys.size == (rows + 127) // 128 * 128 * cols_pad
    seen = np.zeros(phys.size, bool)
    for r in range(rows):
        for c in range(k // 16):
            atom = (r // 128) * (cols_pad // 4) + c // 4
            off = atom * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + c % 4
            assert phys[off] == lin[r, c]
            seen[off] = True
    assert not phys[~seen].any()
