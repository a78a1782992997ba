"""Pins for the CPU oracle: each test checks the oracle against something other
than itself -- values the pages print (tests/golden/pages_values.json), a closed
form, a library routine (NumPy's half-to-even rounding, torch's float8 cast,
NumPy's fp64 matmul), or brute force on tiny inputs.  A plausible slip in the
oracle (dropped term, wrong sign or index, swapped operand, wrong tie rule)
fails at least one of them.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from nvfp4_w4a4_block_b200 import workloads as W

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "pages_values.json")))
E2M1_SET = GOLDEN["e2m1_magnitudes"]["value"]


# ---------------------------------------------------------------------------
# Number formats
# ---------------------------------------------------------------------------

def test_e2m1_decode_is_the_pages_value_set(oracle_mod):
    pos = [oracle_mod.e2m1_value(c) for c in range(8)]
    neg = [oracle_mod.e2m1_value(c | 8) for c in range(8)]
    assert pos == E2M1_SET
    assert neg == [-v for v in E2M1_SET]
    assert max(pos) == 6.0


def _e2m1_rne_numpy(v: np.ndarray) -> np.ndarray:
    """E2M1 round-to-nearest-even via NumPy's half-to-even np.round on each
    binade's grid step (0.5 below 2, 1 in [2,4), 2 from 4), clamped at 6."""
    a = np.abs(v.astype(np.float64))
    step = np.where(a < 2.0, 0.5, np.where(a < 4.0, 1.0, 2.0))
    r = np.minimum(np.round(a / step) * step, 6.0)
    return np.where(np.signbit(v), -r, r)


def test_e2m1_encode_matches_half_to_even_rounding(oracle_mod):
    bits = np.arange(0, 1 << 16, dtype=np.uint32).astype(np.uint16)
    vals = W.bf16_bits_to_f32(bits)
    vals = vals[np.isfinite(vals)]
    # every tie point and its fp32 neighbours, plus saturation
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], dtype=np.float32)
    near = np.concatenate([mids, np.nextafter(mids, np.float32(0)), np.nextafter(mids, np.float32(10))])
    extra = np.array([6.0, 6.5, 7.0, 100.0, 3e38, np.inf, 0.0], dtype=np.float32)
    vals = np.concatenate([vals, near, -near, extra, -extra])
    codes = np.array([oracle_mod.e2m1_encode(v) for v in vals])
    decoded = np.array([oracle_mod.e2m1_value(c) for c in codes])
    expect = _e2m1_rne_numpy(vals)
    assert np.array_equal(decoded, expect)
    # sign bit follows the sign of the input, zero results included
    assert np.array_equal((codes >> 3) & 1, np.signbit(vals).astype(int))


def test_e2m1_tie_cases():
    import oracle
    # Ties go to the even code: 0.25->0, 0.75->1, 1.25->1, 1.75->2, 2.5->2, 3.5->4, 5->4.
    expect = {0.25: 0x0, 0.75: 0x2, 1.25: 0x2, 1.75: 0x4, 2.5: 0x4, 3.5: 0x6, 5.0: 0x6}
    for v, c in expect.items():
        assert oracle.e2m1_encode(v) == c
        assert oracle.e2m1_encode(-v) == c | 8


def test_e4m3_decode_matches_torch_float8(oracle_mod):
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    mine = np.array([oracle_mod.e4m3_value(c) for c in range(256)])
    finite = np.isfinite(ref)
    assert not finite[0x7F] and not finite[0xFF]
    assert np.array_equal(np.isnan(mine), np.isnan(ref))
    assert np.array_equal(mine[finite], ref[finite])
    assert oracle_mod.e4m3_value(0x7E) == 448.0


def test_e4m3_encode_matches_torch_cast_in_range(oracle_mod):
    rng = np.random.default_rng(7)
    bits = np.arange(0, 1 << 15, dtype=np.uint32).astype(np.uint16)       # non-negative bf16
    b = W.bf16_bits_to_f32(bits)
    b = b[np.isfinite(b) & (b <= 448.0)]
    grid = np.array([oracle_mod.e4m3_value(c) for c in range(127)])
    mids = ((grid[1:] + grid[:-1]) / 2).astype(np.float32)
    near = np.concatenate([mids, np.nextafter(mids, np.float32(0)), np.nextafter(mids, np.float32(1e9))])
    rnd = (rng.random(20000) * 448).astype(np.float32)
    tiny = (rng.random(5000) * 2 ** -6).astype(np.float32)
    vals = np.concatenate([b, near[near <= 448], rnd, tiny])
    ref = torch.from_numpy(vals).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    mine = np.array([oracle_mod.e4m3_encode(v) for v in vals], dtype=np.uint8)
    assert np.array_equal(mine, ref)


def test_e4m3_encode_saturates(oracle_mod):
    for v in [448.0, 449.0, 463.9, 464.0, 480.0, 1e6, 3e38, float("inf")]:
        assert oracle_mod.e4m3_encode(v) == 0x7E


def test_e4m3_range_encoder_matches_the_scan_and_torch(oracle_mod):
    """The bulk E4M3 encoder over ranges of fp32 patterns (bisection over the
    table of E4M3 values) gives the scan's codes on a stride through every
    pattern of both signs, NaNs excluded, and torch's float8_e4m3fn cast
    wherever that cast does not overflow (|v| <= 448); every tie and near-tie
    of both signs is included."""
    start, count, step = 0, 1 << 32, 65521
    pats = np.arange(start, count, step, dtype=np.uint64).astype(np.uint32)
    grid = np.array([oracle_mod.e4m3_value(c) for c in range(127)])
    mids = ((grid[1:] + grid[:-1]) / 2).astype(np.float32)
    near = np.concatenate([mids, np.nextafter(mids, np.float32(0)), np.nextafter(mids, np.float32(1e9))])
    near = np.concatenate([near, -near]).view(np.uint32)
    got = np.concatenate([oracle_mod.e4m3_encode_range(int(p), 1) for p in near] +
                         [oracle_mod.e4m3_encode_range(0, 1 << 16)])
    vals = np.concatenate([near, np.arange(0, 1 << 16, dtype=np.uint32)])
    assert np.array_equal(got, oracle_mod.e4m3_encode_patterns(vals))
    f = pats.view(np.float32)
    pats = pats[~np.isnan(f)]
    got = np.empty(pats.size, np.uint8)
    for i, p in enumerate(pats):
        got[i] = oracle_mod.e4m3_encode_range(int(p), 1)[0]
    assert np.array_equal(got, oracle_mod.e4m3_encode_patterns(pats))
    f = pats.view(np.float32)
    ok = np.abs(f) <= 448.0
    ref = torch.from_numpy(f[ok].copy()).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(got[ok], ref)
    nf = near.view(np.float32)
    inside = np.abs(nf) <= 448.0
    assert inside.sum() > 700
    ref = torch.from_numpy(nf[inside].copy()).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got_near = np.concatenate([oracle_mod.e4m3_encode_range(int(p), 1) for p in near[inside]])
    assert np.array_equal(got_near, ref)


def test_e4m3_relative_rounding_error_closed_form(oracle_mod):
    """RNE to 3 mantissa bits: relative error <= 2^-4 in the normal range
    (the pages quote <= 6.2% for re-rounded block scales)."""
    bound = GOLDEN["e4m3_rerounding_bound"]["value"]
    rng = np.random.default_rng(3)
    vals = np.exp(rng.uniform(np.log(2 ** -6), np.log(448.0), 20000)).astype(np.float32)
    worst = 0.0
    for v in vals:
        q = oracle_mod.e4m3_value(oracle_mod.e4m3_encode(v))
        worst = max(worst, abs(q - float(v)) / float(v))
    assert worst <= 2.0 ** -4
    assert worst <= bound + 5e-4
    assert worst > 0.05          # the bound is tight, not vacuous


# ---------------------------------------------------------------------------
# Scales and the codec
# ---------------------------------------------------------------------------

def _bf16(a):
    return W.f32_to_bf16_bits(np.asarray(a, dtype=np.float32))


def test_two_level_identity_on_pages_example(oracle_mod):
    """max(block scale) x global x 6 reproduces the tensor absmax (model card
    §Verification prints 0.261719 = 0.261719)."""
    target = GOLDEN["two_level_identity_example"]["absmax"]
    rng = np.random.default_rng(11)
    w = rng.standard_normal((64, 512)).astype(np.float32) * 0.02
    w = np.clip(w, -0.25, 0.25)
    w[17, 301] = -target
    wb = _bf16(w)
    amax = float(oracle_mod.amax(wb))
    assert abs(amax - target) < 1e-6 * 4            # 0.26171875 in bf16
    q, sf, s = oracle_mod.quantize_dynamic(wb)
    smax = max(oracle_mod.e4m3_value(c) for c in np.unique(sf))
    assert smax == 448.0
    recon = smax * float(s) * 6.0
    assert round(recon, 6) == round(target, 6)
    assert abs(recon - amax) <= 2 * np.spacing(np.float32(amax))
    # the block holding the absmax carries the largest scale byte
    assert sf[17, 301 // 16] == 0x7E


@pytest.mark.parametrize("wl", [W.TINY, W.FUSED_QKVG], ids=lambda w: w.name)
def test_identity_holds_per_segment_for_workloads(oracle_mod, wl):
    w = wl.w() if wl.n * wl.k <= 64 * 2 ** 20 else None
    if w is None:
        pytest.skip("large")
    off = wl.seg_offsets
    s_w = oracle_mod.segment_scales(w, off)
    q, sf = oracle_mod.quantize(w, oracle_mod.row_scales_from_segments(off, s_w))
    for i in range(len(off) - 1):
        seg = sf[off[i]:off[i + 1]]
        assert seg.max() == 0x7E
        amax = float(oracle_mod.amax(w, off[i], off[i + 1]))
        assert abs(448.0 * float(s_w[i]) * 6.0 - amax) <= 2 * np.spacing(np.float32(amax))


def test_roundtrip_error_on_gaussian_weights_is_in_the_pages_range(oracle_mod):
    lo, hi = GOLDEN["roundtrip_relative_error"]["range"]
    wb = W.weights(99, (1024,), 1024, (0.02,))
    q, sf, s = oracle_mod.quantize_dynamic(wb)
    deq = oracle_mod.dequantize(q, sf, s)
    ref = W.bf16_bits_to_f32(wb).astype(np.float64)
    rel = np.linalg.norm(deq - ref) / np.linalg.norm(ref)
    assert lo <= rel <= hi, rel


def test_block_is_sixteen_elements_and_max_over_rms_bound(oracle_mod):
    """A one-hot block has max/RMS = sqrt(16) = 4 exactly, the pages' bound, and
    an outlier moves only its own block's scale and codes (its 15 neighbours)."""
    bs = GOLDEN["block_size"]["value"]
    onehot = np.zeros(bs)
    onehot[5] = 3.0
    assert math.isclose(np.abs(onehot).max() / np.sqrt(np.mean(onehot ** 2)),
                        GOLDEN["block_max_over_rms_bound"]["value"])
    rng = np.random.default_rng(5)
    x = rng.standard_normal((4, 256)).astype(np.float32)
    s = np.float32(2.0 ** -9)          # static global scale, shared by both runs
    q0, sf0 = oracle_mod.quantize(_bf16(x), s)
    x2 = x.copy()
    x2[2, 37] = 100.0                  # outlier in block 2 of row 2
    q1, sf1 = oracle_mod.quantize(_bf16(x2), s)
    diff_sf = np.argwhere(sf0 != sf1)
    assert diff_sf.tolist() == [[2, 37 // bs]]
    diff_q = np.argwhere(q0 != q1)
    assert all(r == 2 and (c * 2) // bs == 37 // bs for r, c in diff_q)
    assert len(diff_q) >= 1


def test_block_scale_is_blockmax_over_six(oracle_mod):
    """Scale byte = E4M3(blockmax / (6 s)); with power-of-two s and blockmax the
    scale is exact, e.g. blockmax 6*2^j under s = 2^-6 gives scale 2^(j+6)."""
    s = 2.0 ** -6
    for j in range(-8, 3):
        bmax = 6.0 * 2.0 ** j
        c = oracle_mod.block_scale(bmax, s)
        assert oracle_mod.e4m3_value(c) == 2.0 ** (j + 6)


def test_nibble_order_and_packing(oracle_mod):
    """Two codes per byte along K (model card: 2688 = 5376/2); lower K index in
    the low nibble."""
    pk = GOLDEN["packing"]["example"]
    x = np.zeros((1, pk["unpacked_k"]), np.float32)
    x[0, 0], x[0, 1] = 0.5, 6.0
    x[0, 2], x[0, 3] = -1.0, 3.0
    s = np.float32(1.0 / 256)              # blockmax 6 -> scale 256 -> divisor 1
    q, sf = oracle_mod.quantize(_bf16(x), s)
    assert q.shape[1] == pk["packed_bytes"]
    assert q[0, 0] == 0x71 and q[0, 1] == 0x5A
    assert oracle_mod.e4m3_value(sf[0, 0]) == 256.0


def test_exactly_representable_inputs_are_lossless(oracle_mod):
    """Values on the E2M1 grid times power-of-two block magnitudes, under a
    power-of-two global scale, survive quantize->dequantize exactly."""
    rng = np.random.default_rng(21)
    rows, k = 8, 256
    grid = np.array(E2M1_SET)
    vals = rng.choice(np.concatenate([grid, -grid]), size=(rows, k))
    for r in range(rows):
        for b in range(k // 16):
            vals[r, b * 16 + rng.integers(16)] = 6.0 * rng.choice([1, -1])
    mult = 2.0 ** rng.integers(-4, 3, size=(rows, k // 16))
    x = vals * np.repeat(mult, 16, axis=1)
    s = np.float32(2.0 ** -6)
    xb = _bf16(x)
    assert np.array_equal(W.bf16_bits_to_f32(xb).astype(np.float64), x)
    q, sf = oracle_mod.quantize(xb, s)
    assert np.array_equal(oracle_mod.dequantize(q, sf, s), x)


def test_zero_tensor_gives_zero_scales_and_codes(oracle_mod):
    xb = _bf16(np.zeros((3, 64)))
    q, sf, s = oracle_mod.quantize_dynamic(xb)
    assert s == 0.0 and not q.any() and not sf.any()


def test_saturating_static_scale(oracle_mod):
    """A static global scale far too small clamps every block scale at 448 and
    every code at +-6."""
    x = np.random.default_rng(2).standard_normal((2, 64)).astype(np.float32) + 3.0
    q, sf = oracle_mod.quantize(_bf16(x), np.float32(1e-6))
    assert (sf == 0x7E).all()
    lo, hi = q & 15, q >> 4
    assert ((lo & 7) == 7).all() and ((hi & 7) == 7).all()


# ---------------------------------------------------------------------------
# Scale-factor physical layout
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("rows,k", [(1, 64), (16, 256), (130, 320), (300, 1024)])
def test_sf_physical_layout_is_a_padded_bijection(oracle_mod, rows, k):
    nb = k // 16
    size = oracle_mod.sf_physical_bytes(rows, k)
    assert size == ((rows + 127) // 128 * 128) * ((nb + 3) // 4 * 4)
    offs = {oracle_mod.sf_offset(r, c, k) for r in range(rows) for c in range(nb)}
    assert len(offs) == rows * nb and max(offs) < size
    sf = np.arange(rows * nb, dtype=np.uint32).astype(np.uint8).reshape(rows, nb) | 1
    phys = oracle_mod.sf_to_physical(sf, k)
    mask = np.zeros(size, bool)
    mask[list(offs)] = True
    assert not phys[~mask].any()          # pads are zero
    # 512-byte atoms: 128 rows x 4 columns; row r%32 owns 16 contiguous bytes
    assert oracle_mod.sf_offset(0, 0, k) == 0
    assert oracle_mod.sf_offset(32, 0, k) == 4 and oracle_mod.sf_offset(1, 0, k) == 16
    if nb > 4:
        assert oracle_mod.sf_offset(0, 4, k) == 512


# ---------------------------------------------------------------------------
# GEMM
# ---------------------------------------------------------------------------

def test_gemm_equals_dense_fp64_matmul_on_representable_inputs(oracle_mod):
    rng = np.random.default_rng(31)
    m, n, k = 12, 40, 128
    grid = np.array(E2M1_SET + [-v for v in E2M1_SET])

    def rep(rows):
        v = rng.choice(grid, size=(rows, k))
        v[:, ::16] = 6.0
        return v * np.repeat(2.0 ** rng.integers(-3, 3, size=(rows, k // 16)), 16, axis=1)

    x, w = rep(m), rep(n)
    sx, sw = np.float32(2.0 ** -6), np.float32(2.0 ** -5)
    qx, sfx = oracle_mod.quantize(_bf16(x), sx)
    qw, sfw = oracle_mod.quantize(_bf16(w), sw)
    y = oracle_mod.linear_rows(qx, sfx, sx, np.arange(m), qw, sfw, np.full(n, sw, np.float32))
    ref = x @ w.T                 # quantization is lossless here
    assert np.array_equal(y, ref)


def test_gemm_matches_brute_force_on_tiny_random_inputs(oracle_mod):
    """Pure-Python triple loop; element values decoded with the pages' E2M1 value
    table and torch's float8_e4m3fn decode, not the oracle's decoders."""
    x, w, off = W.random_case(0, 3, 5, 32, seg_rows=[2, 3])
    ref = oracle_mod.linear_reference(x, w, off)
    s_x, s_w = float(ref["s_x"]), [float(v) for v in ref["s_w"]]
    e4 = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).tolist()

    def val(q, sf, r, j):
        byte = int(q[r, j // 2])
        code = (byte >> 4) if j % 2 else (byte & 15)
        mag = E2M1_SET[code & 7]
        return (-mag if code & 8 else mag) * e4[int(sf[r, j // 16])]

    for i in range(3):
        for c in range(5):
            seg = 0 if c < off[1] else 1
            acc = sum(val(ref["qx"], ref["sfx"], i, j) * val(ref["qw"], ref["sfw"], c, j) for j in range(32))
            assert math.isclose(acc * s_x * s_w[seg], ref["y"][i, c], rel_tol=1e-12, abs_tol=1e-300)


def test_fused_segments_equal_separate_modules(oracle_mod):
    x, w, off = W.random_case(1, 6, 48, 64, seg_rows=[16, 24, 8])
    fused = oracle_mod.linear_reference(x, w, off)
    for i in range(3):
        part = oracle_mod.linear_reference(x, np.ascontiguousarray(w[off[i]:off[i + 1]]), [0, off[i + 1] - off[i]])
        assert np.array_equal(part["y"], fused["y"][:, off[i]:off[i + 1]])
        assert part["s_w"][0] == fused["s_w"][i]


def test_collapsed_max_scale_is_the_pages_mismatch(oracle_mod):
    """Negative control: serving a fused group with the max of the module scales
    and unchanged block scales mis-scales every other segment by its ratio
    (the pages report errors of 0.35 / 0.57 for ratios 1.82x / 2.75x); the
    per-segment epilogue has none of that error."""
    probe = GOLDEN["fused_mismatch_probe"]
    x, w, _ = W.random_case(2, 8, 64, 128)
    off = [0, 32, 64]
    wf = W.bf16_bits_to_f32(w).copy()
    ratio = probe["paired_scale_ratios"][1]
    wf[32:] *= ratio
    w = W.f32_to_bf16_bits(wf)
    good = oracle_mod.linear_reference(x, w, off)
    s_w = good["s_w"]
    assert 2.5 < s_w[1] / s_w[0] < 3.0
    collapsed_cols = np.full(64, s_w.max(), np.float32)
    bad = oracle_mod.linear_rows(good["qx"], good["sfx"], good["s_x"], np.arange(8), good["qw"], good["sfw"],
                                 collapsed_cols)
    ref = good["y"]
    err0 = np.linalg.norm(bad[:, :32] - ref[:, :32]) / np.linalg.norm(ref[:, :32])
    err1 = np.linalg.norm(bad[:, 32:] - ref[:, 32:]) / np.linalg.norm(ref[:, 32:])
    assert abs(err0 - (s_w[1] / s_w[0] - 1)) < 1e-6       # mis-scaled by the ratio
    assert err1 == 0.0
    assert err0 > max(probe["mismatched"])                # O(1e-1) or worse, as reported


def test_tiny_workload_matches_committed_oracle_output(oracle_mod):
    """Regression guard: the committed tiny-workload values (written by
    tests/golden/make_golden.py from the oracle) still come out of it."""
    g = np.load(os.path.join(os.path.dirname(__file__), "golden", "tiny_expected.npz"))
    wl = W.TINY
    x, w = wl.x(), wl.w()
    assert np.array_equal(x, g["x"]) and np.array_equal(w, g["w"])
    ref = oracle_mod.linear_reference(x, w, wl.seg_offsets)
    for key in ("qx", "sfx", "qw", "sfw", "s_w", "y"):
        assert np.array_equal(ref[key], g[key]), key
    assert ref["s_x"] == g["s_x"]
