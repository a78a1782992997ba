"""Test-side helpers: moving seeded bf16 bit patterns to the GPU and the
tolerance metric of the GEMM parity tests (no method arithmetic here)."""
import numpy as np

# GEMM tolerance.  The accumulation error allowed against the fp64 oracle is
# 1e-3 of max(|R|, RMS of R's row) (the row-RMS floor keeps near-cancelled
# outputs from making a relative error undefined).  A bf16 output adds its own
# round-to-nearest-even error, at most 2^-8 of the value (8 significant bits).
GEMM_REL_TOL = 1e-3
BF16_ROUNDING = 2.0 ** -8


def to_cuda_bf16(bits: np.ndarray):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(bits, dtype=np.uint16).view(np.int16))
    return t.view(torch.bfloat16).cuda()


def scaled_error(y: np.ndarray, ref: np.ndarray) -> np.ndarray:
    """|y - ref| / max(|ref|, rms of ref's row), elementwise."""
    ref = np.asarray(ref, dtype=np.float64)
    rms = np.sqrt(np.mean(ref * ref, axis=1, keepdims=True))
    floor = np.maximum(np.abs(ref), rms)
    floor = np.where(floor == 0, 1.0, floor)
    return np.abs(np.asarray(y, dtype=np.float64) - ref) / floor


def assert_gemm_close(y, ref, bf16: bool):
    y = np.asarray(y, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert y.shape == ref.shape
    assert np.isfinite(y).all()
    rms = np.sqrt(np.mean(ref * ref, axis=1, keepdims=True))
    floor = np.where(np.maximum(np.abs(ref), rms) == 0, 1.0, np.maximum(np.abs(ref), rms))
    allowed = GEMM_REL_TOL * floor + (BF16_ROUNDING * np.abs(ref) if bf16 else 0.0)
    bad = np.abs(y - ref) > allowed
    if bad.any():
        i = np.argwhere(bad)[0]
        raise AssertionError(f"{bad.sum()} elements out of tolerance; first {tuple(i)}: "
                             f"y={y[tuple(i)]!r} ref={ref[tuple(i)]!r} "
                             f"max scaled err={scaled_error(y, ref).max():.3e}")


def bf16_rne_from_f32(y32: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (torch's RNE cast), returned as uint16 bits."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(y32, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)
