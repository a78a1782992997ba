"""Seeded synthetic inputs for the NVFP4 W4A4 linear layer.

This module only draws random numbers and shapes them; it holds none of the
quantization arithmetic, so both the CPU oracle (tests only) and the CUDA path
can consume the very same bytes.

Distributions follow the workloads of "Why Gated DeltaNet Survives 4-Bit
Quantization" (hybrid 27B model, hidden size 5120, §2 "Gated DeltaNet in
Qwen3.8-27B"; residual-stream activations with extreme outlier channels,
§5.1 Table 2: hot channels ~100x the median channel, kurtosis ~1,560; weights
near-Gaussian).  The captured activations and the released checkpoints are not
available, so seeded draws stand in for them:

* activations: N(0,1) rows (or Student-t with nu=3 for the heavy-tailed
  prefill case) with a fixed set of outlier channels (columns) scaled up;
* weights: N(0, sigma) with sigma = 0.02 per module; fused modules use a
  different sigma per segment so that their calibrated global scales differ
  (§6 "Per-module calibration vs. fused-GEMM scaling": 1.82x / 2.75x).

Every array is drawn with NumPy's PCG64 from SeedSequence([cfg_id, tensor_id])
in float32 and rounded to bfloat16 (round-to-nearest-even via torch); tensors
are returned as uint16 bit patterns so callers can hand identical bytes to
either side.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List, Optional, Sequence

import numpy as np
import torch

# Tensor ids inside one configuration's seed sequence.
_T_X = 0
_T_W = 1
_T_OUTLIER_COLS = 2


def rng_for(cfg_id: int, tensor_id: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([cfg_id, tensor_id])))


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 -> bfloat16 (RNE, torch's cast) and return the uint16 bit patterns."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bfloat16 bit patterns to float32."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _normal(rng: np.random.Generator, shape, sigma: float = 1.0) -> np.ndarray:
    out = rng.standard_normal(size=shape, dtype=np.float32)
    if sigma != 1.0:
        out *= np.float32(sigma)
    return out


def activations(cfg_id: int, m: int, k: int, dist: str = "normal",
                outlier_frac: float = 0.0, outlier_mult: float = 1.0) -> np.ndarray:
    """X [m, k] as bf16 bits.

    dist: "normal" (N(0,1)) or "student_t3" (standard t, nu=3, not renormalised).
    outlier_frac of the k channels (rounded, at least 1 when frac > 0), drawn
    without replacement from the config's seed, are multiplied by outlier_mult.
    """
    rng = rng_for(cfg_id, _T_X)
    if dist == "normal":
        x = _normal(rng, (m, k))
    elif dist == "student_t3":
        x = rng.standard_t(3, size=(m, k)).astype(np.float32)
    else:
        raise ValueError(f"unknown distribution {dist!r}")
    if outlier_frac > 0.0:
        n_out = max(1, int(round(outlier_frac * k)))
        cols = np.sort(rng_for(cfg_id, _T_OUTLIER_COLS).choice(k, size=n_out, replace=False))
        x[:, cols] *= np.float32(outlier_mult)
    return f32_to_bf16_bits(x)


def weights(cfg_id: int, seg_rows: Sequence[int], k: int, seg_sigma: Sequence[float]) -> np.ndarray:
    """W [sum(seg_rows), k] as bf16 bits; segment s ~ N(0, seg_sigma[s])."""
    rng = rng_for(cfg_id, _T_W)
    parts = [_normal(rng, (r, k), s) for r, s in zip(seg_rows, seg_sigma)]
    return f32_to_bf16_bits(np.concatenate(parts, axis=0))


@dataclasses.dataclass(frozen=True)
class Workload:
    """One linear-layer problem: Y[m, n] = X[m, :] . W[n, :] over K."""
    name: str
    cfg_id: int
    m: int
    k: int
    seg_rows: tuple          # rows of W per fused module (segment), concatenated along N
    seg_sigma: tuple         # weight std-dev per segment
    x_dist: str = "normal"
    outlier_frac: float = 0.0
    outlier_mult: float = 1.0

    @property
    def n(self) -> int:
        return int(sum(self.seg_rows))

    @property
    def seg_offsets(self) -> List[int]:
        off = [0]
        for r in self.seg_rows:
            off.append(off[-1] + int(r))
        return off

    def x(self, m: Optional[int] = None) -> np.ndarray:
        """Activations; the first m rows of the config's draw when m < self.m."""
        full = activations(self.cfg_id, self.m, self.k, self.x_dist, self.outlier_frac, self.outlier_mult)
        return full if m is None else np.ascontiguousarray(full[:m])

    def w(self) -> np.ndarray:
        return weights(self.cfg_id, self.seg_rows, self.k, self.seg_sigma)

    def flops(self, m: Optional[int] = None) -> float:
        return 2.0 * (self.m if m is None else m) * self.n * self.k


# The five problem shapes (hybrid 27B-class dimensions, hidden size 5120).
TINY = Workload("tiny_16x256x128", 0, 16, 256, (128,), (0.02,))
DECODE = Workload("decode_fused_gate_up_M32_K5120_N34816", 1, 32, 5120, (17408, 17408), (0.02, 0.02 * 2.75),
                  "normal", 0.005, 50.0)
PREFILL = Workload("prefill_up_proj_M8192_K5120_N17408", 2, 8192, 5120, (17408,), (0.02,),
                   "student_t3", 0.001, 100.0)
FUSED_QKVG = Workload("fused_qkv_gate_M4096_K5120_N10336", 3, 4096, 5120, (6144, 2048, 2048, 96),
                      (0.02, 0.04, 0.08, 0.16), "normal", 0.005, 50.0)
LONG_DOWN = Workload("long_prefill_down_proj_M32768_K17408_N5120", 4, 32768, 17408, (5120,), (0.02,),
                     "normal", 0.005, 50.0)

ALL: Dict[str, Workload] = {w.name: w for w in (TINY, DECODE, PREFILL, FUSED_QKVG, LONG_DOWN)}
DECODE_M = (1, 8, 32)


def random_case(seed: int, m: int, n: int, k: int, seg_rows: Optional[Sequence[int]] = None,
                x_sigma: float = 1.0, w_sigma: float = 0.02):
    """Small seeded case for parity sweeps: returns (x_bits, w_bits, seg_offsets)."""
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([1000 + seed, m, n, k])))
    x = rng.standard_normal(size=(m, k), dtype=np.float32) * np.float32(x_sigma)
    segs = list(seg_rows) if seg_rows is not None else [n]
    parts = []
    for i, r in enumerate(segs):
        parts.append(rng.standard_normal(size=(r, k), dtype=np.float32) * np.float32(w_sigma * (1 + i)))
    w = np.concatenate(parts, axis=0) if parts else np.zeros((0, k), np.float32)
    off = [0]
    for r in segs:
        off.append(off[-1] + r)
    return f32_to_bf16_bits(x), f32_to_bf16_bits(w), off
