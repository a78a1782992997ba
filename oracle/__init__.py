"""CPU oracle for the NVFP4 W4A4 linear layer -- TEST INFRASTRUCTURE ONLY.

Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg may import
this package.  The product path (the CUDA library and its Python binding) never
does.  The arithmetic lives in nvfp4_oracle.c (plain C, fp64 GEMM); this module
builds it with gcc and marshals NumPy arrays in and out.  See that file's header
for the passages each step follows and the readings taken where the pages are
silent.

Parity status: every function here is pinned by tests/test_oracle_pins.py
(pages' values, closed forms, library routines, brute force).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "nvfp4_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

_lib = None


def build(force: bool = False) -> str:
    """Compile nvfp4_oracle.c into liboracle.so (gcc, OpenMP, no FP contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-ffp-contract=off",
                               "-fno-fast-math", "-std=c11", "-Wall", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        i64, u32, f32, f64, vp = ctypes.c_int64, ctypes.c_uint32, ctypes.c_float, ctypes.c_double, ctypes.c_void_p
        lib.or_e2m1_value.argtypes, lib.or_e2m1_value.restype = [u32], f64
        lib.or_e4m3_value.argtypes, lib.or_e4m3_value.restype = [u32], f64
        lib.or_e2m1_encode.argtypes, lib.or_e2m1_encode.restype = [f32], u32
        lib.or_e4m3_encode.argtypes, lib.or_e4m3_encode.restype = [f32], u32
        lib.or_amax_bf16.argtypes, lib.or_amax_bf16.restype = [vp, i64, i64, i64, i64], f32
        lib.or_global_scale.argtypes, lib.or_global_scale.restype = [f32], f32
        lib.or_block_scale.argtypes, lib.or_block_scale.restype = [f32, f32], u32
        lib.or_quantize.argtypes, lib.or_quantize.restype = [vp, i64, i64, i64, vp, vp, vp], None
        lib.or_dequantize.argtypes, lib.or_dequantize.restype = [vp, vp, i64, i64, vp, vp], None
        lib.or_sf_physical_bytes.argtypes, lib.or_sf_physical_bytes.restype = [i64, i64], i64
        lib.or_sf_offset.argtypes, lib.or_sf_offset.restype = [i64, i64, i64], i64
        lib.or_sf_to_physical.argtypes, lib.or_sf_to_physical.restype = [vp, i64, i64, vp], None
        lib.or_linear_rows.argtypes = [vp, vp, f32, vp, i64, vp, vp, vp, i64, i64, vp]
        lib.or_linear_rows.restype = None
        lib.or_num_threads.argtypes, lib.or_num_threads.restype = [], ctypes.c_int
        lib.or_bf16_from_f64.argtypes, lib.or_bf16_from_f64.restype = [f64], ctypes.c_uint16
        lib.or_dequantize_bf16.argtypes, lib.or_dequantize_bf16.restype = [vp, vp, i64, i64, vp, vp], None
        lib.or_harmonize.argtypes, lib.or_harmonize.restype = [vp, i64, i64, vp, ctypes.c_int, vp], f32
        lib.or_e2m1_encode_patterns.argtypes = [ctypes.c_uint64, ctypes.c_uint64, vp]
        lib.or_e2m1_encode_patterns.restype = None
        lib.or_e4m3_encode_patterns.argtypes, lib.or_e4m3_encode_patterns.restype = [vp, i64, vp], None
        lib.or_e4m3_encode_range.argtypes = [ctypes.c_uint64, ctypes.c_uint64, vp]
        lib.or_e4m3_encode_range.restype = None
        _lib = lib
    return _lib


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"], "oracle expects C-contiguous arrays"
    return a.ctypes.data


# --- formats ---------------------------------------------------------------

def e2m1_value(code: int) -> float:
    return _load().or_e2m1_value(int(code))


def e4m3_value(code: int) -> float:
    return _load().or_e4m3_value(int(code))


def e2m1_encode(v: float) -> int:
    return int(_load().or_e2m1_encode(float(v)))


def e4m3_encode(v: float) -> int:
    return int(_load().or_e4m3_encode(float(v)))


def e2m1_encode_patterns(start: int, count: int) -> np.ndarray:
    """E2M1 codes of the fp32 bit patterns start .. start+count-1 (one byte each)."""
    out = np.empty(count, dtype=np.uint8)
    _load().or_e2m1_encode_patterns(start, count, _ptr(out))
    return out


def e4m3_encode_range(start: int, count: int) -> np.ndarray:
    """E4M3 codes of the fp32 bit patterns start .. start+count-1 (one byte each)."""
    out = np.empty(count, dtype=np.uint8)
    _load().or_e4m3_encode_range(start, count, _ptr(out))
    return out


def e4m3_encode_patterns(pats: np.ndarray) -> np.ndarray:
    """E4M3 codes of the given fp32 bit patterns."""
    pats = np.ascontiguousarray(pats, dtype=np.uint32)
    out = np.empty(pats.size, dtype=np.uint8)
    _load().or_e4m3_encode_patterns(_ptr(pats), pats.size, _ptr(out))
    return out


def num_threads() -> int:
    return int(_load().or_num_threads())


# --- scales ----------------------------------------------------------------

def amax(x_bits: np.ndarray, r0: int = 0, r1: Optional[int] = None) -> np.float32:
    x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
    rows, k = x_bits.shape
    r1 = rows if r1 is None else r1
    return np.float32(_load().or_amax_bf16(_ptr(x_bits), r0, r1, k, k))


def global_scale(a: float) -> np.float32:
    """Per-tensor FP32 global scale = amax / (6 * 448) (dequantization multiplier)."""
    return np.float32(_load().or_global_scale(float(a)))


def block_scale(bmax: float, s: float) -> int:
    return int(_load().or_block_scale(float(bmax), float(s)))


def segment_scales(w_bits: np.ndarray, seg_offsets: Sequence[int]) -> np.ndarray:
    """Global scale of each segment (module) of a row-concatenated weight."""
    return np.array([global_scale(amax(w_bits, seg_offsets[i], seg_offsets[i + 1]))
                     for i in range(len(seg_offsets) - 1)], dtype=np.float32)


def row_scales_from_segments(seg_offsets: Sequence[int], seg_scale: Sequence[float]) -> np.ndarray:
    rows = seg_offsets[-1]
    out = np.empty(rows, dtype=np.float32)
    for i in range(len(seg_offsets) - 1):
        out[seg_offsets[i]:seg_offsets[i + 1]] = np.float32(seg_scale[i])
    return out


# --- quantization ----------------------------------------------------------

def quantize(x_bits: np.ndarray, row_scale) -> tuple:
    """Returns (q [rows, k/2] uint8, sf [rows, k/16] uint8 logical)."""
    x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
    rows, k = x_bits.shape
    assert k % 16 == 0
    rs = np.ascontiguousarray(np.broadcast_to(np.asarray(row_scale, dtype=np.float32), (rows,)))
    q = np.zeros((rows, k // 2), dtype=np.uint8)
    sf = np.zeros((rows, k // 16), dtype=np.uint8)
    if rows:
        _load().or_quantize(_ptr(x_bits), rows, k, k, _ptr(rs), _ptr(q), _ptr(sf))
    return q, sf


def quantize_dynamic(x_bits: np.ndarray) -> tuple:
    """Dynamic per-tensor mode: s = amax/2688, then quantize. Returns (q, sf, s)."""
    s = global_scale(amax(x_bits))
    q, sf = quantize(x_bits, s)
    return q, sf, s


def dequantize(q: np.ndarray, sf: np.ndarray, row_scale) -> np.ndarray:
    q = np.ascontiguousarray(q, dtype=np.uint8)
    sf = np.ascontiguousarray(sf, dtype=np.uint8)
    rows = q.shape[0]
    k = q.shape[1] * 2
    rs = np.ascontiguousarray(np.broadcast_to(np.asarray(row_scale, dtype=np.float32), (rows,)))
    out = np.zeros((rows, k), dtype=np.float64)
    if rows:
        _load().or_dequantize(_ptr(q), _ptr(sf), rows, k, _ptr(rs), _ptr(out))
    return out


def sf_physical_bytes(rows: int, k: int) -> int:
    return int(_load().or_sf_physical_bytes(rows, k))


def sf_offset(r: int, c: int, k: int) -> int:
    return int(_load().or_sf_offset(r, c, k))


def sf_to_physical(sf: np.ndarray, k: int) -> np.ndarray:
    sf = np.ascontiguousarray(sf, dtype=np.uint8)
    rows = sf.shape[0]
    phys = np.zeros(sf_physical_bytes(rows, k), dtype=np.uint8)
    _load().or_sf_to_physical(_ptr(sf), rows, k, _ptr(phys))
    return phys


def import_scales(sf_linear: np.ndarray, k: int) -> np.ndarray:
    """Checkpoint import (R16): a linear-layout block-scale matrix [rows, k/16]
    is the logical matrix; its physical form is the R10 scatter of it."""
    return sf_to_physical(sf_linear, k)


def bf16_from_f64(v: float) -> int:
    """Bits of the bf16 nearest to v (ties to the even significand)."""
    return int(_load().or_bf16_from_f64(float(v)))


def dequantize_bf16(q: np.ndarray, sf: np.ndarray, row_scale) -> np.ndarray:
    """Packed codes + logical scales -> bf16 bit patterns [rows, k] (R14)."""
    q = np.ascontiguousarray(q, dtype=np.uint8)
    sf = np.ascontiguousarray(sf, dtype=np.uint8)
    rows = q.shape[0]
    k = q.shape[1] * 2
    rs = np.ascontiguousarray(np.broadcast_to(np.asarray(row_scale, dtype=np.float32), (rows,)))
    out = np.zeros((rows, k), dtype=np.uint16)
    if rows:
        _load().or_dequantize_bf16(_ptr(q), _ptr(sf), rows, k, _ptr(rs), _ptr(out))
    return out


def harmonize(sf: np.ndarray, seg_offsets: Sequence[int], seg_scale: Sequence[float]) -> tuple:
    """Fold per-module global scales into the block scales of a fused weight (R15).
    Returns (new logical sf [rows, k/16], shared global scale)."""
    out = np.array(sf, dtype=np.uint8, copy=True, order="C")
    rows, nblk = out.shape
    offs = np.ascontiguousarray(np.asarray(seg_offsets, dtype=np.int64))
    sc = np.ascontiguousarray(np.asarray(seg_scale, dtype=np.float32))
    shared = _load().or_harmonize(_ptr(out), rows, nblk * 16, _ptr(offs), len(sc), _ptr(sc))
    return out, np.float32(shared)


# --- GEMM ------------------------------------------------------------------

def linear_rows(qx, sfx, s_x, rows, qw, sfw, col_scale) -> np.ndarray:
    """fp64 Y[rows, :] on dequantized operands, global scales applied."""
    qx = np.ascontiguousarray(qx, dtype=np.uint8)
    sfx = np.ascontiguousarray(sfx, dtype=np.uint8)
    qw = np.ascontiguousarray(qw, dtype=np.uint8)
    sfw = np.ascontiguousarray(sfw, dtype=np.uint8)
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    col_scale = np.ascontiguousarray(np.asarray(col_scale, dtype=np.float32))
    n, k = qw.shape[0], qw.shape[1] * 2
    out = np.zeros((rows.shape[0], n), dtype=np.float64)
    if rows.shape[0] and n:
        _load().or_linear_rows(_ptr(qx), _ptr(sfx), float(s_x), _ptr(rows), rows.shape[0], _ptr(qw), _ptr(sfw),
                               _ptr(col_scale), n, k, _ptr(out))
    return out


def col_scales(seg_offsets: Sequence[int], seg_scale: Sequence[float]) -> np.ndarray:
    return row_scales_from_segments(seg_offsets, seg_scale)


def linear_reference(x_bits: np.ndarray, w_bits: np.ndarray, seg_offsets: Sequence[int],
                     rows=None, act_scale: Optional[float] = None, w_scales=None):
    """The whole layer on the CPU: dynamic (or given) activation scale, per-segment
    weight scales, quantize both operands, fp64 GEMM on the selected rows.

    Returns dict(y=fp64 [len(rows), N], s_x, s_w, qx, sfx, qw, sfw); with `rows`
    given, qx/sfx hold only those rows."""
    s_x = global_scale(amax(x_bits)) if act_scale is None else np.float32(act_scale)
    s_w = segment_scales(w_bits, seg_offsets) if w_scales is None else np.asarray(w_scales, np.float32)
    qw, sfw = quantize(w_bits, row_scales_from_segments(seg_offsets, s_w))
    if rows is None:
        qx, sfx = quantize(x_bits, s_x)
        sel = np.arange(x_bits.shape[0])
    else:
        # Only the selected rows are quantized; the global scale above is the whole tensor's.
        qx, sfx = quantize(np.ascontiguousarray(x_bits[np.asarray(rows)]), s_x)
        sel = np.arange(len(rows))
    y = linear_rows(qx, sfx, s_x, sel, qw, sfw, col_scales(seg_offsets, s_w))
    return dict(y=y, s_x=s_x, s_w=s_w, qx=qx, sfx=sfx, qw=qw, sfw=sfw)
