"""NVFP4 W4A4 linear layer for NVIDIA B200 (sm_100a).

Thin Python binding over the C ABI in include/nvfp4.h (libnvfp4.so, built
in-tree by nvfp4_w4a4_block_b200.build).  This module only marshals arguments:
torch supplies device memory and the current CUDA stream, every step of the
layer runs in the library's CUDA kernels.  There is no CPU fallback: if the
library is missing or the device is not sm_100, calls raise.

Entry points mirror the C names:
  quantize_act(x, gscale=None)            -> (q, sf, s_x)
  pack_weight(w, seg_offsets=None, ...)   -> PackedWeight
  gemm(qx, sfx, s_x, pw, ...)             -> y
  linear(x, pw, act_gscale=None, ...)     -> y      (one module)
  linear_fused(x, pw, act_gscale=None...) -> y      (modules fused along N)
  dequantize(q, sf, k, gscale, ...)       -> y bf16 (expansion of packed rows)
  import_weight_scales(sf_linear, n, k)   -> sf     (checkpoint scales -> tensor-core layout)
  harmonize_scales(pw)                    -> PackedWeight with one shared global scale
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
import threading
from typing import List, Optional, Sequence

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libnvfp4.so")

OK = 0
ERR_INVALID_ARG = 1
ERR_UNSUPPORTED_SHAPE = 2
ERR_MISALIGNED = 3
ERR_NONFINITE = 4
ERR_CUDA = 5
ERR_TIMEOUT = 6
ERR_WORKSPACE = 7
ERR_UNSUPPORTED_DEVICE = 8
ERR_SCRATCH_LIMIT = 9
NOALLOC_SCRATCH_BYTES = 8 << 20

FLAG_F32_OUT = 0x1
FLAG_COLLAPSED_MAX_SCALE = 0x2
FLAG_STATIC_WEIGHTS = 0x4
FLAG_TEST_STALL = 0x100
FLAG_TEST_STALL_LATE = 0x200
MAX_SEGMENTS = 8

EXPORTED = ("nvfp4_status_string", "nvfp4_sf_bytes", "nvfp4_workspace_bytes", "nvfp4_quantize_act",
            "nvfp4_pack_weight", "nvfp4_gemm", "nvfp4_linear", "nvfp4_linear_fused", "nvfp4_get_device_error",
            "nvfp4_set_wait_timeout_ns", "nvfp4_version", "nvfp4_linear_fused_noalloc", "nvfp4_dequantize",
            "nvfp4_import_weight_scales", "nvfp4_harmonize_scales", "nvfp4_launch_count",
            "nvfp4_mma_peak_probe")


class NVFP4Error(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


_lib = None
_lock = threading.Lock()


def lib() -> ctypes.CDLL:
    """The loaded C library; raises if it was not built."""
    global _lib
    if _lib is None:
        with _lock:
            if _lib is None:
                if not os.path.exists(LIB_PATH):
                    raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                                       "`python -m nvfp4_w4a4_block_b200.build` (no CPU fallback exists)")
                L = ctypes.CDLL(LIB_PATH)
                i64, vp, u32, sz, ci = ctypes.c_int64, ctypes.c_void_p, ctypes.c_uint, ctypes.c_size_t, ctypes.c_int
                L.nvfp4_status_string.argtypes, L.nvfp4_status_string.restype = [ci], ctypes.c_char_p
                L.nvfp4_version.argtypes, L.nvfp4_version.restype = [], ctypes.c_char_p
                L.nvfp4_sf_bytes.argtypes, L.nvfp4_sf_bytes.restype = [i64, i64], sz
                L.nvfp4_workspace_bytes.argtypes, L.nvfp4_workspace_bytes.restype = [i64, i64, i64], sz
                L.nvfp4_set_wait_timeout_ns.argtypes, L.nvfp4_set_wait_timeout_ns.restype = [ctypes.c_uint64], None
                L.nvfp4_launch_count.argtypes, L.nvfp4_launch_count.restype = [], ctypes.c_uint64
                L.nvfp4_get_device_error.argtypes, L.nvfp4_get_device_error.restype = [vp], ci
                L.nvfp4_quantize_act.argtypes = [vp, i64, i64, i64, vp, vp, vp, vp, vp, sz, vp]
                L.nvfp4_quantize_act.restype = ci
                L.nvfp4_pack_weight.argtypes = [vp, i64, i64, i64, vp, ci, vp, vp, vp, vp, vp, sz, vp]
                L.nvfp4_pack_weight.restype = ci
                L.nvfp4_gemm.argtypes = [vp, vp, vp, i64, vp, vp, i64, i64, vp, vp, ci, vp, i64, u32, vp]
                L.nvfp4_gemm.restype = ci
                L.nvfp4_linear.argtypes = [vp, i64, i64, i64, vp, vp, vp, vp, i64, vp, i64, u32, vp, sz, vp]
                L.nvfp4_linear.restype = ci
                L.nvfp4_linear_fused.argtypes = [vp, i64, i64, i64, vp, vp, vp, i64, vp, vp, ci, vp, i64, u32, vp,
                                                 sz, vp]
                L.nvfp4_linear_fused.restype = ci
                L.nvfp4_linear_fused_noalloc.argtypes = [vp, i64, i64, i64, vp, vp, vp, i64, vp, vp, ci, vp, i64,
                                                         u32, vp]
                L.nvfp4_linear_fused_noalloc.restype = ci
                L.nvfp4_dequantize.argtypes = [vp, vp, i64, i64, vp, vp, ci, vp, i64, vp]
                L.nvfp4_dequantize.restype = ci
                L.nvfp4_import_weight_scales.argtypes = [vp, i64, i64, i64, vp, vp]
                L.nvfp4_import_weight_scales.restype = ci
                L.nvfp4_harmonize_scales.argtypes = [vp, vp, i64, i64, vp, vp, ci, vp, vp]
                L.nvfp4_harmonize_scales.restype = ci
                L.nvfp4_mma_peak_probe.argtypes = [ci, i64, ci, ctypes.POINTER(ctypes.c_double), vp]
                L.nvfp4_mma_peak_probe.restype = ci
                _lib = L
    return _lib


def status_string(st: int) -> str:
    return lib().nvfp4_status_string(int(st)).decode()


def _check(st: int, where: str):
    if st != OK:
        raise NVFP4Error(st, where)


def sf_bytes(rows: int, k: int) -> int:
    return int(lib().nvfp4_sf_bytes(rows, k))


def workspace_bytes(m: int, n: int, k: int) -> int:
    return int(lib().nvfp4_workspace_bytes(m, n, k))


def launch_count() -> int:
    """Kernel launches this library has enqueued in this process so far."""
    return int(lib().nvfp4_launch_count())


def set_wait_timeout_ns(ns: int):
    lib().nvfp4_set_wait_timeout_ns(int(ns))


def get_device_error(stream=None) -> int:
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return int(lib().nvfp4_get_device_error(ctypes.c_void_p(s.cuda_stream)))


# --------------------------------------------------------------------------
# torch plumbing (memory and streams only)
# --------------------------------------------------------------------------

def _torch():
    import torch
    return torch


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream=None):
    torch = _torch()
    return ctypes.c_void_p((torch.cuda.current_stream() if stream is None else stream).cuda_stream)


def _seg_array(seg_offsets: Optional[Sequence[int]]):
    if seg_offsets is None:
        return None, 1
    arr = (ctypes.c_int64 * len(seg_offsets))(*[int(v) for v in seg_offsets])
    return arr, len(seg_offsets) - 1


_ws_cache = {}


def workspace(m: int, n: int, k: int, device=None):
    """A cached device workspace of at least nvfp4_workspace_bytes(m, n, k)."""
    torch = _torch()
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    need = workspace_bytes(m, n, k)
    buf = _ws_cache.get(dev)
    if buf is None or buf.numel() < need:
        buf = torch.empty(max(need, 1 << 20), dtype=torch.uint8, device=dev)
        _ws_cache[dev] = buf
    return buf


def _check_bf16(t, name):
    torch = _torch()
    if not t.is_cuda or t.dtype != torch.bfloat16 or t.dim() != 2 or t.stride(1) != 1:
        raise ValueError(f"{name} must be a 2-D CUDA bfloat16 tensor with unit inner stride")


@dataclasses.dataclass
class PackedWeight:
    """A pre-packed NVFP4 weight: codes [n, k/2] u8, swizzled scales, per-segment scales."""
    q: object
    sf: object
    gscale: object                      # device float32 [nseg]
    n: int
    k: int
    seg_offsets: List[int]

    @property
    def nseg(self) -> int:
        return len(self.seg_offsets) - 1


def quantize_act(x, gscale=None, q=None, sf=None, gscale_out=None, stream=None):
    """Activation quantization. x: [m, k] bf16 CUDA. gscale: optional device float32 [1]
    static scale (None = dynamic amax/2688). Returns (q, sf, s_x)."""
    torch = _torch()
    _check_bf16(x, "x")
    m, k = x.shape
    q = torch.empty((m, k // 2), dtype=torch.uint8, device=x.device) if q is None else q
    sf = torch.empty(sf_bytes(m, k), dtype=torch.uint8, device=x.device) if sf is None else sf
    gscale_out = torch.empty(1, dtype=torch.float32, device=x.device) if gscale_out is None else gscale_out
    ws = workspace(m, 0, k, x.device)
    st = lib().nvfp4_quantize_act(_ptr(x), m, k, x.stride(0), _ptr(gscale), _ptr(gscale_out), _ptr(q), _ptr(sf),
                                  _ptr(ws), ws.numel(), _stream(stream))
    _check(st, "nvfp4_quantize_act")
    return q, sf, gscale_out


def pack_weight(w, seg_offsets: Optional[Sequence[int]] = None, gscale=None, stream=None) -> PackedWeight:
    """Offline weight packing with one global scale per segment of rows."""
    torch = _torch()
    _check_bf16(w, "w")
    n, k = w.shape
    offs = list(seg_offsets) if seg_offsets is not None else [0, n]
    arr, nseg = _seg_array(offs)
    q = torch.empty((n, k // 2), dtype=torch.uint8, device=w.device)
    sf = torch.empty(sf_bytes(n, k), dtype=torch.uint8, device=w.device)
    gs = torch.empty(nseg, dtype=torch.float32, device=w.device)
    ws = workspace(n, 0, k, w.device)
    st = lib().nvfp4_pack_weight(_ptr(w), n, k, w.stride(0), arr, nseg, _ptr(gscale), _ptr(gs), _ptr(q), _ptr(sf),
                                 _ptr(ws), ws.numel(), _stream(stream))
    _check(st, "nvfp4_pack_weight")
    return PackedWeight(q, sf, gs, n, k, offs)


def _out(m, n, device, flags, out):
    torch = _torch()
    if out is not None:
        return out
    dt = torch.float32 if flags & FLAG_F32_OUT else torch.bfloat16
    return torch.empty((m, n), dtype=dt, device=device)


def gemm(qx, sfx, s_x, m: int, pw: PackedWeight, out=None, flags: int = 0, stream=None):
    """Block-scaled FP4 GEMM + per-segment global-scale epilogue on quantized operands."""
    y = _out(m, pw.n, pw.q.device, flags, out)
    arr, nseg = _seg_array(pw.seg_offsets)
    st = lib().nvfp4_gemm(_ptr(qx), _ptr(sfx), _ptr(s_x), m, _ptr(pw.q), _ptr(pw.sf), pw.n, pw.k, arr,
                          _ptr(pw.gscale), nseg, _ptr(y), y.stride(0), flags, _stream(stream))
    _check(st, "nvfp4_gemm")
    return y


def linear_fused(x, pw: PackedWeight, act_gscale=None, out=None, flags: int = 0, stream=None, ws=None):
    """The whole W4A4 layer for modules fused along N, each with its own weight scale."""
    _check_bf16(x, "x")
    m, k = x.shape
    if k != pw.k:
        raise ValueError("K mismatch")
    y = _out(m, pw.n, x.device, flags, out)
    ws = workspace(m, pw.n, k, x.device) if ws is None else ws
    arr, nseg = _seg_array(pw.seg_offsets)
    st = lib().nvfp4_linear_fused(_ptr(x), m, k, x.stride(0), _ptr(act_gscale), _ptr(pw.q), _ptr(pw.sf), pw.n, arr,
                                  _ptr(pw.gscale), nseg, _ptr(y), y.stride(0), flags, _ptr(ws), ws.numel(),
                                  _stream(stream))
    _check(st, "nvfp4_linear_fused")
    return y


def linear(x, pw: PackedWeight, act_gscale=None, out=None, flags: int = 0, stream=None, ws=None):
    """The whole W4A4 layer for one module (single weight global scale)."""
    _check_bf16(x, "x")
    if pw.nseg != 1:
        raise ValueError("linear() takes a single-module weight; use linear_fused()")
    m, k = x.shape
    y = _out(m, pw.n, x.device, flags, out)
    ws = workspace(m, pw.n, k, x.device) if ws is None else ws
    st = lib().nvfp4_linear(_ptr(x), m, k, x.stride(0), _ptr(act_gscale), _ptr(pw.q), _ptr(pw.sf), _ptr(pw.gscale),
                            pw.n, _ptr(y), y.stride(0), flags, _ptr(ws), ws.numel(), _stream(stream))
    _check(st, "nvfp4_linear")
    return y


def linear_fused_noalloc(x, pw: PackedWeight, act_gscale=None, out=None, flags: int = 0, stream=None):
    """linear_fused without a workspace: the library's own static device scratch
    (NOALLOC_SCRATCH_BYTES per device) holds the activation codes and scales.
    For callers that cannot allocate device memory.  Calls sharing the scratch
    must be ordered on one stream; the first call on a device should come before
    any stream capture."""
    _check_bf16(x, "x")
    m, k = x.shape
    if k != pw.k:
        raise ValueError("K mismatch")
    y = _out(m, pw.n, x.device, flags, out)
    arr, nseg = _seg_array(pw.seg_offsets)
    st = lib().nvfp4_linear_fused_noalloc(_ptr(x), m, k, x.stride(0), _ptr(act_gscale), _ptr(pw.q), _ptr(pw.sf),
                                          pw.n, arr, _ptr(pw.gscale), nseg, _ptr(y), y.stride(0), flags,
                                          _stream(stream))
    _check(st, "nvfp4_linear_fused_noalloc")
    return y


def dequantize(q, sf, k: int, gscale, seg_offsets: Optional[Sequence[int]] = None, out=None, stream=None):
    """Expand packed rows to bf16: value(code) * value(block scale) * s, rounded once.
    q: [rows, k/2] uint8; sf: physical scales; gscale: device float32 [nseg]."""
    torch = _torch()
    rows = q.shape[0]
    y = torch.empty((rows, k), dtype=torch.bfloat16, device=q.device) if out is None else out
    offs = list(seg_offsets) if seg_offsets is not None else [0, rows]
    arr, nseg = _seg_array(offs)
    st = lib().nvfp4_dequantize(_ptr(q), _ptr(sf), rows, k, arr, _ptr(gscale), nseg, _ptr(y), y.stride(0),
                                _stream(stream))
    _check(st, "nvfp4_dequantize")
    return y


def import_weight_scales(sf_linear, n: int, k: int, out=None, stream=None):
    """Checkpoint block scales [n, k/16] (uint8 E4M3, row-major, row stride
    sf_linear.stride(0)) -> the tensor-core layout used by the GEMM."""
    torch = _torch()
    sf = torch.empty(sf_bytes(n, k), dtype=torch.uint8, device=sf_linear.device) if out is None else out
    st = lib().nvfp4_import_weight_scales(_ptr(sf_linear), n, k, sf_linear.stride(0), _ptr(sf), _stream(stream))
    _check(st, "nvfp4_import_weight_scales")
    return sf


def harmonize_scales(pw: PackedWeight, in_place: bool = False, stream=None) -> PackedWeight:
    """Fold the per-module global scales of a fused weight into its block scales
    so that one shared scale (the largest) serves the whole GEMM.  Returns a
    single-segment PackedWeight sharing pw's codes."""
    torch = _torch()
    sf = pw.sf if in_place else torch.empty_like(pw.sf)
    shared = torch.empty(1, dtype=torch.float32, device=pw.sf.device)
    arr, nseg = _seg_array(pw.seg_offsets)
    st = lib().nvfp4_harmonize_scales(_ptr(pw.sf), _ptr(sf), pw.n, pw.k, arr, _ptr(pw.gscale), nseg, _ptr(shared),
                                      _stream(stream))
    _check(st, "nvfp4_harmonize_scales")
    return PackedWeight(pw.q, sf, shared, pw.n, pw.k, [0, pw.n])


def mma_peak_probe(iters: int, pairs: Optional[int] = None, with_scale_copies: bool = False, stream=None) -> float:
    """Enqueue one launch of the dense FP4 tensor-core probe (measurement only,
    see nvfp4_mma_peak_probe) and return its MMA flops; time it with CUDA events
    on the same stream.  pairs defaults to half the SM count (every SM)."""
    torch = _torch()
    if pairs is None:
        pairs = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count // 2
    flops = ctypes.c_double(0.0)
    st = lib().nvfp4_mma_peak_probe(int(pairs), int(iters), 1 if with_scale_copies else 0, ctypes.byref(flops),
                                    _stream(stream))
    _check(st, "nvfp4_mma_peak_probe")
    return flops.value

