"""The C-ABI library loads on a machine without a GPU, exports every entry point
include/nvfp4.h declares, and rejects bad arguments on the host before any CUDA
call.  (No compute call is made here.)"""
import ctypes
import os
import re

import pytest

import nvfp4_w4a4_block_b200 as nv
from nvfp4_w4a4_block_b200 import build as nvbuild

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "nvfp4.h")


@pytest.fixture(scope="module")
def L():
    nvbuild.build()
    return nv.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(nvfp4_[a-z0-9_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(L):
    names = declared_functions()
    assert len(names) >= 10
    for name in names:
        assert hasattr(L, name), name
    assert set(names) == set(nv.EXPORTED)


def test_status_strings(L):
    for st in range(9):
        assert nv.status_string(st) not in ("", "unknown status")
    assert nv.status_string(99) == "unknown status"


def test_sf_bytes_layout_sizes(L):
    assert nv.sf_bytes(1, 64) == 128 * 4
    assert nv.sf_bytes(128, 256) == 128 * 16
    assert nv.sf_bytes(129, 320) == 256 * 20
    assert nv.sf_bytes(16, 256) == 128 * 16
    assert nv.sf_bytes(-1, 64) == 0 and nv.sf_bytes(4, 8) == 0


def test_workspace_grows_with_activation(L):
    a, b = nv.workspace_bytes(1, 0, 5120), nv.workspace_bytes(32, 0, 5120)
    assert 0 < a < b
    assert nv.workspace_bytes(8192, 17408, 5120) >= 8192 * 5120 // 2 + nv.sf_bytes(8192, 5120)


FAKE = 0x10000          # 16-byte aligned, never dereferenced: validation fails first
MIS = 0x10001


def test_quantize_validation(L):
    f = L.nvfp4_quantize_act
    assert f(None, 4, 64, 64, None, FAKE, FAKE, FAKE, FAKE, 1 << 20, None) == nv.ERR_INVALID_ARG
    assert f(FAKE, 4, 48, 48, None, FAKE, FAKE, FAKE, FAKE, 1 << 20, None) == nv.ERR_UNSUPPORTED_SHAPE
    assert f(MIS, 4, 64, 64, None, FAKE, FAKE, FAKE, FAKE, 1 << 20, None) == nv.ERR_MISALIGNED
    assert f(FAKE, 4, 64, 68, None, FAKE, FAKE, FAKE, FAKE, 1 << 20, None) == nv.ERR_MISALIGNED
    assert f(FAKE, 4, 64, 32, None, FAKE, FAKE, FAKE, FAKE, 1 << 20, None) == nv.ERR_INVALID_ARG
    assert f(FAKE, 4, 64, 64, None, None, FAKE, FAKE, FAKE, 1 << 20, None) == nv.ERR_INVALID_ARG
    assert f(FAKE, 4, 64, 64, None, FAKE, FAKE, FAKE, None, 0, None) == nv.ERR_WORKSPACE
    assert f(FAKE, -1, 64, 64, None, FAKE, FAKE, FAKE, FAKE, 1 << 20, None) == nv.ERR_INVALID_ARG
    assert f(FAKE, 0, 64, 64, None, FAKE, FAKE, FAKE, FAKE, 1 << 20, None) == nv.OK     # empty: no-op


def _segs(*v):
    return (ctypes.c_int64 * len(v))(*v)


def test_gemm_validation(L):
    g = L.nvfp4_gemm
    ok = dict(qx=FAKE, sfx=FAKE, sx=FAKE, m=4, qw=FAKE, sfw=FAKE, n=64, k=128, seg=None, sw=FAKE, nseg=1, y=FAKE,
              ldy=64, flags=0)

    def call(**kw):
        a = dict(ok, **kw)
        return g(a["qx"], a["sfx"], a["sx"], a["m"], a["qw"], a["sfw"], a["n"], a["k"], a["seg"], a["sw"], a["nseg"],
                 a["y"], a["ldy"], a["flags"], None)

    assert call(k=96) == nv.ERR_UNSUPPORTED_SHAPE
    assert call(n=60, ldy=60) == nv.ERR_UNSUPPORTED_SHAPE
    assert call(qw=None) == nv.ERR_INVALID_ARG
    assert call(sw=None) == nv.ERR_INVALID_ARG
    assert call(y=MIS) == nv.ERR_MISALIGNED
    assert call(ldy=60) == nv.ERR_INVALID_ARG
    assert call(ldy=68) == nv.ERR_MISALIGNED
    assert call(flags=0x8) == nv.ERR_INVALID_ARG
    assert call(flags=nv.FLAG_STATIC_WEIGHTS | nv.FLAG_F32_OUT, m=0, ldy=64) == nv.OK
    assert call(nseg=2) == nv.ERR_INVALID_ARG                       # NULL table needs nseg == 1
    assert call(seg=_segs(0, 32, 64), nseg=2, m=0) == nv.OK
    assert call(seg=_segs(0, 32, 60), nseg=2) == nv.ERR_INVALID_ARG  # last != N
    assert call(seg=_segs(0, 36, 64), nseg=2) == nv.ERR_UNSUPPORTED_SHAPE
    assert call(seg=_segs(0, 32, 32, 64), nseg=3) == nv.ERR_INVALID_ARG
    assert call(seg=_segs(*range(0, 80, 8)), nseg=9, n=72, ldy=72) == nv.ERR_UNSUPPORTED_SHAPE
    assert call(m=0) == nv.OK


def test_linear_validation(L):
    f = L.nvfp4_linear
    assert f(FAKE, 4, 128, 128, None, FAKE, FAKE, FAKE, 64, FAKE, 64, 0, None, 0, None) == nv.ERR_WORKSPACE
    assert f(FAKE, 4, 128, 128, None, FAKE, FAKE, FAKE, 64, FAKE, 64, 0, FAKE, 16, None) == nv.ERR_WORKSPACE
    assert f(None, 4, 128, 128, None, FAKE, FAKE, FAKE, 64, FAKE, 64, 0, FAKE, 1 << 30, None) == nv.ERR_INVALID_ARG


def test_pack_validation(L):
    f = L.nvfp4_pack_weight
    assert f(FAKE, 64, 128, 128, _segs(0, 16, 64), 2, None, FAKE, FAKE, FAKE, None, 0, None) == nv.ERR_WORKSPACE
    assert f(FAKE, 64, 128, 128, _segs(0, 70, 64), 2, None, FAKE, FAKE, FAKE, FAKE, 1 << 20, None) == \
        nv.ERR_INVALID_ARG
    assert f(FAKE, 0, 128, 128, None, 1, None, FAKE, FAKE, FAKE, FAKE, 1 << 20, None) == nv.ERR_INVALID_ARG


def test_dequantize_validation(L):
    f = L.nvfp4_dequantize
    assert f(FAKE, FAKE, 4, 96, None, FAKE, 1, FAKE, 96, None) == nv.ERR_UNSUPPORTED_SHAPE
    assert f(FAKE, FAKE, -1, 64, None, FAKE, 1, FAKE, 64, None) == nv.ERR_INVALID_ARG
    assert f(FAKE, FAKE, 4, 64, None, FAKE, 1, FAKE, 32, None) == nv.ERR_INVALID_ARG        # ldy < k
    assert f(None, FAKE, 4, 64, None, FAKE, 1, FAKE, 64, None) == nv.ERR_INVALID_ARG
    assert f(FAKE, FAKE, 4, 64, None, None, 1, FAKE, 64, None) == nv.ERR_INVALID_ARG
    assert f(MIS, FAKE, 4, 64, None, FAKE, 1, FAKE, 64, None) == nv.ERR_MISALIGNED
    assert f(FAKE, FAKE, 4, 64, None, FAKE, 1, FAKE, 68, None) == nv.ERR_MISALIGNED        # row stride
    assert f(FAKE, FAKE, 16, 64, _segs(0, 8, 12), FAKE, 2, FAKE, 64, None) == nv.ERR_INVALID_ARG  # last != rows
    assert f(FAKE, FAKE, 16, 64, _segs(0, 4, 16), FAKE, 2, FAKE, 64, None) == nv.ERR_UNSUPPORTED_SHAPE
    assert f(FAKE, FAKE, 0, 64, None, FAKE, 1, FAKE, 64, None) == nv.OK                     # empty: no-op


def test_import_scales_validation(L):
    f = L.nvfp4_import_weight_scales
    assert f(FAKE, 4, 96, 8, FAKE, None) == nv.ERR_UNSUPPORTED_SHAPE
    assert f(FAKE, 4, 128, 4, FAKE, None) == nv.ERR_INVALID_ARG          # ld < k/16
    assert f(FAKE, 4, 128, 10, FAKE, None) == nv.ERR_MISALIGNED          # ld % 4
    assert f(FAKE + 2, 4, 128, 8, FAKE + 0x10000, None) == nv.ERR_MISALIGNED
    assert f(FAKE, 4, 128, 8, FAKE + 8, None) == nv.ERR_MISALIGNED       # output not 16-byte aligned
    assert f(FAKE, 4, 128, 8, FAKE + 16, None) == nv.ERR_INVALID_ARG     # overlaps the input
    assert f(None, 4, 128, 8, FAKE, None) == nv.ERR_INVALID_ARG
    assert f(FAKE, 0, 128, 8, FAKE, None) == nv.OK                       # empty: no-op


def test_harmonize_validation(L):
    f = L.nvfp4_harmonize_scales
    assert f(FAKE, FAKE, 0, 128, None, FAKE, 1, FAKE, None) == nv.ERR_INVALID_ARG
    assert f(FAKE, FAKE, 64, 96, None, FAKE, 1, FAKE, None) == nv.ERR_UNSUPPORTED_SHAPE
    assert f(FAKE, FAKE, 64, 128, _segs(0, 16, 60), FAKE, 2, FAKE, None) == nv.ERR_INVALID_ARG
    assert f(FAKE, FAKE, 64, 128, None, FAKE, 1, None, None) == nv.ERR_INVALID_ARG         # no shared-scale slot
    assert f(MIS, FAKE, 64, 128, None, FAKE, 1, FAKE, None) == nv.ERR_MISALIGNED
    assert f(FAKE, FAKE + 16, 64, 128, None, FAKE, 1, FAKE, None) == nv.ERR_INVALID_ARG    # partial overlap


def test_noalloc_validation_and_exact_scratch_limit(L):
    """The no-allocation entry checks the shape before its scratch limit (a
    malformed call gets nvfp4_linear_fused's status), and at K = 5120 the
    largest problem its 8 MiB scratch takes is 2895 tokens: 2896 is rejected on
    the host with NVFP4_ERR_SCRATCH_LIMIT before any CUDA call."""
    f = L.nvfp4_linear_fused_noalloc

    def call(m, k, x=FAKE, ldx=None):
        return f(x, m, k, k if ldx is None else ldx, None, FAKE, FAKE, 64, None, FAKE, 1, FAKE, 64, 0, None)

    assert call(100000, 96) == nv.ERR_UNSUPPORTED_SHAPE          # K % 64 before the size limit
    assert call(100000, 128, x=MIS) == nv.ERR_MISALIGNED
    assert call(100000, 128, ldx=64) == nv.ERR_INVALID_ARG
    assert call(-1, 128) == nv.ERR_INVALID_ARG
    assert call(2896, 5120) == nv.ERR_SCRATCH_LIMIT
    assert call(848, 17408) == nv.ERR_SCRATCH_LIMIT
    assert nv.workspace_bytes(2895, 0, 5120) <= nv.NOALLOC_SCRATCH_BYTES < nv.workspace_bytes(2896, 0, 5120)
    assert nv.workspace_bytes(847, 0, 17408) <= nv.NOALLOC_SCRATCH_BYTES < nv.workspace_bytes(848, 0, 17408)


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    import importlib
    mod = importlib.import_module("nvfp4_w4a4_block_b200")
    monkeypatch.setattr(mod, "_lib", None)
    monkeypatch.setattr(mod, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="no CPU fallback"):
        mod.lib()
