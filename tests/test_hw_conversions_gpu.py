"""The hardware conversions the quantizers rely on, checked against the
oracle's definitions over whole ranges of fp32 inputs on the GPU itself.

The quantizers round with the hardware conversions `cvt.rn.satfinite.e2m1x2.f32`
(element codes, R7: nearest E2M1 value, ties to the even code, saturation at 6,
sign kept) and `cvt.rn.satfinite.e4m3x2.f32` (block scales, R5).  A small probe
kernel (built here with nvcc, test-only; it shares nothing with the library)
converts every fp32 bit pattern of a range and the codes are compared byte for
byte with the oracle's encoders:

  * E2M1: every finite pattern and both infinities (4.28e9 inputs);
  * E4M3: every finite pattern of both signs and both infinities (the block
    scales are non-negative; harmonization also folds sign-bit scale bytes of
    imported checkpoints, whose products are negative), plus each midpoint
    between neighbouring E4M3 values and its two fp32 neighbours listed on
    their own.

NaN inputs are not compared: no step of the layer feeds one to a conversion
except a non-finite tensor, whose codes are unspecified (its amax is reported
as non-finite), and harmonization keeps NaN scale bytes without converting
them.
"""
import ctypes
import os
import subprocess

import numpy as np
import pytest

import oracle

pytestmark = pytest.mark.gpu

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

PROBE = r"""
#include <cuda_runtime.h>

__device__ __forceinline__ unsigned int e2m1_pair(float hi, float lo)
{
    unsigned short h;
    asm("{\n\t.reg .b8 b;\n\tcvt.rn.satfinite.e2m1x2.f32 b, %1, %2;\n\tcvt.u16.u8 %0, b;\n\t}"
        : "=h"(h) : "f"(hi), "f"(lo));
    return h;
}

// One byte per pattern: out[i] = E2M1 code of the fp32 with bits start + i.
// Each thread converts 8 consecutive patterns (the conversion writes its first
// operand to the high nibble).
__global__ void e2m1_range_probe(unsigned long long start, unsigned long long groups, uint2 *out)
{
    const unsigned long long stride = (unsigned long long)gridDim.x * blockDim.x;
    for (unsigned long long g = blockIdx.x * (unsigned long long)blockDim.x + threadIdx.x; g < groups; g += stride) {
        const unsigned int u = (unsigned int)(start + 8ull * g);
        unsigned int w[2];
        for (int h = 0; h < 2; ++h) {
            unsigned int acc = 0;
            for (int j = 0; j < 2; ++j) {
                const unsigned int b = u + 4 * h + 2 * j;
                const unsigned int p = e2m1_pair(__uint_as_float(b + 1), __uint_as_float(b));
                acc |= ((p & 15u) | ((p >> 4) << 8)) << (16 * j);
            }
            w[h] = acc;
        }
        out[g] = make_uint2(w[0], w[1]);
    }
}

// out[i] = E4M3 code of the fp32 with bits start + i; each thread converts
// 4 consecutive patterns (two conversions of a pair each).
__global__ void e4m3_range_probe(unsigned long long start, unsigned long long groups, unsigned int *out)
{
    const unsigned long long stride = (unsigned long long)gridDim.x * blockDim.x;
    for (unsigned long long g = blockIdx.x * (unsigned long long)blockDim.x + threadIdx.x; g < groups; g += stride) {
        const unsigned int u = (unsigned int)(start + 4ull * g);
        unsigned int w = 0;
        for (int j = 0; j < 2; ++j) {
            unsigned short h;
            asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;"
                : "=h"(h) : "f"(__uint_as_float(u + 2 * j + 1)), "f"(__uint_as_float(u + 2 * j)));
            w |= (unsigned int)h << (16 * j);
        }
        out[g] = w;
    }
}

__global__ void e4m3_list_probe(const unsigned int *pats, long long count, unsigned char *out)
{
    const long long stride = (long long)gridDim.x * blockDim.x;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < count; i += stride) {
        unsigned short h;
        asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(h) : "f"(0.0f), "f"(__uint_as_float(pats[i])));
        out[i] = (unsigned char)(h & 0xFF);
    }
}

extern "C" int probe_e2m1_range(unsigned long long start, unsigned long long count, void *out)
{
    if (count % 8 != 0) return -1;
    e2m1_range_probe<<<1184, 256>>>(start, count / 8, (uint2 *)out);
    return (int)cudaDeviceSynchronize();
}

extern "C" int probe_e4m3_range(unsigned long long start, unsigned long long count, void *out)
{
    if (count % 4 != 0) return -1;
    e4m3_range_probe<<<1184, 256>>>(start, count / 4, (unsigned int *)out);
    return (int)cudaDeviceSynchronize();
}

extern "C" int probe_e4m3_list(const void *pats, long long count, void *out)
{
    e4m3_list_probe<<<1184, 256>>>((const unsigned int *)pats, count, (unsigned char *)out);
    return (int)cudaDeviceSynchronize();
}
"""


@pytest.fixture(scope="module")
def probe(tmp_path_factory):
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.init()
    d = tmp_path_factory.mktemp("hwcvt")
    src = d / "probe.cu"
    src.write_text(PROBE)
    lib = d / "probe.so"
    subprocess.check_call([NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-O2", "-shared",
                           "-Xcompiler", "-fPIC", "-o", str(lib), str(src)])
    L = ctypes.CDLL(str(lib))
    vp, i64, u64 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_uint64
    L.probe_e2m1_range.argtypes, L.probe_e2m1_range.restype = [u64, u64, vp], ctypes.c_int
    L.probe_e4m3_list.argtypes, L.probe_e4m3_list.restype = [vp, i64, vp], ctypes.c_int
    L.probe_e4m3_range.argtypes, L.probe_e4m3_range.restype = [u64, u64, vp], ctypes.c_int
    return L


def _first_mismatch(pats, got, want, what):
    if not np.array_equal(got, want):
        i = int(np.flatnonzero(got != want)[0])
        raise AssertionError(f"{what} of pattern {int(pats(i)):#010x}: gpu {got[i]:#x}, oracle {want[i]:#x}")


def _list(L, fn, pats):
    import torch
    dev = torch.from_numpy(pats.view(np.int32)).cuda()
    out = torch.empty(pats.size, dtype=torch.uint8, device="cuda")
    assert getattr(L, fn)(dev.data_ptr(), pats.size, out.data_ptr()) == 0
    return out.cpu().numpy()


def test_e2m1_conversion_matches_oracle_on_every_finite_pattern(probe):
    import torch
    chunk = 1 << 27
    last = 0x7F800000                                   # +inf; the patterns above it are NaN
    out = torch.empty(chunk, dtype=torch.uint8, device="cuda")
    for sign in (0, 0x80000000):
        for start in range(0, last + 1, chunk):
            count = min(chunk, last + 1 - start)
            first = sign + start
            run = (count + 7) // 8 * 8                  # the probe converts runs of 8 patterns
            assert probe.probe_e2m1_range(first, run, out.data_ptr()) == 0
            got = out[:count].cpu().numpy()
            want = oracle.e2m1_encode_patterns(first, count)
            _first_mismatch(lambda i: first + i, got, want, "E2M1 code")


def test_e4m3_conversion_matches_oracle_on_every_finite_pattern(probe):
    import torch
    chunk = 1 << 27
    last = 0x7F800000                                   # +inf; the patterns above it are NaN
    out = torch.empty(chunk, dtype=torch.uint8, device="cuda")
    for sign in (0, 0x80000000):
        for start in range(0, last + 1, chunk):
            count = min(chunk, last + 1 - start)
            first = sign + start
            run = (count + 3) // 4 * 4                  # the probe converts runs of 4 patterns
            assert probe.probe_e4m3_range(first, run, out.data_ptr()) == 0
            got = out[:count].cpu().numpy()
            want = oracle.e4m3_encode_range(first, count)
            _first_mismatch(lambda i: first + i, got, want, "E4M3 code")


def test_e4m3_conversion_matches_oracle_including_every_tie(probe):
    grid = np.array([oracle.e4m3_value(c) for c in range(127)], np.float64)
    mids = ((grid[1:] + grid[:-1]) / 2).astype(np.float32)
    near = np.concatenate([mids, np.nextafter(mids, np.float32(0)), np.nextafter(mids, np.float32(1e9))])
    dense = np.arange(0, 0x43E80000, 256, dtype=np.uint32)            # [0, 464] at 2^-15 relative spacing
    edges = np.array([0x43E00000, 0x43E80000, 0x7F7FFFFF, 0x7F800000], np.uint32)   # 448, 464, FLT_MAX, inf
    pats = np.concatenate([dense, near.view(np.uint32), edges])
    got = _list(probe, "probe_e4m3_list", pats)
    want = oracle.e4m3_encode_patterns(pats)
    _first_mismatch(lambda i: pats[i], got, want, "E4M3 code")
