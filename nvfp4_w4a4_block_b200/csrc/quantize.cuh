// quantize.cuh -- NVFP4 quantization kernels (activations per call, weights offline).
//
// Method ("Why Gated DeltaNet Survives 4-Bit Quantization", §2 "NVFP4"): each run
// of 16 consecutive elements along K gets one E4M3 block scale set to blockmax/6
// relative to an FP32 per-tensor global scale; elements are rounded to E2M1.
// Arithmetic order (identical on the CPU reference, element for element):
//   s    = amax / 2688                        (fp32, dynamic mode; else the given s)
//   sb   = E4M3_rn_satfinite(min(bmax / (s*6), 448))   (0 when s*6 == 0)
//   d    = value(sb) * s;  r = d == 0 ? 0 : min(1/d, FLT_MAX)
//   code = E2M1_rn_satfinite(x * r)           two codes per byte, lower K index low
//
// Kernel design (HBM-bound): one thread owns 8 consecutive bf16 (one 16-byte
// load), two neighbouring lanes own a 16-element block and exchange their
// halves' maxima with one shuffle; eight lanes cover four blocks of one row,
// whose four scale bytes are contiguous in the tensor-core layout and leave in
// one 32-bit store.  The codes of a thread leave in one 32-bit store, so a warp
// writes 128 contiguous bytes.  The amax pass reduces in bf16 bit space
// (|x| bits = x & 0x7FFF; integer max orders finite < inf < NaN) and writes one
// partial per CTA, which the encode pass reduces again -- no atomics, no
// workspace initialisation, deterministic.
#pragma once

#include <cfloat>
#include <cstdint>
#include <cuda_bf16.h>

#include "sm100_ptx.cuh"

namespace nvfp4 {

constexpr int kQuantThreads = 256;
constexpr int kMaxSeg = 8;

__device__ __forceinline__ void raise_device_error(unsigned code)
{
    atomicCAS(&g_device_error, 0u, code);
}

// ------------------------------------------------------------------ helpers

// |bf16| bit patterns: per-halfword unsigned max over a 16-byte chunk.
__device__ __forceinline__ uint32_t absmax_bits8(const uint4 &v)
{
    const uint32_t m = 0x7FFF7FFFu;
    uint32_t a = __vmaxu2(v.x & m, v.y & m);
    uint32_t b = __vmaxu2(v.z & m, v.w & m);
    uint32_t c = __vmaxu2(a, b);
    return max(c >> 16, c & 0xFFFFu);
}

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// E4M3 (satfinite, round-to-nearest-even) of a non-negative finite fp32 <= 448.
__device__ __forceinline__ uint32_t f32_to_e4m3(float v)
{
    uint16_t h;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(h) : "f"(0.0f), "f"(v));
    return h & 0xFFu;
}

// Exact decode of an E4M3 byte, sign included (the quantizers' block scales are
// non-negative; the expansion and harmonization of imported scales rely on a
// sign-bit byte decoding to a negative value).  0x7F and 0xFF decode to NaN.
__device__ __forceinline__ float e4m3_to_f32(uint32_t code)
{
    uint32_t h2;
    uint16_t in = static_cast<uint16_t>(code & 0xFFu);
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(in));
    return __half2float(__ushort_as_half(static_cast<unsigned short>(h2 & 0xFFFFu)));
}

// Eight fp32 -> four bytes of E2M1 codes (round-to-nearest-even, saturating);
// element 2i in bits 8i..8i+3, element 2i+1 in bits 8i+4..8i+7.  The cvt puts its
// first source operand in the high nibble, so each pair is passed (odd, even).
__device__ __forceinline__ uint32_t f32x8_to_e2m1x8(float v0, float v1, float v2, float v3, float v4, float v5,
                                                    float v6, float v7)
{
    uint32_t out;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(out)
        : "f"(v0), "f"(v1), "f"(v2), "f"(v3), "f"(v4), "f"(v5), "f"(v6), "f"(v7));
    return out;
}

__device__ __forceinline__ int64_t sf_atom_offset(int64_t row, int64_t kb, int64_t kb_pad)
{
    return ((row >> 7) * (kb_pad >> 2) + (kb >> 2)) * 512 + (row & 31) * 16 + ((row >> 5) & 3) * 4;
}

// Zeroes the scale bytes of the pad rows [rows, rows_pad), all of which lie in
// the last 128-row block.  Thread i of the launch takes the 4-byte word i of
// that block's atoms (consecutive threads, consecutive words); the word holds
// row ((i % 128) / 4) + 32 * (i % 4) of its atom.
__device__ __forceinline__ void zero_pad_scales(uint8_t *sf, int64_t rows, int64_t rows_pad, int64_t kb_pad,
                                                int64_t gtid, int64_t nthreads)
{
    const int64_t last = (rows_pad >> 7) - 1;                  // last 128-row block
    const int valid = static_cast<int>(rows - last * 128);     // its rows that hold data
    if (valid >= 128)
        return;
    const int64_t atoms = kb_pad >> 2;
    uint32_t *block = reinterpret_cast<uint32_t *>(sf + last * atoms * 512);
    for (int64_t i = gtid; i < atoms * 128; i += nthreads) {
        const int w = static_cast<int>(i & 127);
        if (((w >> 2) | ((w & 3) << 5)) >= valid)
            block[i] = 0u;
    }
}

// ------------------------------------------------------------------ amax

struct AmaxParams {
    const uint16_t *x;
    int64_t row_begin, row_end, k, ldx;
    uint32_t *partial;   // one entry per CTA
};

__global__ void __launch_bounds__(kQuantThreads) amax_partial_kernel(AmaxParams p)
{
    // Launched without a programmatic dependency, so everything before it in the
    // stream has completed; the encode pass may start its prologue right away.
    pdl_launch_dependents();
    const int64_t upr = p.k >> 3;                          // 16-byte units per row
    const int64_t rows = p.row_end - p.row_begin;
    const int64_t nthreads = static_cast<int64_t>(gridDim.x) * blockDim.x;
    const int64_t gtid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    // Each thread walks four interleaved streams of units; (row, col) advance
    // by a precomputed step so that no division sits in the loop.
    const int64_t step = 4 * nthreads, step_r = step / upr, step_c = step % upr;
    int64_t row[4], col[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int64_t u = gtid + j * nthreads;
        row[j] = u / upr;
        col[j] = u % upr;
    }
    uint32_t best = 0;
    while (row[0] < rows) {
        uint4 v[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            if (row[j] < rows)
                v[j] = __ldg(reinterpret_cast<const uint4 *>(p.x + (p.row_begin + row[j]) * p.ldx + col[j] * 8));
            else
                v[j] = make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            best = max(best, absmax_bits8(v[j]));
            col[j] += step_c;
            row[j] += step_r;
            if (col[j] >= upr) {
                col[j] -= upr;
                ++row[j];
            }
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        best = max(best, __shfl_xor_sync(0xFFFFFFFFu, best, o));
    __shared__ uint32_t warp_best[kQuantThreads / 32];
    if ((threadIdx.x & 31) == 0)
        warp_best[threadIdx.x >> 5] = best;
    __syncthreads();
    if (threadIdx.x == 0) {
        uint32_t b = 0;
        for (int w = 0; w < kQuantThreads / 32; ++w)
            b = max(b, warp_best[w]);
        p.partial[blockIdx.x] = b;
    }
}

// ------------------------------------------------------------------ encode

struct QuantParams {
    const uint16_t *x;
    int64_t rows, k, ldx;
    uint32_t *q;                 // packed codes, viewed as 32-bit words (8 codes)
    uint8_t *sf;                 // physical scale buffer
    int64_t rows_pad, kb_pad;    // padded scale-layout extents
    int nseg;
    int64_t seg_end[kMaxSeg];    // row end of each segment (last == rows)
    const float *static_scale;   // [nseg] or nullptr (dynamic)
    const uint32_t *partial;     // [nseg][npartial] amax partials (dynamic)
    int npartial;
    float *scale_out;            // [nseg]
    uint64_t timeout_ns;         // bound on the cluster kernel's wait for its peers' maxima
};

__global__ void __launch_bounds__(kQuantThreads) quantize_kernel(QuantParams p)
{
    __shared__ float s_scale[kMaxSeg];
    __shared__ float s_dg[kMaxSeg];
    const int lane = threadIdx.x & 31;

    // Wait for the amax pass (and everything before it), then let the GEMM that
    // follows start: from this point every kernel before this one has completed,
    // so the GEMM may stream weights while the codes below are being written.
    pdl_wait_prerequisites();
    pdl_launch_dependents();

    if (threadIdx.x < 32 * p.nseg && (threadIdx.x >> 5) < kMaxSeg) {
        // Per-segment global scale: given, or amax / 2688 from the amax partials.
        const int seg = threadIdx.x >> 5;
        float s;
        bool finite;
        if (p.static_scale != nullptr) {
            s = p.static_scale[seg];
            finite = isfinite(s) && s >= 0.0f;
        } else {
            uint32_t b = 0;
            for (int i = lane; i < p.npartial; i += 32)
                b = max(b, p.partial[seg * p.npartial + i]);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1)
                b = max(b, __shfl_xor_sync(0xFFFFFFFFu, b, o));
            finite = b < 0x7F80u;
            const float amax = __uint_as_float(b << 16);
            s = __fdiv_rn(amax, 2688.0f);
        }
        if (lane == 0) {
            if (!finite) {
                raise_device_error(4u /* NVFP4_ERR_NONFINITE */);
                s = 0.0f;
            }
            s_scale[seg] = s;
            s_dg[seg] = __fmul_rn(s, 6.0f);
            if (blockIdx.x == 0)
                p.scale_out[seg] = s;
        }
    }
    __syncthreads();

    const int64_t upr = p.k >> 3;
    const int64_t nthreads = static_cast<int64_t>(gridDim.x) * blockDim.x;
    const int64_t gtid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    // Four interleaved unit streams per thread; (row, col) advance by a fixed
    // step, so the loop holds no division.  Lane pairs (2i, 2i+1) always hold
    // the two halves of one 16-element block, lanes 8g..8g+7 four aligned blocks
    // of one row (nthreads is a multiple of 256 and upr of 8).
    const int64_t step = 4 * nthreads, step_r = step / upr, step_c = step % upr;
    int64_t row[4], col[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int64_t u = gtid + j * nthreads;
        row[j] = u / upr;
        col[j] = u % upr;
    }
    // Warp-uniform trip count: lane 0's first stream decides.
    int64_t wrow = __shfl_sync(0xFFFFFFFFu, row[0], 0);
    int64_t wcol = __shfl_sync(0xFFFFFFFFu, col[0], 0);

    while (wrow < p.rows) {
        uint4 v[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            if (row[j] < p.rows)
                v[j] = __ldg(reinterpret_cast<const uint4 *>(p.x + row[j] * p.ldx + col[j] * 8));
            else
                v[j] = make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const bool active = row[j] < p.rows;
            const int64_t r_ = active ? row[j] : 0;
            const int64_t c8 = col[j];

            uint32_t bm = absmax_bits8(v[j]);
            bm = max(bm, __shfl_xor_sync(0xFFFFFFFFu, bm, 1));
            const float bmax = __uint_as_float(bm << 16);

            int seg = 0;
#pragma unroll
            for (int s = 0; s < kMaxSeg - 1; ++s)
                seg += (s + 1 < p.nseg && r_ >= p.seg_end[s]) ? 1 : 0;
            const float s = s_scale[seg];
            const float dg = s_dg[seg];

            const float sbf = (dg == 0.0f) ? 0.0f : fminf(__fdiv_rn(bmax, dg), 448.0f);
            const uint32_t sb = f32_to_e4m3(sbf);
            const float d = __fmul_rn(e4m3_to_f32(sb), s);
            const float r = (d == 0.0f) ? 0.0f : fminf(__frcp_rn(d), FLT_MAX);

            const uint32_t w0 = v[j].x, w1 = v[j].y, w2 = v[j].z, w3 = v[j].w;
            const uint32_t codes = f32x8_to_e2m1x8(
                __fmul_rn(bf16lo(w0), r), __fmul_rn(bf16hi(w0), r), __fmul_rn(bf16lo(w1), r),
                __fmul_rn(bf16hi(w1), r), __fmul_rn(bf16lo(w2), r), __fmul_rn(bf16hi(w2), r),
                __fmul_rn(bf16lo(w3), r), __fmul_rn(bf16hi(w3), r));
            if (active)
                p.q[r_ * upr + c8] = codes;

            // Lanes 8g, 8g+2, 8g+4, 8g+6 hold the scales of four consecutive blocks
            // (k-block index = c8/2, aligned to 4) of one row: one 32-bit store.
            const uint32_t s1 = __shfl_down_sync(0xFFFFFFFFu, sb, 2);
            const uint32_t s2 = __shfl_down_sync(0xFFFFFFFFu, sb, 4);
            const uint32_t s3 = __shfl_down_sync(0xFFFFFFFFu, sb, 6);
            if (active && (lane & 7) == 0)
                *reinterpret_cast<uint32_t *>(p.sf + sf_atom_offset(r_, c8 >> 1, p.kb_pad)) =
                    sb | (s1 << 8) | (s2 << 16) | (s3 << 24);

            col[j] += step_c;
            row[j] += step_r;
            if (col[j] >= upr) {
                col[j] -= upr;
                ++row[j];
            }
        }
        wcol += step_c;
        wrow += step_r;
        if (wcol >= upr) {
            wcol -= upr;
            ++wrow;
        }
    }

    zero_pad_scales(p.sf, p.rows, p.rows_pad, p.kb_pad, gtid, nthreads);
}

// ------------------------------------------------------------------ encode, one cluster

// Decode-sized activations in one launch: a cluster of kClusterCtas CTAs (16:
// a non-portable cluster size the launcher opts into) holds the whole tensor in
// registers (at most UNITS 16-byte units per thread), reduces the
// absolute maximum over the cluster through distributed shared memory when the
// scale is dynamic, and encodes from the same registers -- one read of X, no
// amax pass, no workspace.  Unit-to-lane mapping, arithmetic and stores are
// those of quantize_kernel.
// Instances (units per thread x threads per CTA):
//   5 x 512   up to 327680 elements; 63 registers, so that a CTA fits beside the
//             two decode GEMM CTAs still running on an SM when it starts;
//   5 x 1024  up to 655360 elements (128 tokens at K = 5120), half the serial
//             work per thread of 10 x 512; a whole register file per CTA;
//   12 x 512  up to 786432 elements; 127 registers, a whole register file.
constexpr int kClusterCtas = 16;
constexpr int kClusterThreads = 512;

template <int UNITS, int THREADS>
__global__ void __cluster_dims__(kClusterCtas, 1, 1) __launch_bounds__(THREADS)
    quantize_cluster_kernel(QuantParams p)
{
    __shared__ uint32_t s_red[THREADS / 32];
    __shared__ uint32_t s_peer_max[kClusterCtas];        // entry r: CTA r's maximum, pushed by CTA r
    __shared__ __align__(8) uint64_t s_pushes;           // completes when all kClusterCtas entries landed
    __shared__ float s_sc[2];
    __shared__ int s_abort;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();

    // The exchange of CTA maxima: every CTA stores its maximum into entry `rank`
    // of every CTA's s_peer_max (itself included) with st.async, whose bytes
    // complete the receiver's s_pushes.  A cluster barrier phase (arrive here,
    // wait just before the first push) orders each barrier's initialisation
    // before any push; its latency hides under the loads.  A second phase
    // (arrive once the pushes to this CTA have landed, wait at the very end)
    // keeps every CTA resident until its own pushes have been received.
    // With a given (calibrated) scale there is nothing to exchange: no CTA of
    // the cluster touches another's shared memory and no barrier phase is used.
    const bool given = p.static_scale != nullptr;
    if (!given) {
        if (threadIdx.x == 0) {
            mbar_init(&s_pushes, 1);
            s_abort = 0;
            fence_barrier_init();
            mbar_arrive_expect_tx(&s_pushes, 4u * kClusterCtas);
        }
        cluster_arrive_release();
    }

    pdl_wait_prerequisites();
    pdl_launch_dependents();

    const int64_t upr = p.k >> 3;
    const int64_t total = p.rows * upr;
    const int64_t nthreads = static_cast<int64_t>(kClusterCtas) * THREADS;
    const int64_t gtid = static_cast<int64_t>(rank) * THREADS + threadIdx.x;
    // Unit j of this thread is gtid + j * nthreads; its (row, column) advance by a
    // fixed step, so only the first needs a division.
    // The launch covers at most kClusterCtas * THREADS * UNITS
    // units, so a unit's row and column fit in 32 bits.
    const int step_r = static_cast<int>(nthreads / upr), step_c = static_cast<int>(nthreads % upr);
    int row[UNITS], col[UNITS];
    row[0] = static_cast<int>(gtid / upr);
    col[0] = static_cast<int>(gtid % upr);
#pragma unroll
    for (int j = 1; j < UNITS; ++j) {
        row[j] = row[j - 1] + step_r;
        col[j] = col[j - 1] + step_c;
        if (col[j] >= upr) {
            col[j] -= upr;
            ++row[j];
        }
    }
    uint4 v[UNITS];
    uint32_t b = 0;
#pragma unroll
    for (int j = 0; j < UNITS; ++j) {
        v[j] = row[j] < p.rows ? __ldg(reinterpret_cast<const uint4 *>(p.x + static_cast<int64_t>(row[j]) * p.ldx +
                                                                    col[j] * 8))
                               : make_uint4(0, 0, 0, 0);
        b = max(b, absmax_bits8(v[j]));
    }
    if (!given) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            b = max(b, __shfl_xor_sync(0xFFFFFFFFu, b, o));
        if (lane == 0)
            s_red[threadIdx.x >> 5] = b;
        __syncthreads();
        cluster_wait_acquire();                          // every CTA's s_pushes is initialised
        if (threadIdx.x < 32) {
            uint32_t m = lane < THREADS / 32 ? s_red[lane] : 0u;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1)
                m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
            if (lane < kClusterCtas)
                st_async_remote_u32(map_to_rank(smem_u32(&s_peer_max[rank]), static_cast<uint32_t>(lane)), m,
                                    map_to_rank(smem_u32(&s_pushes), static_cast<uint32_t>(lane)));
            const bool ok = __all_sync(0xFFFFFFFFu, mbar_wait_bounded(&s_pushes, 0, &s_abort, p.timeout_ns));
            if (lane == 0) {
                uint32_t g = 0;
                for (int r = 0; r < kClusterCtas; ++r)
                    g = max(g, s_peer_max[r]);
                float sv = __fdiv_rn(__uint_as_float(g << 16), 2688.0f);
                if (!ok) {
                    raise_device_error(6u /* NVFP4_ERR_TIMEOUT */);
                    sv = 0.0f;
                } else if (g >= 0x7F80u) {
                    if (rank == 0)
                        raise_device_error(4u /* NVFP4_ERR_NONFINITE */);
                    sv = 0.0f;
                }
                s_sc[0] = sv;
                s_sc[1] = __fmul_rn(sv, 6.0f);
                if (rank == 0)
                    p.scale_out[0] = sv;
            }
        }
    } else if (threadIdx.x == 0) {
        float sv = p.static_scale[0];
        if (!(isfinite(sv) && sv >= 0.0f)) {
            if (rank == 0)
                raise_device_error(4u /* NVFP4_ERR_NONFINITE */);
            sv = 0.0f;
        }
        s_sc[0] = sv;
        s_sc[1] = __fmul_rn(sv, 6.0f);
        if (rank == 0)
            p.scale_out[0] = sv;
    }
    __syncthreads();
    if (!given)
        cluster_arrive_relaxed();                        // the pushes to this CTA have landed
    const float s = s_sc[0], dg = s_sc[1];

#pragma unroll
    for (int j = 0; j < UNITS; ++j) {
        const int64_t u = gtid + j * nthreads;
        if (__shfl_sync(0xFFFFFFFFu, u, 0) >= total)       // warp-uniform: lane 0 holds the warp's first unit
            break;
        const bool active = u < total;
        const int64_t r_ = active ? row[j] : 0;
        const int64_t c8 = active ? col[j] : 0;
        uint32_t bm = absmax_bits8(v[j]);
        bm = max(bm, __shfl_xor_sync(0xFFFFFFFFu, bm, 1));
        const float bmax = __uint_as_float(bm << 16);
        const float sbf = (dg == 0.0f) ? 0.0f : fminf(__fdiv_rn(bmax, dg), 448.0f);
        const uint32_t sb = f32_to_e4m3(sbf);
        const float d = __fmul_rn(e4m3_to_f32(sb), s);
        const float r = (d == 0.0f) ? 0.0f : fminf(__frcp_rn(d), FLT_MAX);
        const uint32_t w0 = v[j].x, w1 = v[j].y, w2 = v[j].z, w3 = v[j].w;
        const uint32_t codes = f32x8_to_e2m1x8(
            __fmul_rn(bf16lo(w0), r), __fmul_rn(bf16hi(w0), r), __fmul_rn(bf16lo(w1), r),
            __fmul_rn(bf16hi(w1), r), __fmul_rn(bf16lo(w2), r), __fmul_rn(bf16hi(w2), r),
            __fmul_rn(bf16lo(w3), r), __fmul_rn(bf16hi(w3), r));
        if (active)
            p.q[r_ * upr + c8] = codes;
        const uint32_t s1 = __shfl_down_sync(0xFFFFFFFFu, sb, 2);
        const uint32_t s2 = __shfl_down_sync(0xFFFFFFFFu, sb, 4);
        const uint32_t s3 = __shfl_down_sync(0xFFFFFFFFu, sb, 6);
        if (active && (lane & 7) == 0)
            *reinterpret_cast<uint32_t *>(p.sf + sf_atom_offset(r_, c8 >> 1, p.kb_pad)) =
                sb | (s1 << 8) | (s2 << 16) | (s3 << 24);
    }

    zero_pad_scales(p.sf, p.rows, p.rows_pad, p.kb_pad, gtid, nthreads);
    if (!given)
        cluster_wait_acquire();                          // every push from this CTA has been received
}

// ------------------------------------------------------------------ encode, tiled

// Large tensors: one CTA iteration owns a tile of 128 rows x 64 columns, i.e.
// exactly one 512-byte scale atom.  Thread t owns row t/2 and two whole
// 16-element blocks (64 contiguous input bytes -> 16 bytes of codes, two scale
// bytes); the atom is assembled in shared memory and leaves as 32 x 16-byte
// stores, so every output sector is written whole.  The next tile's four 16-byte
// loads are issued before the current tile is encoded.  Element arithmetic is
// identical to quantize_kernel (and to the CPU reference).
struct TileQuantParams {
    const uint16_t *x;
    int64_t rows, k, ldx;
    uint8_t *q;
    uint8_t *sf;
    int64_t row_tiles, col_tiles;    // ceil(rows/128), k/64
    int nseg;
    int64_t seg_end[kMaxSeg];
    const float *static_scale;
    const uint32_t *partial;
    int npartial;
    float *scale_out;
};

__device__ __forceinline__ uint64_t f32x2_mul(uint64_t a, uint64_t b)
{
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

// One 16-element block (8 words of bf16 pairs) -> 8 bytes of codes, scale byte.
__device__ __forceinline__ uint2 encode_block16(const uint32_t (&w)[8], const float *rcp, float dg, uint32_t &sb_out)
{
    const uint32_t msk = 0x7FFF7FFFu;
    uint32_t a = __vmaxu2(__vmaxu2(w[0] & msk, w[1] & msk), __vmaxu2(w[2] & msk, w[3] & msk));
    uint32_t b = __vmaxu2(__vmaxu2(w[4] & msk, w[5] & msk), __vmaxu2(w[6] & msk, w[7] & msk));
    uint32_t c = __vmaxu2(a, b);
    const float bmax = __uint_as_float(max(c >> 16, c & 0xFFFFu) << 16);
    const float sbf = (dg == 0.0f) ? 0.0f : fminf(__fdiv_rn(bmax, dg), 448.0f);
    const uint32_t sb = f32_to_e4m3(sbf);
    const float r = rcp[sb];                 // min(1 / (value(sb) * s), FLT_MAX), or 0
    const uint64_t rr = (static_cast<uint64_t>(__float_as_uint(r)) << 32) | __float_as_uint(r);
    float v[16];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const uint64_t pair = (static_cast<uint64_t>(w[i] & 0xFFFF0000u) << 32) | (w[i] << 16);
        const uint64_t prod = f32x2_mul(pair, rr);
        v[2 * i] = __uint_as_float(static_cast<uint32_t>(prod));
        v[2 * i + 1] = __uint_as_float(static_cast<uint32_t>(prod >> 32));
    }
    sb_out = sb;
    return make_uint2(f32x8_to_e2m1x8(v[0], v[1], v[2], v[3], v[4], v[5], v[6], v[7]),
                      f32x8_to_e2m1x8(v[8], v[9], v[10], v[11], v[12], v[13], v[14], v[15]));
}

__global__ void __launch_bounds__(kQuantThreads) quantize_tile_kernel(TileQuantParams p)
{
    __shared__ float s_scale[kMaxSeg];
    __shared__ float s_dg[kMaxSeg];
    __shared__ __align__(16) uint32_t s_atom[2][128];
    // Per segment, the element multiplier of every block-scale code c:
    // r = min(1 / (value(c) * s), FLT_MAX), 0 when value(c) * s == 0 -- the same
    // fp32 operations as computing it per block, done once per CTA.
    __shared__ float s_rcp[kMaxSeg][128];
    const int lane = threadIdx.x & 31;

    pdl_wait_prerequisites();
    pdl_launch_dependents();

    if (threadIdx.x < 32 * p.nseg && (threadIdx.x >> 5) < kMaxSeg) {
        const int seg = threadIdx.x >> 5;
        float s;
        bool finite;
        if (p.static_scale != nullptr) {
            s = p.static_scale[seg];
            finite = isfinite(s) && s >= 0.0f;
        } else {
            uint32_t b = 0;
            for (int i = lane; i < p.npartial; i += 32)
                b = max(b, p.partial[seg * p.npartial + i]);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1)
                b = max(b, __shfl_xor_sync(0xFFFFFFFFu, b, o));
            finite = b < 0x7F80u;
            s = __fdiv_rn(__uint_as_float(b << 16), 2688.0f);
        }
        if (lane == 0) {
            if (!finite) {
                raise_device_error(4u /* NVFP4_ERR_NONFINITE */);
                s = 0.0f;
            }
            s_scale[seg] = s;
            s_dg[seg] = __fmul_rn(s, 6.0f);
            if (blockIdx.x == 0)
                p.scale_out[seg] = s;
        }
    }
    __syncthreads();
    for (int idx = threadIdx.x; idx < p.nseg * 128; idx += blockDim.x) {
        const float d = __fmul_rn(e4m3_to_f32(static_cast<uint32_t>(idx & 127)), s_scale[idx >> 7]);
        s_rcp[idx >> 7][idx & 127] = (d == 0.0f) ? 0.0f : fminf(__frcp_rn(d), FLT_MAX);
    }
    __syncthreads();

    const int rl = threadIdx.x >> 1;                 // row inside the tile
    const int half = threadIdx.x & 1;                // columns [32*half, 32*half + 32) of the tile
    int buf = 0;
    // Tiles are visited grid-stride in row-tile-major order; (rt, ct) advance by a
    // fixed step instead of being divided out of the tile index.
    const int64_t step_r = gridDim.x / p.col_tiles, step_c = gridDim.x % p.col_tiles;
    int64_t rt = blockIdx.x / p.col_tiles, ct = blockIdx.x % p.col_tiles;
    auto advance = [&](int64_t &r, int64_t &c) {
        c += step_c;
        r += step_r;
        if (c >= p.col_tiles) {
            c -= p.col_tiles;
            ++r;
        }
    };
    auto load = [&](int64_t r, int64_t c, uint4 (&v)[4]) {
        const int64_t row = r * 128 + rl;
        if (r < p.row_tiles && row < p.rows) {
            const uint4 *src = reinterpret_cast<const uint4 *>(p.x + row * p.ldx + c * 64 + half * 32);
#pragma unroll
            for (int i = 0; i < 4; ++i)
                v[i] = __ldcs(src + i);
        } else {
#pragma unroll
            for (int i = 0; i < 4; ++i)
                v[i] = make_uint4(0, 0, 0, 0);
        }
    };
    uint4 cur[4];
    load(rt, ct, cur);
    while (rt < p.row_tiles) {
        int64_t rn = rt, cn = ct;
        advance(rn, cn);
        uint4 nxt[4];
        load(rn, cn, nxt);

        const int64_t row = rt * 128 + rl;
        const bool valid = row < p.rows;
        int seg = 0;
        if (p.nseg > 1) {
#pragma unroll
            for (int s = 0; s < kMaxSeg - 1; ++s)
                seg += (s + 1 < p.nseg && row >= p.seg_end[s]) ? 1 : 0;
        }
        const float *rcp = s_rcp[seg];
        const float dg = s_dg[seg];

        const uint32_t w0[8] = {cur[0].x, cur[0].y, cur[0].z, cur[0].w, cur[1].x, cur[1].y, cur[1].z, cur[1].w};
        const uint32_t w1[8] = {cur[2].x, cur[2].y, cur[2].z, cur[2].w, cur[3].x, cur[3].y, cur[3].z, cur[3].w};
        uint32_t sb0, sb1;
        const uint2 c0 = encode_block16(w0, rcp, dg, sb0);
        const uint2 c1 = encode_block16(w1, rcp, dg, sb1);
        if (valid)
            *reinterpret_cast<uint4 *>(p.q + row * (p.k >> 1) + ct * 32 + half * 16) = make_uint4(c0.x, c0.y, c1.x, c1.y);

        // Scale bytes of blocks (2*half, 2*half+1); the even lane assembles the row's four.
        const uint32_t mine = valid ? (sb0 | (sb1 << 8)) : 0u;
        const uint32_t other = __shfl_down_sync(0xFFFFFFFFu, mine, 1);
        if (half == 0)
            s_atom[buf][(rl & 31) * 4 + (rl >> 5)] = mine | (other << 16);
        __syncthreads();
        if (threadIdx.x < 32) {
            const uint4 v = reinterpret_cast<const uint4 *>(s_atom[buf])[threadIdx.x];
            *reinterpret_cast<uint4 *>(p.sf + (rt * p.col_tiles + ct) * 512 + threadIdx.x * 16) = v;
        }
        buf ^= 1;
#pragma unroll
        for (int i = 0; i < 4; ++i)
            cur[i] = nxt[i];
        rt = rn;
        ct = cn;
    }
}

}  // namespace nvfp4
