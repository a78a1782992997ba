// convert.cuh -- kernels that rewrite packed NVFP4 tensors rather than multiply
// them: expansion to bf16, checkpoint import of linear-layout block scales, and
// harmonization of a fused group's global scales.  All three are HBM-bound
// streams over the packed bytes.
//
//   * Expansion ("Gemma-4-31B-IT-NVFP4-FP8attn-text" model card, §Limitations:
//     a packed checkpoint is expanded to BF16 to load it elsewhere).  Element j
//     of row r becomes the bf16 nearest to value(code) * value(block scale) * s,
//     rounded once (ties to even).  Per 16-element block only eight magnitudes
//     occur; they are rounded exactly once per block into an 8-entry table, and
//     each element is a table look-up (byte permutes) plus its sign bit.
//   * Import ("Why Gated DeltaNet Survives 4-Bit Quantization", §3 "Checkpoints";
//     model card §Verification: packed codes, per-block E4M3 weight_scale and the
//     FP32 weight_scale_2): a [rows, K/16] block-scale matrix is scattered into
//     the tensor-core atom layout; the packed codes are already in the layout the
//     GEMM reads.
//   * Harmonization (same paper, §6 "Per-module calibration vs. fused-GEMM
//     scaling", the checkpoint-side repair): the fused group takes the largest of
//     its modules' global scales and every block scale of module i is re-rounded
//     to E4M3 after multiplying it by s_i / s_shared (both in fp32).
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "quantize.cuh"

namespace nvfp4 {
namespace convert {

constexpr int kThreads = 256;

// ------------------------------------------------------------------ exact bf16 rounding

// bf16 bits of the value p * s rounded once to nearest (ties to even), for p with
// at most 6 significant bits (an E2M1 value times an E4M3 value) and s any fp32.
// The exact product then has at most 30 significant bits, so the fp32 product hi
// is exact up to its rounding error lo = fma(p, s, -hi) as long as the lowest of
// those bits, 2^29 below the leading one, is not below fp32's smallest subnormal
// 2^-149: i.e. for |hi| >= 2^-120.  hi rounds to the same bf16 as p * s unless hi
// sits exactly on a bf16 midpoint, where the sign of lo decides.  Smaller
// products go through fp64, where the product is exact.  (A p with more bits
// would need a higher threshold: 2^-102 for 24 bits.)
__device__ __forceinline__ uint32_t bf16_bits_of_product(float p, float s)
{
    const float hi = __fmul_rn(p, s);
    const uint32_t u = __float_as_uint(hi);
    const uint32_t mag = u & 0x7FFFFFFFu;
    if (mag >= 0x7F800000u)                           // inf (or NaN from inf * 0)
        return (u >> 16) | (mag > 0x7F800000u ? 0x40u : 0u);
    if (mag == 0u)
        return u >> 16;
    if (mag < 0x03800000u) {                          // |hi| < 2^-120
        const __nv_bfloat16 b = __double2bfloat16(static_cast<double>(p) * static_cast<double>(s));
        return static_cast<uint32_t>(__bfloat16_as_ushort(b));
    }
    uint32_t r = (u + 0x7FFFu + ((u >> 16) & 1u)) >> 16;
    if ((u & 0xFFFFu) == 0x8000u) {
        const float lo = __fmaf_rn(p, s, -hi);
        if (lo != 0.0f)
            r = (u >> 16) + (((lo > 0.0f) == (hi > 0.0f)) ? 1u : 0u);
    }
    return r & 0xFFFFu;
}

// E2M1 magnitude code (0..7) -> value (0, 0.5, 1, 1.5, 2, 3, 4, 6).
__device__ __forceinline__ float e2m1_magnitude(uint32_t m)
{
    if (m < 2u)
        return 0.5f * static_cast<float>(m);
    return __uint_as_float(((126u + (m >> 1)) << 23) | ((m & 1u) << 22));
}

// The eight bf16 magnitudes of one block, split into a low-byte table (lo0: entries
// 0..3, lo1: 4..7) and a high-byte table, for byte-permute look-ups.  The E2M1
// magnitudes are 1 and 1.5 times powers of two, and rounding commutes with a
// power-of-two scaling while both values stay normal; so only value(sb)*s and
// 1.5*value(sb)*s are rounded, and the rest are exponent shifts of those two.
// Outside that range every entry is rounded on its own.
struct BlockTable {
    uint32_t lo0, lo1, hi0, hi1;
};

__device__ __forceinline__ BlockTable block_table(float sd, float s)
{
    uint32_t e[8];
    e[0] = 0u;
    const uint32_t c1 = bf16_bits_of_product(sd, s);
    const uint32_t c15 = bf16_bits_of_product(1.5f * sd, s);       // exact: sd has 4 significant bits
    const uint32_t x1 = (c1 >> 7) & 0xFFu, x15 = (c15 >> 7) & 0xFFu;
    if (x1 >= 3u && x1 <= 252u && x15 >= 2u && x15 <= 252u) {
        e[1] = c1 - 0x80u;       // 0.5
        e[2] = c1;               // 1
        e[3] = c15;              // 1.5
        e[4] = c1 + 0x80u;       // 2
        e[5] = c15 + 0x80u;      // 3
        e[6] = c1 + 0x100u;      // 4
        e[7] = c15 + 0x100u;     // 6
    } else {
#pragma unroll
        for (int m = 1; m < 8; ++m)
            e[m] = bf16_bits_of_product(e2m1_magnitude(m) * sd, s);   // e2m1 * e4m3 is exact in fp32
    }
    // e[i] holds a bf16 pattern in its low 16 bits; gather low and high bytes.
    const uint32_t x01 = __byte_perm(e[0], e[1], 0x5410u), x23 = __byte_perm(e[2], e[3], 0x5410u);
    const uint32_t x45 = __byte_perm(e[4], e[5], 0x5410u), x67 = __byte_perm(e[6], e[7], 0x5410u);
    BlockTable t;
    t.lo0 = __byte_perm(x01, x23, 0x6420u);
    t.hi0 = __byte_perm(x01, x23, 0x7531u);
    t.lo1 = __byte_perm(x45, x67, 0x6420u);
    t.hi1 = __byte_perm(x45, x67, 0x7531u);
    return t;
}

// PTX byte permute in its default mode: selector nibble n's low three bits pick
// byte n of the result from {a (bytes 0..3), b (bytes 4..7)}; with the nibble's
// bit 3 set the result byte is the picked byte's bit 7 replicated (0x00 / 0xFF).
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel)
{
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

// Four codes (nibbles 0..3 of `w`, element order) -> two words of bf16 pairs.
// The high-byte table may carry the block scale's sign in bit 7 of every entry.
__device__ __forceinline__ void expand4(const BlockTable &t, uint32_t w, uint32_t &out0, uint32_t &out1)
{
    const uint32_t sel = w & 0x7777u;                          // magnitude indices
    const uint32_t lo = prmt(t.lo0, t.lo1, sel);               // low bytes of elements 0..3
    // Code signs (bit 3 of each nibble) as bit 7 of element bytes 0..3: the
    // sign-replicating picks read codes 0 and 2 from w << 4 (their sign bits at 7
    // and 15) and codes 1 and 3 from w itself (at 7 and 15).
    const uint32_t sg = prmt(w << 4, w, 0xD9C8u) & 0x80808080u;
    const uint32_t hi = prmt(t.hi0, t.hi1, sel) ^ sg;          // high bytes of elements 0..3
    out0 = prmt(lo, hi, 0x5140u);
    out1 = prmt(lo, hi, 0x7362u);
}

// ------------------------------------------------------------------ expansion

struct ExpandParams {
    const uint8_t *q;          // [rows, k/2]
    const uint8_t *sf;         // physical scales
    uint16_t *y;               // bf16 [rows, ldy]
    int64_t rows, k, ldy;
    int64_t row_tiles, col_tiles;   // 128-row x 64-column tiles (one scale atom each)
    int nseg;
    int64_t seg_end[kMaxSeg];
    const float *gscale;       // [nseg] device
};

// A block's eight bf16 magnitudes depend only on its scale byte and its
// segment's global scale, so each CTA first tabulates them for all 128
// non-negative E4M3 codes of every segment (16 bytes per entry, at most 16 KB of
// shared memory).  One tile = 128 rows x 64 elements = one 512-byte scale atom;
// thread t expands 8 consecutive elements (4 bytes of codes -> one 16-byte bf16
// store) in each of the rows t/8 + 32j, j = 0..3, so a warp's store covers four
// whole 128-byte row segments; its four scale bytes sit in one 16-byte word of
// the atom.  The next tile's codes and scales are loaded before the current
// tile is expanded.  A scale byte with its sign bit set negates the block.
__global__ void __launch_bounds__(kThreads) expand_kernel(ExpandParams p)
{
    __shared__ uint4 s_lut[kMaxSeg * 128];
    for (int idx = threadIdx.x; idx < p.nseg * 128; idx += blockDim.x) {
        const BlockTable tb = block_table(e4m3_to_f32(static_cast<uint32_t>(idx & 127)), p.gscale[idx >> 7]);
        s_lut[idx] = make_uint4(tb.lo0, tb.lo1, tb.hi0, tb.hi1);
    }
    __syncthreads();
    const int g = threadIdx.x & 7;              // 8-element group inside the 64 columns
    const int rsub = threadIdx.x >> 3;          // row inside each 32-row quarter
    const int64_t tiles = p.row_tiles * p.col_tiles;
    const int64_t kh = p.k >> 1;
    // (row tile, column tile) advance by a precomputed step: no division in the loop.
    const int64_t step_r = gridDim.x / p.col_tiles, step_c = gridDim.x % p.col_tiles;
    auto load = [&](int64_t t, int64_t rt, int64_t ct, uint4 &sfw, uint32_t (&codes)[4]) {
        sfw = __ldg(reinterpret_cast<const uint4 *>(p.sf + t * 512 + rsub * 16));
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int64_t row = rt * 128 + j * 32 + rsub;
            codes[j] = row < p.rows ? __ldg(reinterpret_cast<const uint32_t *>(p.q + row * kh + ct * 32 + g * 4)) : 0u;
        }
    };

    int64_t t = blockIdx.x;
    int64_t rt = t / p.col_tiles, ct = t % p.col_tiles;
    uint4 sfw = make_uint4(0, 0, 0, 0);
    uint32_t codes[4] = {0u, 0u, 0u, 0u};
    if (t < tiles)
        load(t, rt, ct, sfw, codes);
    for (; t < tiles; t += gridDim.x) {
        int64_t nrt = rt + step_r, nct = ct + step_c;
        if (nct >= p.col_tiles) {
            nct -= p.col_tiles;
            ++nrt;
        }
        const uint32_t sfv[4] = {sfw.x, sfw.y, sfw.z, sfw.w};
        const uint32_t cur[4] = {codes[0], codes[1], codes[2], codes[3]};
        if (t + gridDim.x < tiles)
            load(t + gridDim.x, nrt, nct, sfw, codes);   // next tile's loads in flight during the expansion
        // The thread's rows in this tile are row0 + 32 j; the segment index only
        // moves forward along them, and the output pointer advances by 32 rows.
        const int64_t row0 = rt * 128 + rsub;
        const int64_t left = row0 >= p.rows ? 0 : (p.rows - row0 + 31) >> 5;   // rows of the thread in this tile
        const int rows_here = left < 4 ? static_cast<int>(left) : 4;
        uint16_t *out = p.y + row0 * p.ldy + ct * 64 + g * 8;
        int seg = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            if (j >= rows_here)
                break;
            while (seg < p.nseg - 1 && row0 + 32 * j >= p.seg_end[seg])
                ++seg;
            const uint32_t sb = (sfv[j] >> (8 * (g >> 1))) & 0xFFu;
            const uint4 tv = s_lut[seg * 128 + (sb & 0x7Fu)];
            // A scale byte with its sign bit set negates the block: flip bit 7 of
            // every high-byte table entry once instead of every output element.
            const uint32_t neg = (sb & 0x80u) ? 0x80808080u : 0u;
            const BlockTable tb = {tv.x, tv.y, tv.z ^ neg, tv.w ^ neg};
            uint4 o;
            expand4(tb, cur[j], o.x, o.y);
            expand4(tb, cur[j] >> 16, o.z, o.w);
            *reinterpret_cast<uint4 *>(out) = o;
            out += 32 * p.ldy;
        }
        rt = nrt;
        ct = nct;
    }
}

// ------------------------------------------------------------------ checkpoint import

struct ImportParams {
    const uint8_t *lin;        // [rows, k/16] bytes, row stride ld (bytes, multiple of 4)
    uint8_t *sf;               // physical scales
    int64_t rows, ld;
    int64_t row_tiles, atoms_k;     // tiles are 128 rows x 16 atoms (64 scale columns)
    int64_t col_groups;             // ceil(atoms_k / 16)
};


// One tile = 128 rows x 64 scale columns (16 atoms).  The rows are read as
// 4-byte words (one atom's four columns), 16 words per row, two rows per warp
// instruction; they are transposed through shared memory (row stride 17 words:
// no bank conflicts) and the 16 atoms leave as one contiguous 8 KB run of
// 16-byte stores.
__global__ void __launch_bounds__(kThreads) import_scales_kernel(ImportParams p)
{
    __shared__ uint32_t tile[128][17];
    const int64_t tiles = p.row_tiles * p.col_groups;
    const int64_t step_r = gridDim.x / p.col_groups, step_c = gridDim.x % p.col_groups;
    int64_t rt = blockIdx.x / p.col_groups, cg = blockIdx.x % p.col_groups;
    for (int64_t t = blockIdx.x; t < tiles; t += gridDim.x) {
        const int64_t a0 = cg * 16;
        const int natoms = static_cast<int>(p.atoms_k - a0 < 16 ? p.atoms_k - a0 : 16);
        const int w = threadIdx.x & 15;
#pragma unroll
        for (int r0 = 0; r0 < 128; r0 += kThreads / 16) {
            const int r = r0 + (threadIdx.x >> 4);
            const int64_t row = rt * 128 + r;
            tile[r][w] = (row < p.rows && w < natoms)
                             ? __ldg(reinterpret_cast<const uint32_t *>(p.lin + row * p.ld + (a0 + w) * 4))
                             : 0u;
        }
        __syncthreads();
        for (int i = threadIdx.x; i < natoms * 32; i += blockDim.x) {
            const int a = i >> 5, r = i & 31;        // atom, and row inside a 32-row quarter
            *reinterpret_cast<uint4 *>(p.sf + (rt * p.atoms_k + a0 + a) * 512 + r * 16) =
                make_uint4(tile[r][a], tile[32 + r][a], tile[64 + r][a], tile[96 + r][a]);
        }
        __syncthreads();
        rt += step_r;
        cg += step_c;
        if (cg >= p.col_groups) {
            cg -= p.col_groups;
            ++rt;
        }
    }
}

// ------------------------------------------------------------------ harmonization

struct HarmonizeParams {
    const uint8_t *sf_in;
    uint8_t *sf_out;           // may alias sf_in
    int64_t rows, atoms_k;     // atoms along K per 128-row block
    int64_t units;             // 16-byte words of the physical buffer
    int nseg;
    int64_t seg_end[kMaxSeg];
    const float *gscale;       // [nseg] device
    float *shared_out;         // 1 float, device
};

// Thread handles one 16-byte word of an atom: rows 32j + (word index) of the
// atom's 128-row block, j = 0..3, four scale columns each.  Each CTA derives the
// shared scale and the per-module ratios itself from the device scales.
__global__ void __launch_bounds__(kThreads) harmonize_kernel(HarmonizeParams p)
{
    __shared__ float s_ratio[kMaxSeg];
    __shared__ int s_state;                    // 0 fold, 1 copy unchanged (all zero), 2 bad scale
    // Per segment, the folded byte of every scale byte b:
    // E4M3(value(b) * ratio) -- the same fp32 operations as folding it in place.
    __shared__ uint8_t s_fold[kMaxSeg][256];
    __shared__ int64_t s_end[kMaxSeg];
    if (threadIdx.x == 0) {
#pragma unroll
        for (int i = 0; i < kMaxSeg; ++i)
            s_end[i] = p.seg_end[i];
        float shared = 0.0f;
        int bad = 0;
        for (int i = 0; i < p.nseg; ++i) {
            const float g = p.gscale[i];
            if (!(g >= 0.0f) || isinf(g))
                bad = 1;
            else
                shared = fmaxf(shared, g);
        }
        s_state = bad ? 2 : (shared == 0.0f ? 1 : 0);
        for (int i = 0; i < kMaxSeg; ++i)
            s_ratio[i] = (!bad && shared != 0.0f && i < p.nseg) ? __fdiv_rn(p.gscale[i], shared) : 1.0f;
        if (blockIdx.x == 0) {
            *p.shared_out = bad ? __int_as_float(0x7FC00000) : shared;
            if (bad)
                raise_device_error(4u /* NVFP4_ERR_NONFINITE */);
        }
    }
    __syncthreads();
    const int state = s_state;
    if (state == 2)
        return;                                // leave the scales as they are
    if (state == 0) {
        for (int idx = threadIdx.x; idx < p.nseg * 256; idx += blockDim.x) {
            const uint32_t b = static_cast<uint32_t>(idx & 255);
            const float folded = __fmul_rn(e4m3_to_f32(b), s_ratio[idx >> 8]);
            // A NaN byte (0x7F, 0xFF) stays as it is (NaN times the ratio is NaN).
            s_fold[idx >> 8][b] = (b & 0x7Fu) == 0x7Fu ? static_cast<uint8_t>(b) : static_cast<uint8_t>(f32_to_e4m3(folded));
        }
        __syncthreads();
    }
    const int atoms_k = static_cast<int>(p.atoms_k);
    const int64_t nthreads = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t u = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; u < p.units; u += nthreads) {
        uint4 v = __ldg(reinterpret_cast<const uint4 *>(p.sf_in) + u);
        if (state == 0) {
            // Word u is line w of atom u / 32: rows 128 rb + 32 j + w (j = 0..3) of
            // 128-row block rb; the segment index only moves forward along them.
            const int64_t rb = static_cast<int64_t>(static_cast<uint32_t>(u >> 5) / static_cast<uint32_t>(atoms_k));
            const int w = static_cast<int>(u & 31);
            uint32_t words[4] = {v.x, v.y, v.z, v.w};
            int seg = 0;
            uint32_t nan_bytes = 0;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int64_t row = rb * 128 + j * 32 + w;
                if (row < p.rows) {            // pad rows stay as they are
                    while (seg < p.nseg - 1 && row >= s_end[seg])
                        ++seg;
                    const uint8_t *f = s_fold[seg];
                    const uint32_t x = words[j];
                    // A byte of x is a NaN code iff its low 7 bits are all set:
                    // t has a zero byte exactly there (zero-byte test on t).
                    const uint32_t t = (x & 0x7F7F7F7Fu) ^ 0x7F7F7F7Fu;
                    nan_bytes |= (t - 0x01010101u) & ~t & 0x80808080u;
                    words[j] = static_cast<uint32_t>(f[x & 0xFFu]) | (static_cast<uint32_t>(f[(x >> 8) & 0xFFu]) << 8) |
                               (static_cast<uint32_t>(f[(x >> 16) & 0xFFu]) << 16) |
                               (static_cast<uint32_t>(f[x >> 24]) << 24);
                }
            }
            v = make_uint4(words[0], words[1], words[2], words[3]);
            if (nan_bytes != 0)
                raise_device_error(4u /* NVFP4_ERR_NONFINITE */);
        }
        reinterpret_cast<uint4 *>(p.sf_out)[u] = v;
    }
}

}  // namespace convert
}  // namespace nvfp4
