/*
 * nvfp4_oracle.c -- plain, slow CPU reference for the NVFP4 W4A4 linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or calls
 * this file; only the tests, the smoke check and the benchmark's CPU-baseline leg
 * do.  It shares no code, header, table or constant generator with the CUDA
 * library.
 *
 * What it follows:
 *  - "Why Gated DeltaNet Survives 4-Bit Quantization", §2 "NVFP4": values are
 *    E2M1 (4 bits), one E4M3 scale per 16-element block set to blockmax/6, one
 *    FP32 scale per tensor; W4A4 quantizes weights and activations alike and the
 *    GEMM consumes both.
 *  - same paper, §5 intro: "fake quantization" (quantize, dequantize, continue in
 *    high precision) -- the GEMM below dequantizes and accumulates in fp64.
 *  - same paper, §6 "Per-module calibration vs. fused-GEMM scaling": each module
 *    of a fused GEMM keeps its own FP32 global scale; collapsing them to the
 *    maximum without touching the block scales is the mismatch that paragraph
 *    describes (kept here only as a negative control).
 *  - "Gemma-4-31B-IT-NVFP4-FP8attn-text" model card, §Verification: the stored
 *    per-tensor scale satisfies max(block scale) x global x 6 = absmax, 6 being
 *    the largest E2M1 magnitude, so the global scale is the dequantization
 *    multiplier absmax / (6 * 448); §Limitations: packed uint8 holding two codes
 *    per byte along the input dimension.
 *
 * Readings where the pages are silent (each one is listed in the design notes):
 *  R1  amax is the exact max |x| over the tensor (segment) in fp32.
 *  R2  s = amax / 2688 in fp32 round-to-nearest (2688 = 6 * 448).
 *  R4  d_g = s * 6 (fp32); sb_f = min(bmax / d_g, 448) (fp32); d_g == 0 -> sb_f = 0.
 *  R5  sb = E4M3(sb_f): nearest E4M3 (FN, bias 7, subnormals kept, max 448)
 *      value, ties to the even code, saturating at 448 (0x7E); never 0x7F.
 *  R6  sd = value(sb); d = sd * s (fp32); r = 0 if d == 0 else min(1/d, FLT_MAX).
 *  R7  v = x * r (fp32); code = E2M1(v): nearest grid value, ties to the even
 *      code, |v| beyond 6 saturates to 6; the sign bit is the sign of v, so
 *      negative values that round to zero encode as 0x8.
 *  R9  byte j of a packed row holds code(2j) in bits 0..3 and code(2j+1) in
 *      bits 4..7.
 *  R10 physical scale layout consumed by the tensor cores: rows padded to 128,
 *      scale columns padded to 4; 512-byte atoms of 128 rows x 4 scale columns,
 *      atoms ordered K-fastest; inside an atom byte (r%32)*16 + ((r%128)/32)*4 + c%4.
 *      Pad bytes are 0.
 *  R11 GEMM: exact fp64 sum over k of value(code_x)*sd_x * value(code_w)*sd_w,
 *      then times s_x and times s_w of the column's segment, in fp64.
 *  R14 Dequantization to bf16 (the model card's "expand to BF16"): each element
 *      is value(code) * value(block scale) * s, a product that is exact in fp64
 *      (2 + 4 + 24 significant bits), rounded once to the nearest bf16, ties to
 *      the even significand.
 *  R15 Harmonization of a fused group ("Why Gated DeltaNet Survives 4-Bit
 *      Quantization", §6, the checkpoint-side repair): the group's shared global
 *      scale is the largest of its modules' scales, s_shared = max_i s_i, and
 *      every block scale of module i becomes E4M3(value(sb) * (s_i / s_shared)),
 *      ratio and product in fp32 round-to-nearest, then R5's rounding.  With the
 *      largest scale as the shared one every ratio is <= 1, so no folded scale
 *      can pass 448 and the re-rounding error stays within E4M3's half ulp
 *      (2^-4 relative in the normal range; the paper reports <= 6.2%).
 *      A NaN block-scale byte (0x7F or 0xFF; only a corrupt checkpoint holds
 *      one) stays as it is: NaN times the ratio is NaN under IEEE rules, and
 *      E4M3's NaN code keeps its sign bit.
 *  R16 Checkpoint import: a linear-layout block-scale matrix [rows, K/16]
 *      (one E4M3 byte per block, rows contiguous) is the logical matrix that
 *      R10 scatters; the packed codes need no change (same nibble order, R9).
 *
 * Build: gcc -O2 -fopenmp -fPIC -shared -ffp-contract=off -fno-fast-math
 */
#include <float.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------------ */
/* Number formats                                                            */
/* ------------------------------------------------------------------------ */

/* E2M1: bit 3 sign, bits 2..1 exponent (bias 1), bit 0 mantissa.
 * Exponent field 0 is subnormal: 0.m x 2^0 = m/2.  Magnitudes 0,0.5,1,1.5,2,3,4,6. */
double or_e2m1_value(uint32_t code)
{
    uint32_t sign = (code >> 3) & 1u, e = (code >> 1) & 3u, m = code & 1u;
    double mag;
    if (e == 0)
        mag = 0.5 * (double)m;
    else
        mag = ldexp(1.0 + 0.5 * (double)m, (int)e - 1);
    return sign ? -mag : mag;
}

/* E4M3, "FN" flavour: bit 7 sign, bits 6..3 exponent (bias 7), bits 2..0 mantissa.
 * No infinities; exponent 15 with mantissa 7 is NaN; largest finite 448 (0x7E).
 * Exponent field 0 is subnormal: m/8 x 2^-6. */
double or_e4m3_value(uint32_t code)
{
    uint32_t sign = (code >> 7) & 1u, e = (code >> 3) & 15u, m = code & 7u;
    double mag;
    if (e == 15 && m == 7)
        return NAN;
    if (e == 0)
        mag = ldexp((double)m / 8.0, -6);
    else
        mag = ldexp(1.0 + (double)m / 8.0, (int)e - 7);
    return sign ? -mag : mag;
}

/* Index of the representable magnitude nearest to a >= 0 among codes
 * 0..ncodes-1 (ascending values); a tie goes to the even code; anything past
 * the last value is that last value (saturation). */
static uint32_t nearest_code(double a, double (*value)(uint32_t), uint32_t ncodes)
{
    double top = value(ncodes - 1);
    if (!(a <= top))
        return ncodes - 1;
    uint32_t best = 0;
    double best_dist = fabs(a - value(0));
    for (uint32_t c = 1; c < ncodes; ++c) {
        double dist = fabs(a - value(c));
        if (dist < best_dist || (dist == best_dist && (c & 1u) == 0)) {
            best = c;
            best_dist = dist;
        }
    }
    return best;
}

/* E2M1 encode with round-to-nearest-even and saturation at 6 (R7). */
uint32_t or_e2m1_encode(float v)
{
    uint32_t sign = signbit(v) ? 8u : 0u;
    return sign | nearest_code(fabs((double)v), or_e2m1_value, 8);
}

/* E4M3 encode of a non-negative scale with round-to-nearest-even and
 * saturation at 448 (R5); the 127 finite non-negative codes are searched. */
uint32_t or_e4m3_encode(float v)
{
    uint32_t sign = signbit(v) ? 0x80u : 0u;
    return sign | nearest_code(fabs((double)v), or_e4m3_value, 127);
}

float or_bf16_to_f32(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* ------------------------------------------------------------------------ */
/* Scales                                                                    */
/* ------------------------------------------------------------------------ */

/* R1: max |x| over rows [r0, r1) of a bf16 matrix with row stride ld. */
float or_amax_bf16(const uint16_t *x, int64_t r0, int64_t r1, int64_t k, int64_t ld)
{
    float amax = 0.0f;
    for (int64_t r = r0; r < r1; ++r)
        for (int64_t j = 0; j < k; ++j) {
            float a = fabsf(or_bf16_to_f32(x[r * ld + j]));
            if (a > amax || isnan(a))
                amax = a;
        }
    return amax;
}

/* R2: per-tensor global scale, the dequantization multiplier. */
float or_global_scale(float amax)
{
    float six_times_448 = 6.0f * 448.0f; /* 2688, exact */
    return amax / six_times_448;
}

/* R4 + R5: E4M3 block scale for a block with max magnitude bmax under global s. */
uint32_t or_block_scale(float bmax, float s)
{
    float d_g = s * 6.0f;
    float sb_f = (d_g == 0.0f) ? 0.0f : bmax / d_g;
    if (sb_f > 448.0f)
        sb_f = 448.0f;
    return or_e4m3_encode(sb_f);
}

/* ------------------------------------------------------------------------ */
/* Quantization of rows                                                      */
/* ------------------------------------------------------------------------ */

/* Quantize rows of a bf16 matrix X[rows, k] (row stride ld, k % 16 == 0).
 * row_scale[r] is the FP32 global scale of the row's tensor (segment).
 * Outputs: q[rows, k/2] packed codes (R9), sf[rows, k/16] logical E4M3 block
 * scales, one byte per 16-element block along k. */
void or_quantize(const uint16_t *x, int64_t rows, int64_t k, int64_t ld, const float *row_scale,
                 uint8_t *q, uint8_t *sf)
{
    const int64_t nblk = k / 16;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        const float s = row_scale[r];
        for (int64_t b = 0; b < nblk; ++b) {
            const uint16_t *blk = x + r * ld + b * 16;
            float vals[16];
            float bmax = 0.0f;
            for (int i = 0; i < 16; ++i) {
                vals[i] = or_bf16_to_f32(blk[i]);
                if (fabsf(vals[i]) > bmax)
                    bmax = fabsf(vals[i]);
            }
            uint32_t sb = or_block_scale(bmax, s);                  /* R4, R5 */
            float sd = (float)or_e4m3_value(sb);
            float d = sd * s;                                       /* R6 */
            float rcp = 0.0f;
            if (d != 0.0f) {
                rcp = 1.0f / d;
                if (rcp > FLT_MAX)
                    rcp = FLT_MAX;
            }
            sf[r * nblk + b] = (uint8_t)sb;
            for (int i = 0; i < 16; i += 2) {                       /* R7, R9 */
                float v0 = vals[i] * rcp;
                float v1 = vals[i + 1] * rcp;
                uint32_t lo = or_e2m1_encode(v0), hi = or_e2m1_encode(v1);
                q[r * (k / 2) + b * 8 + i / 2] = (uint8_t)(lo | (hi << 4));
            }
        }
    }
}

/* Dequantize packed rows back to fp64 values (global scale included). */
void or_dequantize(const uint8_t *q, const uint8_t *sf, int64_t rows, int64_t k, const float *row_scale,
                   double *out)
{
    const int64_t nblk = k / 16;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t j = 0; j < k; ++j) {
            uint8_t byte = q[r * (k / 2) + j / 2];
            uint32_t code = (j & 1) ? (byte >> 4) : (byte & 15u);
            out[r * k + j] = or_e2m1_value(code) * or_e4m3_value(sf[r * nblk + j / 16]) * (double)row_scale[r];
        }
}

/* ------------------------------------------------------------------------ */
/* Physical scale-factor layout (R10)                                        */
/* ------------------------------------------------------------------------ */

int64_t or_sf_physical_bytes(int64_t rows, int64_t k)
{
    int64_t rows_pad = (rows + 127) / 128 * 128;
    int64_t cols_pad = ((k / 16) + 3) / 4 * 4;
    return rows_pad * cols_pad;
}

int64_t or_sf_offset(int64_t r, int64_t c, int64_t k)
{
    int64_t cols_pad = ((k / 16) + 3) / 4 * 4;
    int64_t atoms_per_row_block = cols_pad / 4;
    int64_t atom = (r / 128) * atoms_per_row_block + c / 4;
    return atom * 512 + (r % 32) * 16 + ((r % 128) / 32) * 4 + (c % 4);
}

/* Scatter logical sf[rows, k/16] into the physical buffer (pads zero). */
void or_sf_to_physical(const uint8_t *sf, int64_t rows, int64_t k, uint8_t *phys)
{
    memset(phys, 0, (size_t)or_sf_physical_bytes(rows, k));
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < k / 16; ++c)
            phys[or_sf_offset(r, c, k)] = sf[r * (k / 16) + c];
}

/* ------------------------------------------------------------------------ */
/* GEMM on dequantized operands (R11)                                        */
/* ------------------------------------------------------------------------ */

/* out[i, n] (i over the nsel selected activation rows) =
 *   sum_k deq(Qx)[rows[i], k] * deq(Qw)[n, k]  with per-operand E4M3 block scales,
 * times s_x times col_scale[n], all in fp64.  col_scale[n] is the weight global
 * scale of the segment that holds output column n. */
void or_linear_rows(const uint8_t *qx, const uint8_t *sfx, float s_x, const int64_t *rows, int64_t nsel,
                    const uint8_t *qw, const uint8_t *sfw, const float *col_scale, int64_t n, int64_t k,
                    double *out)
{
    const int64_t nblk = k / 16;
    double *xd = (double *)malloc(sizeof(double) * (size_t)(nsel * k));
    for (int64_t i = 0; i < nsel; ++i)
        for (int64_t j = 0; j < k; ++j) {
            uint8_t byte = qx[rows[i] * (k / 2) + j / 2];
            uint32_t code = (j & 1) ? (byte >> 4) : (byte & 15u);
            xd[i * k + j] = or_e2m1_value(code) * or_e4m3_value(sfx[rows[i] * nblk + j / 16]);
        }
#pragma omp parallel
    {
        double *wd = (double *)malloc(sizeof(double) * (size_t)k);
#pragma omp for schedule(static)
        for (int64_t c = 0; c < n; ++c) {
            for (int64_t j = 0; j < k; ++j) {
                uint8_t byte = qw[c * (k / 2) + j / 2];
                uint32_t code = (j & 1) ? (byte >> 4) : (byte & 15u);
                wd[j] = or_e2m1_value(code) * or_e4m3_value(sfw[c * nblk + j / 16]);
            }
            for (int64_t i = 0; i < nsel; ++i) {
                double acc = 0.0;
                for (int64_t j = 0; j < k; ++j)
                    acc += xd[i * k + j] * wd[j];
                out[i * n + c] = acc * (double)s_x * (double)col_scale[c];
            }
        }
        free(wd);
    }
    free(xd);
}

int or_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ------------------------------------------------------------------------ */
/* bf16 rounding and dequantization to bf16 (R14)                            */
/* ------------------------------------------------------------------------ */

/* Nearest bf16 (8 significant bits, fp32's exponent range, subnormals kept) to
 * a double; a tie goes to the even significand; a magnitude at or past the
 * largest finite value plus half an ulp becomes infinity.  Returns the bits. */
uint16_t or_bf16_from_f64(double v)
{
    if (isnan(v))
        return 0x7FC0u;
    uint16_t sign = signbit(v) ? 0x8000u : 0u;
    double a = fabs(v);
    if (a == 0.0)
        return sign;
    if (isinf(a))
        return (uint16_t)(sign | 0x7F80u);
    int e;
    frexp(a, &e);                        /* a in [2^(e-1), 2^e) */
    int qexp = e - 8;                    /* spacing of 8-significant-bit values there */
    if (qexp < -133)                     /* subnormal spacing 2^-126 * 2^-7 */
        qexp = -133;
    double r = nearbyint(ldexp(a, -qexp));   /* exact scaling; nearest integer, ties to even */
    double rounded = ldexp(r, qexp);
    if (rounded >= ldexp(1.0, 128))
        return (uint16_t)(sign | 0x7F80u);
    float f = (float)rounded;            /* exact: at most 8 significant bits, inside fp32's range */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return (uint16_t)(sign | ((u >> 16) & 0x7FFFu));
}

/* Dequantize packed rows to bf16: out[r, j] = bf16(value(code) * value(sf) * s_r). */
void or_dequantize_bf16(const uint8_t *q, const uint8_t *sf, int64_t rows, int64_t k, const float *row_scale,
                        uint16_t *out)
{
    const int64_t nblk = k / 16;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t j = 0; j < k; ++j) {
            uint8_t byte = q[r * (k / 2) + j / 2];
            uint32_t code = (j & 1) ? (byte >> 4) : (byte & 15u);
            double exact = or_e2m1_value(code) * or_e4m3_value(sf[r * nblk + j / 16]) * (double)row_scale[r];
            out[r * k + j] = or_bf16_from_f64(exact);
        }
}

/* ------------------------------------------------------------------------ */
/* Harmonization of a fused group (R15)                                      */
/* ------------------------------------------------------------------------ */

/* Rewrites the logical block scales sf[rows, k/16] of a weight whose row
 * segments [seg_offsets[i], seg_offsets[i+1]) carry global scales seg_scale[i]
 * so that the whole weight uses one global scale, which is returned.  A
 * non-finite or negative scale leaves sf untouched and returns NaN; an all-zero
 * group (shared scale 0) is left as it is. */
float or_harmonize(uint8_t *sf, int64_t rows, int64_t k, const int64_t *seg_offsets, int nseg,
                   const float *seg_scale)
{
    (void)rows;
    float shared = 0.0f;
    for (int i = 0; i < nseg; ++i) {
        if (!isfinite(seg_scale[i]) || seg_scale[i] < 0.0f)
            return NAN;
        if (seg_scale[i] > shared)
            shared = seg_scale[i];
    }
    if (shared == 0.0f)
        return shared;
    const int64_t nblk = k / 16;
    for (int i = 0; i < nseg; ++i) {
        float ratio = seg_scale[i] / shared;                 /* fp32, <= 1 */
        for (int64_t r = seg_offsets[i]; r < seg_offsets[i + 1]; ++r)
            for (int64_t c = 0; c < nblk; ++c) {
                uint8_t b = sf[r * nblk + c];
                if ((b & 0x7Fu) == 0x7Fu)     /* NaN code: NaN times the ratio is NaN, the byte stays */
                    continue;
                float folded = (float)or_e4m3_value(b) * ratio;   /* fp32 product */
                sf[r * nblk + c] = (uint8_t)or_e4m3_encode(folded);
            }
    }
    return shared;
}

/* ------------------------------------------------------------------------ */
/* Bulk encodes for comparisons over whole ranges of fp32 bit patterns      */
/* ------------------------------------------------------------------------ */

/* out[i] = E2M1 code (R7) of the fp32 whose bit pattern is start + i. */
void or_e2m1_encode_patterns(uint64_t start, uint64_t count, uint8_t *out)
{
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < (int64_t)count; ++i) {
        uint32_t u = (uint32_t)(start + (uint64_t)i);
        float v;
        memcpy(&v, &u, sizeof v);
        out[i] = (uint8_t)or_e2m1_encode(v);
    }
}

/* out[i] = E4M3 code (R5) of the fp32 whose bit pattern is pats[i]. */
void or_e4m3_encode_patterns(const uint32_t *pats, int64_t count, uint8_t *out)
{
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < count; ++i) {
        float v;
        memcpy(&v, &pats[i], sizeof v);
        out[i] = (uint8_t)or_e4m3_encode(v);
    }
}

/* out[i] = E4M3 code (R5) of the fp32 whose bit pattern is start + i, for
 * whole ranges of patterns.  The rule is or_e4m3_encode's -- the nearest of
 * the 127 finite non-negative E4M3 values to |v|, a tie to the even code,
 * saturation at 448, the sign bit of v -- with the nearest value found by
 * bisection over a table of those values instead of a scan. */
void or_e4m3_encode_range(uint64_t start, uint64_t count, uint8_t *out)
{
    double tab[127];
    for (uint32_t c = 0; c < 127; ++c)
        tab[c] = or_e4m3_value(c);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < (int64_t)count; ++i) {
        uint32_t u = (uint32_t)(start + (uint64_t)i);
        float v;
        memcpy(&v, &u, sizeof v);
        uint32_t sign = signbit(v) ? 0x80u : 0u;
        double a = fabs((double)v);
        uint32_t code;
        if (!(a <= tab[126])) {
            code = 126;                       /* beyond 448 (or NaN): saturate */
        } else {
            uint32_t lo = 0, hi = 126;        /* invariant: tab[lo] <= a <= tab[hi] */
            if (a == tab[0])
                hi = 0;
            while (hi - lo > 1) {
                uint32_t mid = (lo + hi) / 2;
                if (tab[mid] <= a)
                    lo = mid;
                else
                    hi = mid;
            }
            double dl = a - tab[lo], dh = tab[hi] - a;
            if (dl < dh)
                code = lo;
            else if (dh < dl)
                code = hi;
            else
                code = (lo & 1u) == 0 ? lo : hi;
        }
        out[i] = (uint8_t)(sign | code);
    }
}

