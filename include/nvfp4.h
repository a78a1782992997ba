/*
 * nvfp4.h -- C ABI of the NVFP4 W4A4 linear layer for NVIDIA B200 (sm_100a).
 *
 * The layer is Y = X . W^T with both operands in NVFP4, as described in
 * "Why Gated DeltaNet Survives 4-Bit Quantization: NVFP4 W4A4 for the Recurrent
 * Half of a Hybrid 27B LLM", §2 "NVFP4": values are E2M1 (4-bit), each run of 16
 * consecutive elements along K shares one E4M3 block scale (blockmax/6), and a
 * tensor carries one FP32 global scale.  The FP32 global scale s stored and
 * consumed here is the dequantization multiplier, s = absmax / (6 * 448)
 * (Gemma-4-31B-IT-NVFP4-FP8attn-text model card, §Verification:
 * max(block scale) x s x 6 = absmax).
 *
 * Three steps run on the GPU:
 *   1. activation quantization (amax -> s_x, 16-element E4M3 block scales,
 *      E2M1 codes packed two per byte);
 *   2. block-scaled FP4 GEMM with FP32 accumulation on the tcgen05 tensor cores;
 *   3. an epilogue that multiplies each output column by s_x * s_w[segment]
 *      and writes bf16.  A fused GEMM over several modules concatenated along N
 *      keeps one weight global scale per module (segment); "Why Gated DeltaNet
 *      Survives 4-Bit Quantization", §6 "Per-module calibration vs. fused-GEMM
 *      scaling", shows what goes wrong when those are collapsed to one.
 *
 * Conventions for every entry point
 *   - All pointers marked "device" are CUDA device (or managed) pointers; the
 *     caller allocates and owns every buffer, including the workspace.  The
 *     library allocates no device memory; its only device memory of its own is
 *     the static scratch array of nvfp4_linear_fused_noalloc (see there).
 *   - Work is enqueued asynchronously on `stream` (a cudaStream_t; NULL is the
 *     legacy default stream).  No entry point synchronizes, except
 *     nvfp4_get_device_error().
 *   - Arguments are validated on the host before anything is enqueued; a call
 *     that returns an error enqueued nothing.  CUDA launch failures map to
 *     NVFP4_ERR_CUDA (cudaGetLastError() is consumed).
 *   - Conditions only the GPU can see (non-finite amax, a pipeline wait that
 *     ran out) are recorded in a per-device error word, read and cleared by
 *     nvfp4_get_device_error().
 *
 * Layouts
 *   X, W    bf16, row-major, [rows, K] with a row stride (ld*) in elements;
 *           ld* * 2 bytes and the base address must be multiples of 16.
 *   Q       packed E2M1 codes, [rows, K/2] bytes, row stride K/2; byte j of a
 *           row holds the code of element 2j in bits 0..3 and of element 2j+1
 *           in bits 4..7.  Code bits: sign (bit 3), exponent (bits 2..1, bias 1),
 *           mantissa (bit 0).
 *   SF      E4M3 block scales in the tensor-core layout: rows padded to 128,
 *           scale columns (K/16) padded to 4; 512-byte atoms of 128 rows x 4
 *           scale columns, atoms ordered K-fastest ((r/128)*ceil(K/64) + c/4);
 *           inside an atom the byte of (r, c) is at (r%32)*16 + ((r%128)/32)*4
 *           + c%4.  Pad bytes are written as 0.  Size: nvfp4_sf_bytes().
 *   Y       bf16 (or fp32 with NVFP4_FLAG_F32_OUT), row-major [M, N], row
 *           stride ldy elements (16-byte aligned rows).
 *
 * Shape limits: K % 64 == 0, N % 8 == 0, M >= 0 (M == 0 is a no-op),
 * 1 <= nseg <= NVFP4_MAX_SEGMENTS, segment offsets strictly increasing from 0
 * to the segmented extent (N, or the row count), interior offsets multiples of 8.
 *
 * Environment: NVFP4_NO_CLUSTER_QUANTIZER=1 (read once per device, at the first
 * call on it) makes decode-sized activations take the amax pass + per-unit
 * encoder instead of the one-launch 16-CTA cluster quantizer, as happens anyway
 * on a device or partition that cannot hold such a cluster.  Results are the
 * same bytes either way.
 */
#ifndef NVFP4_H_
#define NVFP4_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *nvfp4_stream_t; /* same type as cudaStream_t */

#define NVFP4_MAX_SEGMENTS 8

typedef enum {
    NVFP4_OK = 0,
    NVFP4_ERR_INVALID_ARG = 1,        /* null pointer, negative size, bad segment table, unknown flag */
    NVFP4_ERR_UNSUPPORTED_SHAPE = 2,  /* K % 64, N % 8, too many segments, size overflow */
    NVFP4_ERR_MISALIGNED = 3,         /* pointer or row stride not 16-byte aligned */
    NVFP4_ERR_NONFINITE = 4,          /* device saw a non-finite amax or static scale */
    NVFP4_ERR_CUDA = 5,               /* a CUDA runtime/driver call failed */
    NVFP4_ERR_TIMEOUT = 6,            /* a bounded pipeline wait inside a kernel ran out */
    NVFP4_ERR_WORKSPACE = 7,          /* workspace null or smaller than nvfp4_workspace_bytes() */
    NVFP4_ERR_UNSUPPORTED_DEVICE = 8, /* current device is not sm_100 */
    NVFP4_ERR_SCRATCH_LIMIT = 9       /* problem too large for nvfp4_linear_fused_noalloc's static scratch */
} nvfp4_status;

/* Flags for nvfp4_gemm / nvfp4_linear / nvfp4_linear_fused. */
#define NVFP4_FLAG_F32_OUT 0x1u              /* write fp32 instead of bf16 (numerics checks) */
#define NVFP4_FLAG_COLLAPSED_MAX_SCALE 0x2u  /* negative control: every column uses s_x * max(s_w),
                                                the mismatch of "Why Gated DeltaNet Survives
                                                4-Bit Quantization", §6; never for serving */
#define NVFP4_FLAG_STATIC_WEIGHTS 0x4u       /* nvfp4_gemm: the caller guarantees that no work still
                                                pending on the device writes the packed weight codes or
                                                block scales (e.g. weights packed once at load time), so
                                                the GEMM may request its first weight stages before it
                                                waits for the preceding kernel in the stream to finish,
                                                overlapping that kernel's end (activations, global
                                                scales and the output are still touched only after the
                                                wait).  Results are unchanged.  nvfp4_linear and
                                                nvfp4_linear_fused accept it and always do this behind
                                                their own quantizer.  A deployment option; no paper
                                                counterpart. */
#define NVFP4_FLAG_TEST_STALL 0x100u         /* testing only: the GEMM's producer withholds its second
                                                K stage, so a bounded pipeline wait runs out; the call
                                                writes no valid output and records NVFP4_ERR_TIMEOUT in
                                                the device error word (pair it with a short
                                                nvfp4_set_wait_timeout_ns).  No paper counterpart. */
#define NVFP4_FLAG_TEST_STALL_LATE 0x200u    /* testing only, as NVFP4_FLAG_TEST_STALL but the stage
                                                withheld is the last K stage of each CTA pair's second
                                                output tile (of each CTA's tile in the decode kernel),
                                                after earlier tiles completed.  No paper counterpart. */

/* Human-readable name of a status code (static string, never NULL). */
const char *nvfp4_status_string(nvfp4_status st);

/* Bytes of a physical SF buffer for `rows` rows of K elements:
 * ceil(rows/128)*128 * ceil(K/16/4)*4.  Returns 0 for invalid input. */
size_t nvfp4_sf_bytes(int64_t rows, int64_t k);

/* Bytes of device workspace that nvfp4_quantize_act / nvfp4_linear /
 * nvfp4_linear_fused / nvfp4_pack_weight need for an [m, k] activation
 * (or weight) operand.  The workspace needs no initialisation and its contents
 * after a call are unspecified; calls sharing one workspace must be ordered on
 * one stream. */
size_t nvfp4_workspace_bytes(int64_t m, int64_t n, int64_t k);

/* Activation quantization (step 1).
 * x           device bf16 [m, k], row stride ldx.
 * gscale_in   device float: static (calibrated) global scale s_x, or NULL for
 *             the dynamic per-tensor scale s_x = amax(|x|) / 2688 computed on the GPU.
 * gscale_out  device float, receives the s_x used (may alias gscale_in).
 * q           device [m, k/2] bytes (packed codes).
 * sf          device nvfp4_sf_bytes(m, k) bytes (swizzled block scales, pads zeroed).
 * workspace   device, >= nvfp4_workspace_bytes(m, 0, k) bytes. */
nvfp4_status nvfp4_quantize_act(const void *x, int64_t m, int64_t k, int64_t ldx,
                                const float *gscale_in, float *gscale_out,
                                uint8_t *q, uint8_t *sf,
                                void *workspace, size_t ws_bytes, nvfp4_stream_t stream);

/* Offline weight packing: the same codec applied to W [n, k] (row stride ldw),
 * one global scale per segment (module) of rows.
 * seg_offsets host int64[nseg+1] (0 = seg_offsets[0] < ... < seg_offsets[nseg] = n),
 *             or NULL with nseg == 1 for a single module.
 * gscale_in   device float[nseg] static scales, or NULL for amax/2688 per segment.
 * gscale_out  device float[nseg], receives the scales used.
 * q, sf       device outputs as for nvfp4_quantize_act, for n rows.
 * workspace   device, >= nvfp4_workspace_bytes(n, 0, k) bytes. */
nvfp4_status nvfp4_pack_weight(const void *w, int64_t n, int64_t k, int64_t ldw,
                               const int64_t *seg_offsets, int nseg,
                               const float *gscale_in, float *gscale_out,
                               uint8_t *q, uint8_t *sf,
                               void *workspace, size_t ws_bytes, nvfp4_stream_t stream);

/* Block-scaled FP4 GEMM + epilogue on already-quantized operands (steps 2, 3).
 * qx, sfx, s_x  device activation codes [m, k/2], scales, global scale (1 float).
 * qw, sfw       device weight codes [n, k/2] and scales.
 * seg_offsets   host int64[nseg+1] column segments (NULL with nseg == 1).
 * seg_gscales   device float[nseg] weight global scale per segment.
 * y             device [m, n] output (bf16, or fp32 with NVFP4_FLAG_F32_OUT), row stride ldy.
 * flags         NVFP4_FLAG_* bits.
 * Needs no workspace.
 * Errors (host-checked, nothing enqueued): NVFP4_ERR_INVALID_ARG for m < 0,
 * n <= 0, k <= 0, an unknown flag bit, a NULL operand (activation operands and
 * y may be NULL only when m == 0), ldy < n, or a malformed segment table;
 * NVFP4_ERR_UNSUPPORTED_SHAPE for k % 64 != 0, n % 8 != 0, an interior segment
 * offset not a multiple of 8, nseg > NVFP4_MAX_SEGMENTS, or sizes beyond the
 * 32-bit tile indexing; NVFP4_ERR_MISALIGNED for an operand or y not 16-byte
 * aligned or a y row stride not a multiple of 16 bytes.  A wait that runs out
 * on the GPU shows up later as NVFP4_ERR_TIMEOUT from nvfp4_get_device_error. */
nvfp4_status nvfp4_gemm(const uint8_t *qx, const uint8_t *sfx, const float *s_x, int64_t m,
                        const uint8_t *qw, const uint8_t *sfw, int64_t n, int64_t k,
                        const int64_t *seg_offsets, const float *seg_gscales, int nseg,
                        void *y, int64_t ldy, unsigned flags, nvfp4_stream_t stream);

/* The whole layer for one module: quantize x, GEMM against the packed weight,
 * epilogue with s_x * s_w.  act_gscale: device static s_x or NULL (dynamic).
 * workspace >= nvfp4_workspace_bytes(m, n, k). */
nvfp4_status nvfp4_linear(const void *x, int64_t m, int64_t k, int64_t ldx, const float *act_gscale,
                          const uint8_t *qw, const uint8_t *sfw, const float *w_gscale, int64_t n,
                          void *y, int64_t ldy, unsigned flags,
                          void *workspace, size_t ws_bytes, nvfp4_stream_t stream);

/* The whole layer for modules fused along N (e.g. q/k/v/gate projections
 * concatenated into one GEMM), each keeping its own weight global scale:
 * column j of segment i is scaled by s_x * seg_gscales[i] ("Why Gated DeltaNet
 * Survives 4-Bit Quantization", §6 "Per-module calibration vs. fused-GEMM scaling").
 * seg_offsets host int64[nseg+1]; seg_gscales device float[nseg].
 * Errors: those of nvfp4_gemm for the GEMM's arguments and of
 * nvfp4_quantize_act for x, plus NVFP4_ERR_WORKSPACE for a NULL, unaligned or
 * too small workspace.  A non-finite activation amax or act_gscale is reported
 * by nvfp4_get_device_error as NVFP4_ERR_NONFINITE (the codes are then those of
 * scale 0). */
nvfp4_status nvfp4_linear_fused(const void *x, int64_t m, int64_t k, int64_t ldx, const float *act_gscale,
                                const uint8_t *qw, const uint8_t *sfw, int64_t n,
                                const int64_t *seg_offsets, const float *seg_gscales, int nseg,
                                void *y, int64_t ldy, unsigned flags,
                                void *workspace, size_t ws_bytes, nvfp4_stream_t stream);

/* Bytes of the static device scratch behind nvfp4_linear_fused_noalloc.  Every
 * device that loads this library holds this much device memory until the
 * process exits. */
#define NVFP4_NOALLOC_SCRATCH_BYTES (8u << 20)

/* The fused layer without a workspace argument, for callers that cannot
 * allocate device memory: code hosted inside a runtime that owns all device
 * memory and gives its plugins no allocator, or latency-critical paths where a
 * cudaMalloc (which may synchronize the device) is not acceptable.  The paper
 * has no counterpart to this entry point; it is a deployment convenience.
 *
 * Arguments, layouts, results and errors are those of nvfp4_linear_fused.  The
 * activation codes, scales, global scale and amax partials go to a static
 * device array of NVFP4_NOALLOC_SCRATCH_BYTES inside the library instead of a
 * caller workspace; a problem whose nvfp4_workspace_bytes(m, n, k) exceeds that
 * size is rejected with NVFP4_ERR_SCRATCH_LIMIT before anything is enqueued
 * (at K = 5120 that allows up to 2895 tokens; 847 at K = 17408).  Malformed
 * arguments get the status nvfp4_linear_fused would give them.
 *
 * The first call on a device looks up the array's device address (a one-time
 * set-up with that device current, made again if the device's context was
 * replaced, e.g. by cudaDeviceReset); make that first call before any stream
 * capture.  The call allocates nothing.  All calls share the one array and it
 * keeps the last call's contents; nothing in it needs to start at zero.  Calls
 * whose work overlaps on the GPU (different streams without ordering between
 * them) race on the array: order them on one stream. */
nvfp4_status nvfp4_linear_fused_noalloc(const void *x, int64_t m, int64_t k, int64_t ldx, const float *act_gscale,
                                        const uint8_t *qw, const uint8_t *sfw, int64_t n,
                                        const int64_t *seg_offsets, const float *seg_gscales, int nseg,
                                        void *y, int64_t ldy, unsigned flags, nvfp4_stream_t stream);

/* Expansion of packed NVFP4 rows to bf16 (the "expand to BF16" step of the
 * Gemma-4-31B-IT-NVFP4-FP8attn-text model card, §Limitations; it is the
 * inverse of the encoding of "Why Gated DeltaNet Survives 4-Bit Quantization",
 * §2 "NVFP4").  Element (r, j) is
 *     y[r, j] = bf16( value(code[r, j]) * value(sf[r, j/16]) * s[segment(r)] )
 * where the product is exact and is rounded once to the nearest bf16, ties to
 * the even significand.
 * q            device [rows, k/2] packed codes (16-byte aligned).
 * sf           device block scales in the tensor-core layout (nvfp4_sf_bytes(rows, k)).
 * seg_offsets  host int64[nseg+1] row segments (NULL with nseg == 1).
 * seg_gscales  device float[nseg] global scale of each segment; they must be
 *              finite and non-negative, as every global scale of the format is
 *              (any other value gives unspecified values).
 * y            device bf16 [rows, k] with row stride ldy elements (16-byte aligned rows).
 * K % 64 == 0; any row count (rows == 0 is a no-op).  Needs no workspace. */
nvfp4_status nvfp4_dequantize(const uint8_t *q, const uint8_t *sf, int64_t rows, int64_t k,
                              const int64_t *seg_offsets, const float *seg_gscales, int nseg,
                              void *y, int64_t ldy, nvfp4_stream_t stream);

/* Checkpoint import of block scales.  NVFP4 checkpoints store, per linear
 * layer, the packed codes (uint8 [n, k/2], the same nibble order as Q above,
 * so they are used as they are), the E4M3 block scales as a plain row-major
 * matrix [n, k/16] (one byte per 16-element block) and the FP32 global scale,
 * which is the dequantization multiplier s of this library ("Why Gated
 * DeltaNet Survives 4-Bit Quantization", §3 "Checkpoints"; model card
 * §Verification: max(block scale) x global x 6 = absmax).  This call
 * rewrites the row-major block-scale matrix into the tensor-core layout.
 * sf_linear  device [n, k/16] bytes with row stride ld_sf bytes (ld_sf >= k/16,
 *            ld_sf % 4 == 0, base 4-byte aligned).
 * sf_out     device nvfp4_sf_bytes(n, k) bytes, 16-byte aligned, not
 *            overlapping sf_linear; pad bytes are written as 0.
 * n == 0 is a no-op.  Needs no workspace. */
nvfp4_status nvfp4_import_weight_scales(const uint8_t *sf_linear, int64_t n, int64_t k, int64_t ld_sf,
                                        uint8_t *sf_out, nvfp4_stream_t stream);

/* Harmonization of a fused group: the checkpoint-side repair of "Why Gated
 * DeltaNet Survives 4-Bit Quantization", §6 "Per-module calibration vs.
 * fused-GEMM scaling".  The modules concatenated along N keep their packed
 * codes; the group gets one global scale s_shared = max_i seg_gscales[i], and
 * every block scale of module i becomes
 *     E4M3_rne_satfinite( value(sb) * (seg_gscales[i] / s_shared) )
 * with the ratio and the product in fp32.  Every ratio is <= 1, so no folded
 * scale passes 448; the re-rounding error is at most half an E4M3 ulp (2^-4
 * relative in the normal range; the paper reports <= 6.2%).  Afterwards the
 * weight can be served by a single-scale GEMM (nvfp4_linear with *w_gscale =
 * s_shared).
 * sf_in, sf_out   device block scales in the tensor-core layout
 *                 (nvfp4_sf_bytes(n, k)), 16-byte aligned; sf_out may equal
 *                 sf_in (in place) but must not partially overlap it.
 * seg_offsets     host int64[nseg+1] (NULL with nseg == 1).
 * seg_gscales     device float[nseg].
 * shared_gscale_out device float, receives s_shared.
 * A negative or non-finite module scale leaves the scales unchanged, writes
 * NaN to *shared_gscale_out and records NVFP4_ERR_NONFINITE in the device error
 * word.  A NaN block-scale byte (0x7F or 0xFF, which only a corrupt checkpoint
 * holds) is kept as it is (NaN times the ratio is NaN) while the other bytes
 * fold as usual, and the call records NVFP4_ERR_NONFINITE.  An all-zero group
 * is left unchanged (s_shared = 0).  Pad rows are copied unchanged.  Needs no
 * workspace. */
nvfp4_status nvfp4_harmonize_scales(const uint8_t *sf_in, uint8_t *sf_out, int64_t n, int64_t k,
                                    const int64_t *seg_offsets, const float *seg_gscales, int nseg,
                                    float *shared_gscale_out, nvfp4_stream_t stream);

/* Synchronizes `stream`, then returns and clears the current device's error
 * word: NVFP4_ERR_NONFINITE, NVFP4_ERR_TIMEOUT, or NVFP4_OK. */
nvfp4_status nvfp4_get_device_error(nvfp4_stream_t stream);

/* Upper bound, in nanoseconds, of every pipeline wait inside the GEMM kernel
 * on the current process (default 2e9).  A wait that runs out makes the kernel
 * record NVFP4_ERR_TIMEOUT, drain its in-flight copies, release its tensor
 * memory and return.  Values below 1000 are raised to 1000. */
void nvfp4_set_wait_timeout_ns(uint64_t ns);

/* Number of kernel launches this library has enqueued in this process so far
 * (every entry point, every device).  Instrumentation for callers that count
 * device work, e.g. the launches recorded into a CUDA graph; the paper has no
 * counterpart. */
uint64_t nvfp4_launch_count(void);

/* Measurement helper, not a step of the layer: the dense block-scaled FP4
 * tensor-core rate of this device, the denominator for the GEMM's "fraction of
 * peak" (the paper's W4A4 GEMM runs on native 4-bit tensor cores, "Why Gated
 * DeltaNet Survives 4-Bit Quantization", §2 "NVFP4"; it quotes no rate).
 * Enqueues on `stream` one launch in which each of `pairs` CTA pairs (one CTA
 * per SM; at most half the SM count) issues `iters` x 4 of the GEMM's own
 * instruction, tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.block16 with
 * M = 256, N = 256, K = 64, into one accumulator from operands and scales
 * resident in shared memory -- no global-memory traffic.  With
 * with_scale_copies != 0 every four MMAs are preceded by the GEMM's three
 * per-stage scale-factor copies into tensor memory.  *flops receives the
 * launch's MMA flops (2 * 256 * 256 * 64 * 4 * iters * pairs); time the launch
 * with CUDA events on `stream`.  Keep one launch under a few seconds: its final
 * wait is bounded at 10 s and then records NVFP4_ERR_TIMEOUT.  Errors:
 * NVFP4_ERR_INVALID_ARG (pairs < 1, iters < 1, flops NULL),
 * NVFP4_ERR_UNSUPPORTED_SHAPE (more pairs than SMs / 2). */
nvfp4_status nvfp4_mma_peak_probe(int pairs, int64_t iters, int with_scale_copies, double *flops,
                                  nvfp4_stream_t stream);

/* Library version string. */
const char *nvfp4_version(void);

#ifdef __cplusplus
}
#endif

#endif /* NVFP4_H_ */
