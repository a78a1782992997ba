// gemm_sm100.cuh -- block-scaled FP4 GEMM with the global-scale epilogue (sm_100a).
//
// Computes Y[m, n] = alpha[n] * sum_k (e2m1(Qx[m,k]) * e4m3(SFx[m,k/16])) *
//                                     (e2m1(Qw[n,k]) * e4m3(SFw[n,k/16]))
// with FP32 accumulation in tensor memory and alpha[n] = s_x * s_w[segment(n)],
// the W4A4 GEMM of "Why Gated DeltaNet Survives 4-Bit Quantization" (§2 "NVFP4":
// the GEMM runs on native 4-bit tensor cores) with the per-module global scales
// of a fused GEMM kept apart (§6 "Per-module calibration vs. fused-GEMM scaling").
//
// Structure (one CTA per SM, persistent over 128 x 256 output tiles):
//   warp 0       TMA producer: per 256-deep K stage, one tiled TMA load of the
//                activation codes (128 rows x 128 B, 128-byte swizzle), one of the
//                weight codes (256 rows x 128 B) and bulk copies of the matching
//                512-byte scale atoms, all completing on the stage's mbarrier.
//   warp 1       MMA issuer (one thread): tcgen05.cp of the scale atoms into
//                tensor memory, four tcgen05.mma kind::mxf4nvf4 block16 (K = 64
//                each) into the 128 x 256 FP32 accumulator, tcgen05.commit to
//                release the stage, and a final commit to hand the tile over.
//   warps 2..5   epilogue: tcgen05.ld of the accumulator (each warp its 32-lane
//                quarter), scale by alpha, convert to bf16, store.
// The shared-memory ring has 4 stages of 54 KB.  Every wait is bounded; on a
// timeout the kernel records an error, drains its copies, frees tensor memory
// and returns.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "sm100_ptx.cuh"

namespace nvfp4 {

namespace gemm {

constexpr int BM = 128;                 // tile rows (activations; TMEM lanes)
constexpr int BN = 256;                 // tile columns (weights; MMA N)
constexpr int BK = 256;                 // K elements per stage (128 bytes per row)
constexpr int STAGES = 4;
constexpr int KB = BK / 64;             // MMAs (K = 64) per stage
constexpr int A_BYTES = BM * BK / 2;    // 16 KB
constexpr int B_BYTES = BN * BK / 2;    // 32 KB
constexpr int SFA_BYTES = (BM / 128) * KB * 512;
constexpr int SFB_BYTES = (BN / 128) * KB * 512;
constexpr int THREADS = 192;
constexpr int TMEM_COLS = 512;
constexpr int TMEM_SFA_COL = BN;                 // after the accumulator
constexpr int TMEM_SFB_COL = BN + KB * 4;        // 4 columns per SFA atom
constexpr uint64_t DRAIN_TIMEOUT_NS = 1000000000ull;

constexpr int OFF_A = 0;
constexpr int OFF_B = OFF_A + STAGES * A_BYTES;
constexpr int OFF_SFA = OFF_B + STAGES * B_BYTES;
constexpr int OFF_SFB = OFF_SFA + STAGES * SFA_BYTES;
constexpr int OFF_BAR = OFF_SFB + STAGES * SFB_BYTES;
constexpr int NUM_BARS = 2 * STAGES + 3;         // full, empty, acc_full, acc_empty, final
constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
constexpr int SMEM_BYTES = OFF_MISC + 64;
constexpr int SMEM_ALLOC = SMEM_BYTES + 1024;    // slack for 1024-byte alignment

static_assert(SMEM_ALLOC <= 232448, "shared memory budget");
static_assert(TMEM_SFB_COL + KB * 8 <= TMEM_COLS, "tensor memory budget");

constexpr unsigned FLAG_F32_OUT = 1u;
constexpr unsigned FLAG_COLLAPSED = 2u;

struct Params {
    const uint8_t *sfa;          // activation scales, physical layout
    const uint8_t *sfb;          // weight scales, physical layout
    int m, n, k;
    int tiles_m, tiles_n, k_stages;
    int64_t atoms_k;             // 512-byte scale atoms per 128-row block = K/64
    void *y;
    int64_t ldy;
    const float *s_x;            // [1]
    const float *s_w;            // [nseg]
    int nseg;
    int seg_end[8];              // column end of each segment
    unsigned flags;
    uint64_t timeout_ns;
};

__device__ __forceinline__ float column_alpha(const Params &p, float sx, float swmax, int col)
{
    if (p.flags & FLAG_COLLAPSED)
        return sx * swmax;
    int seg = 0;
#pragma unroll
    for (int s = 0; s < 7; ++s)
        seg += (s + 1 < p.nseg && col >= p.seg_end[s]) ? 1 : 0;
    return sx * p.s_w[seg];
}

// Scale one thread's 32 accumulator columns (row m, columns nc..nc+31) by their
// alpha and store them (bf16, or fp32 with FLAG_F32_OUT); columns >= n are skipped
// in groups of 8 (n % 8 == 0).
__device__ __forceinline__ void store_chunk(const Params &p, const uint32_t (&r)[32], int m, int nc, float sx,
                                            float swmax, bool f32_out)
{
    const float a_lo = column_alpha(p, sx, swmax, nc);
    const float a_hi = column_alpha(p, sx, swmax, min(nc + 31, p.n - 1));
    float v[32];
    if (a_lo == a_hi) {
#pragma unroll
        for (int i = 0; i < 32; ++i)
            v[i] = __uint_as_float(r[i]) * a_lo;
    } else {
#pragma unroll
        for (int i = 0; i < 32; ++i)
            v[i] = __uint_as_float(r[i]) * column_alpha(p, sx, swmax, min(nc + i, p.n - 1));
    }
    if (!f32_out) {
        __nv_bfloat16 *dst = reinterpret_cast<__nv_bfloat16 *>(p.y) + static_cast<int64_t>(m) * p.ldy + nc;
#pragma unroll
        for (int g = 0; g < 4; ++g) {
            if (nc + g * 8 < p.n) {
                uint4 o;
                __nv_bfloat162 h0 = __floats2bfloat162_rn(v[g * 8 + 0], v[g * 8 + 1]);
                __nv_bfloat162 h1 = __floats2bfloat162_rn(v[g * 8 + 2], v[g * 8 + 3]);
                __nv_bfloat162 h2 = __floats2bfloat162_rn(v[g * 8 + 4], v[g * 8 + 5]);
                __nv_bfloat162 h3 = __floats2bfloat162_rn(v[g * 8 + 6], v[g * 8 + 7]);
                o.x = *reinterpret_cast<uint32_t *>(&h0);
                o.y = *reinterpret_cast<uint32_t *>(&h1);
                o.z = *reinterpret_cast<uint32_t *>(&h2);
                o.w = *reinterpret_cast<uint32_t *>(&h3);
                *reinterpret_cast<uint4 *>(dst + g * 8) = o;
            }
        }
    } else {
        float *dst = reinterpret_cast<float *>(p.y) + static_cast<int64_t>(m) * p.ldy + nc;
#pragma unroll
        for (int g = 0; g < 4; ++g) {
            if (nc + g * 8 < p.n) {
                *reinterpret_cast<float4 *>(dst + g * 8) =
                    make_float4(v[g * 8 + 0], v[g * 8 + 1], v[g * 8 + 2], v[g * 8 + 3]);
                *reinterpret_cast<float4 *>(dst + g * 8 + 4) =
                    make_float4(v[g * 8 + 4], v[g * 8 + 5], v[g * 8 + 6], v[g * 8 + 7]);
            }
        }
    }
}

__global__ void __launch_bounds__(THREADS, 1)
    nvfp4_gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                      const Params p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + OFF_BAR);
    uint64_t *full = bars;
    uint64_t *empty = bars + STAGES;
    uint64_t *acc_full = bars + 2 * STAGES;
    uint64_t *acc_empty = acc_full + 1;
    uint64_t *final_bar = acc_full + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + OFF_MISC + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int num_tiles = p.tiles_m * p.tiles_n;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(acc_full, 1);
        mbar_init(acc_empty, 4);
        mbar_init(final_bar, 1);
        *abort_flag = 0;
        fence_barrier_init();
        prefetch_tensormap(&tm_a);
        prefetch_tensormap(&tm_b);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            pdl_wait_prerequisites();            // activation codes come from the preceding kernel
            int stage = 0;
            uint32_t phase = 0;
            uint32_t issued_mask = 0, issued_phase = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
                const int mb = tile / p.tiles_n, nb = tile % p.tiles_n;
                const int nh = min(2, (p.n - nb * BN + 127) / 128);      // 128-row weight-scale blocks present
                for (int ks = 0; ks < p.k_stages; ++ks) {
                    if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, abort_flag, p.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    const int nkb = min(KB, static_cast<int>(p.atoms_k) - ks * KB);
                    const uint32_t bytes = A_BYTES + B_BYTES + nkb * 512 * (1 + nh);
                    mbar_arrive_expect_tx(&full[stage], bytes);
                    tma_load_2d(smem + OFF_A + stage * A_BYTES, &tm_a, ks * (BK / 2), mb * BM, &full[stage]);
                    tma_load_2d(smem + OFF_B + stage * B_BYTES, &tm_b, ks * (BK / 2), nb * BN, &full[stage]);
                    bulk_load(smem + OFF_SFA + stage * SFA_BYTES,
                              p.sfa + (static_cast<int64_t>(mb) * p.atoms_k + ks * KB) * 512, nkb * 512,
                              &full[stage]);
                    for (int h = 0; h < nh; ++h)
                        bulk_load(smem + OFF_SFB + stage * SFB_BYTES + h * (KB * 512),
                                  p.sfb + (static_cast<int64_t>(nb * 2 + h) * p.atoms_k + ks * KB) * 512,
                                  nkb * 512, &full[stage]);
                    issued_mask |= 1u << stage;
                    issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            // Every copy this thread issued must have landed before the CTA exits.
            for (int s = 0; s < STAGES; ++s)
                if (issued_mask & (1u << s)) {
                    volatile int no_abort = 0;
                    if (!mbar_wait_bounded(&full[s], (issued_phase >> s) & 1u, &no_abort, DRAIN_TIMEOUT_NS))
                        *abort_flag = 1;
                }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc = make_idesc_nvfp4(BM, BN);
            const uint32_t acc = tmem_base;
            const uint32_t sfa_t = tmem_base + TMEM_SFA_COL;
            const uint32_t sfb_t = tmem_base + TMEM_SFB_COL;
            const uint32_t a0 = smem_u32(smem + OFF_A), b0 = smem_u32(smem + OFF_B);
            const uint32_t sfa0 = smem_u32(smem + OFF_SFA), sfb0 = smem_u32(smem + OFF_SFB);
            int stage = 0;
            uint32_t phase = 0, acc_phase = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
                if (!mbar_wait_bounded(acc_empty, acc_phase ^ 1u, abort_flag, p.timeout_ns))
                    break;
                tc_fence_after();
                for (int ks = 0; ks < p.k_stages; ++ks) {
                    if (!mbar_wait_bounded(&full[stage], phase, abort_flag, p.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const int nkb = min(KB, static_cast<int>(p.atoms_k) - ks * KB);
                    for (int kb = 0; kb < nkb; ++kb) {
                        tc_cp_32x128b_warpx4(sfa_t + kb * 4,
                                             make_smem_desc(sfa0 + stage * SFA_BYTES + kb * 512, 0, 128, 0));
                        tc_cp_32x128b_warpx4(sfb_t + kb * 8,
                                             make_smem_desc(sfb0 + stage * SFB_BYTES + kb * 512, 0, 128, 0));
                        tc_cp_32x128b_warpx4(sfb_t + kb * 8 + 4,
                                             make_smem_desc(sfb0 + stage * SFB_BYTES + KB * 512 + kb * 512, 0,
                                                            128, 0));
                    }
                    for (int kb = 0; kb < nkb; ++kb) {
                        const uint64_t ad = make_smem_desc(a0 + stage * A_BYTES + kb * 32, 16, 1024, 2);
                        const uint64_t bd = make_smem_desc(b0 + stage * B_BYTES + kb * 32, 16, 1024, 2);
                        tc_mma_nvfp4(acc, ad, bd, idesc, sfa_t + kb * 4, sfb_t + kb * 8, (ks | kb) != 0);
                    }
                    tc_commit(&empty[stage]);
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok)
                    break;
                tc_commit(acc_full);
                acc_phase ^= 1u;
            }
            // Wait for every tensor-core operation issued above before TMEM is freed.
            tc_commit(final_bar);
            volatile int no_abort = 0;
            if (!mbar_wait_bounded(final_bar, 0, &no_abort, DRAIN_TIMEOUT_NS))
                *abort_flag = 1;
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int quarter = warp & 3;                    // TMEM lanes this warp may read
        const int row_in_tile = quarter * 32 + lane;
        pdl_wait_prerequisites();
        const float sx = *p.s_x;
        float swmax = p.s_w[0];
        for (int s = 1; s < p.nseg; ++s)
            swmax = fmaxf(swmax, p.s_w[s]);
        const bool f32_out = (p.flags & FLAG_F32_OUT) != 0;
        uint32_t acc_phase = 0;
        for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
            const int mb = tile / p.tiles_n, nb = tile % p.tiles_n;
            if (!mbar_wait_bounded(acc_full, acc_phase, abort_flag, p.timeout_ns))
                break;
            tc_fence_after();
            const int m = mb * BM + row_in_tile;
            const int n0 = nb * BN;
#pragma unroll 1
            for (int chunk = 0; chunk < BN / 32; ++chunk) {
                uint32_t r[32];
                __syncwarp();                                // tcgen05.ld needs the whole warp converged
                tmem_ld_32x32b_x32(tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + chunk * 32, r);
                tmem_ld_wait();
                const int nc = n0 + chunk * 32;
                if (m < p.m && nc < p.n)
                    store_chunk(p, r, m, nc, sx, swmax, f32_out);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(acc_empty);
            acc_phase ^= 1u;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 0 && *abort_flag)
        atomicCAS(&g_device_error, 0u, 6u /* NVFP4_ERR_TIMEOUT */);
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem_base, TMEM_COLS);
    }
}

}  // namespace gemm
}  // namespace nvfp4
