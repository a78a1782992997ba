// gemm_decode.cuh -- block-scaled FP4 GEMM for few tokens (M <= 128), sm_100a.
//
// Same product and epilogue as gemm_pair.cuh ("Why Gated DeltaNet Survives 4-Bit
// Quantization", §2 "NVFP4"; per-module global scales of §6), organised for the
// decode regime, which that paper calls weight-bandwidth-bound (§4) and where it
// attributes the remaining loss to small-batch activation quantization (§9):
//
//   * Operands are swapped: the weight tile (128 rows of N) is the MMA's A operand,
//     so it fills the 128 tensor-memory lanes, and the tokens are the MMA's N
//     (T = 8, 16, 32, 64 or 128).  No tile carries zero padding of the token dimension
//     beyond T, and a stage is ~22-28 KB instead of 54 KB.
//   * One CTA owns one 128-row weight tile over the whole K; two CTAs fit on an SM,
//     so N/128 tiles (272 for N = 34816) are all resident at once and each SM keeps
//     2 x (STAGES-1) weight stages in flight.
//   * The kernel is launched with programmatic stream serialization: its set-up
//     (barriers, tensor memory, descriptor prefetch) overlaps the end of the
//     preceding kernel, and no global memory is touched before griddepcontrol.wait
//     -- except behind this library's activation quantizer, where the producer
//     streams the first STAGES weight stages before the wait, i.e. while the
//     quantizer is still running.  Once it has issued its last load it lets the
//     next kernel in the stream be scheduled.
//
// Roles: warp 0 producer (TMA + bulk copies), warp 1 MMA issuer (one elected lane),
// warps 2..5 epilogue (tcgen05.ld of the 128 x T accumulator, x alpha(n), the tile
// staged as [token][128 columns] in the idle stage buffers (weights and tokens), then 16-byte stores
// along each token's row of Y).
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "sm100_ptx.cuh"

namespace nvfp4 {
namespace decode {

constexpr int BW = 128;                 // weight rows per tile (MMA M, TMEM lanes)
constexpr int BK = 256;                 // K elements per stage (128 bytes per row)
constexpr int KB = BK / 64;             // MMAs per stage
constexpr int A_BYTES = BW * BK / 2;    // 16 KB of weight codes
constexpr int SF_BYTES = KB * 512;      // one 128-row scale atom per K=64 block
constexpr int THREADS = 192;
constexpr uint64_t DRAIN_TIMEOUT_NS = 1000000000ull;
constexpr int SMEM_LIMIT = 113 * 1024;  // two CTAs per SM

constexpr unsigned FLAG_F32_OUT = 1u;
constexpr unsigned FLAG_COLLAPSED = 2u;

// Ring depth: as many stages as fit, but at most four.  Measured over decode
// calls at K = 5120, N = 34816 back to back: with 8 tokens per tile five stages
// fit, and the four-stage ring was 0.3-0.7 us per call faster (1, 8 tokens);
// three stages were slower again (also at 32 tokens, where four is the most
// that fits).
constexpr int MAX_STAGES = 4;

template <int T>
struct Cfg {
    static constexpr int B_BYTES = T * BK / 2;                              // token codes per stage
    static constexpr int STAGE = A_BYTES + B_BYTES + 2 * SF_BYTES;
    static constexpr int FIT = (SMEM_LIMIT - 1024 - 256) / STAGE;
    static constexpr int STAGES = FIT < MAX_STAGES ? FIT : MAX_STAGES;
    static constexpr int OFF_A = 0;
    static constexpr int OFF_B = OFF_A + STAGES * A_BYTES;
    static constexpr int OFF_SFA = OFF_B + STAGES * B_BYTES;
    static constexpr int OFF_SFB = OFF_SFA + STAGES * SF_BYTES;
    static constexpr int OFF_BAR = OFF_SFB + STAGES * SF_BYTES;
    static constexpr int OFF_MISC = OFF_BAR + (2 * STAGES + 2) * 8;
    static constexpr int SMEM_ALLOC = OFF_MISC + 64 + 1024;
    static constexpr int TMEM_SFA = T;                 // columns after the accumulator
    static constexpr int TMEM_SFB = T + KB * 4;
    static constexpr int TMEM_COLS = (T + KB * 8 <= 32)    ? 32
                                     : (T + KB * 8 <= 64)  ? 64
                                     : (T + KB * 8 <= 128) ? 128
                                                           : 256;   // two CTAs per SM: at most 256 each
    static_assert(STAGES >= 3, "pipeline depth");
    static_assert(SMEM_ALLOC <= SMEM_LIMIT, "two CTAs per SM");
    static_assert(B_BYTES % 1024 == 0, "swizzle atoms stay 1024-byte aligned");
    static_assert(OFF_SFA >= T * BW * 4, "the epilogue stages a fp32 tile in the operand buffers");
    static_assert(TMEM_COLS <= 256, "two CTAs per SM share the 512 tensor-memory columns");
};

struct Params {
    const uint8_t *sfw;          // weight scales (A operand)
    const uint8_t *sfx;          // activation scales (B operand), one 128-row block
    int m, n, k;
    int64_t atoms_k;             // K/64
    int k_stages;
    void *y;
    int64_t ldy;
    const float *s_x;
    const float *s_w;
    int nseg;
    int seg_end[8];
    unsigned flags;
    uint64_t timeout_ns;
    int stall_stage;             // testing: K stage whose loads are withheld (-1: none)
    int early_weights;           // 1: the first weight stages are requested before griddepcontrol.wait
                                 //    (the preceding kernel is this library's quantizer, which writes
                                 //    no weights); 0: no global access before the wait
};

template <int T>
__global__ void __launch_bounds__(THREADS, 2)
    nvfp4_gemm_decode_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_x,
                             const Params p)
{
    using C = Cfg<T>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR);
    uint64_t *empty = full + C::STAGES;
    uint64_t *acc_full = full + 2 * C::STAGES;
    uint64_t *final_bar = acc_full + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int w0 = blockIdx.x * BW;              // first weight row (output column) of the tile

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(acc_full, 1);
        mbar_init(final_bar, 1);
        *abort_flag = 0;
        fence_barrier_init();
        prefetch_tensormap(&tm_w);
        prefetch_tensormap(&tm_x);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        // The whole warp walks the schedule (operands stay warp-uniform); one
        // elected lane issues the copies.
        const int pre = min(C::STAGES, p.k_stages);
        if (!p.early_weights)
            pdl_wait_prerequisites();            // the predecessor may write any input
        // Weight stages first: behind the quantizer they do not depend on the preceding kernel.
        for (int ks = 0; ks < pre; ++ks) {
            const int nkb = min(KB, static_cast<int>(p.atoms_k) - ks * KB);
            const uint8_t *sfw_src = p.sfw + (static_cast<int64_t>(blockIdx.x) * p.atoms_k + ks * KB) * 512;
            // Testing hook: withholding one stage (no arrival, no copies) makes the
            // MMA issuer's bounded wait on it run out.
            if (ks != p.stall_stage && elect_one()) {
                mbar_arrive_expect_tx(&full[ks], A_BYTES + C::B_BYTES + 2 * nkb * 512);
                tma_load_2d(smem + C::OFF_A + ks * A_BYTES, &tm_w, ks * (BK / 2), w0, &full[ks]);
                bulk_load(smem + C::OFF_SFA + ks * SF_BYTES, sfw_src, nkb * 512, &full[ks]);
            }
            __syncwarp();
        }
        pdl_wait_prerequisites();                // activation codes/scales are now written
        for (int ks = 0; ks < pre; ++ks) {
            const int nkb = min(KB, static_cast<int>(p.atoms_k) - ks * KB);
            if (ks != p.stall_stage && elect_one()) {
                tma_load_2d(smem + C::OFF_B + ks * C::B_BYTES, &tm_x, ks * (BK / 2), 0, &full[ks]);
                bulk_load(smem + C::OFF_SFB + ks * SF_BYTES, p.sfx + static_cast<int64_t>(ks * KB) * 512, nkb * 512,
                          &full[ks]);
            }
            __syncwarp();
        }
        int stage = pre % C::STAGES;
        uint32_t phase = (pre == C::STAGES) ? 1u : 0u;
        int issued = pre;
        for (int ks = pre; ks < p.k_stages; ++ks) {
            if (!__all_sync(0xFFFFFFFFu, mbar_wait_bounded(&empty[stage], phase ^ 1u, abort_flag, p.timeout_ns)))
                break;
            const int nkb = min(KB, static_cast<int>(p.atoms_k) - ks * KB);
            const uint8_t *sfw_src = p.sfw + (static_cast<int64_t>(blockIdx.x) * p.atoms_k + ks * KB) * 512;
            if (ks != p.stall_stage && elect_one()) {
                mbar_arrive_expect_tx(&full[stage], A_BYTES + C::B_BYTES + 2 * nkb * 512);
                tma_load_2d(smem + C::OFF_A + stage * A_BYTES, &tm_w, ks * (BK / 2), w0, &full[stage]);
                bulk_load(smem + C::OFF_SFA + stage * SF_BYTES, sfw_src, nkb * 512, &full[stage]);
                tma_load_2d(smem + C::OFF_B + stage * C::B_BYTES, &tm_x, ks * (BK / 2), 0, &full[stage]);
                bulk_load(smem + C::OFF_SFB + stage * SF_BYTES, p.sfx + static_cast<int64_t>(ks * KB) * 512,
                          nkb * 512, &full[stage]);
            }
            __syncwarp();
            issued = ks + 1;
            if (++stage == C::STAGES) {
                stage = 0;
                phase ^= 1u;
            }
        }
        // Nothing is left to issue: let the next kernel in the stream be scheduled
        // into the slots this grid frees (it waits for this grid's completion
        // before it reads anything this grid writes).
        pdl_launch_dependents();
        // Every stage issued must have landed before the CTA exits: the last
        // min(STAGES, issued) issues are the only ones possibly in flight.
        for (int j = 0; j < min(C::STAGES, issued); ++j) {
            const int ks = issued - 1 - j;
            if (ks == p.stall_stage)
                continue;                        // withheld: nothing in flight
            const int s = ks % C::STAGES;
            const uint32_t ph = static_cast<uint32_t>((ks / C::STAGES) & 1);
            volatile int no_abort = 0;
            if (!__all_sync(0xFFFFFFFFu, mbar_wait_bounded(&full[s], ph, &no_abort, DRAIN_TIMEOUT_NS)))
                *abort_flag = 1;
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        // Warp-wide loop; the elected lane (lane 0 of the converged warp) issues
        // every copy, MMA and commit, so its commits cover all its MMAs.
        const uint32_t idesc = make_idesc_nvfp4(BW, T);
        const uint32_t sfa_t = tmem_base + C::TMEM_SFA;
        const uint32_t sfb_t = tmem_base + C::TMEM_SFB;
        const uint32_t a0 = smem_u32(smem + C::OFF_A), b0 = smem_u32(smem + C::OFF_B);
        const uint32_t sfa0 = smem_u32(smem + C::OFF_SFA), sfb0 = smem_u32(smem + C::OFF_SFB);
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        for (int ks = 0; ks < p.k_stages; ++ks) {
            ok = __all_sync(0xFFFFFFFFu, mbar_wait_bounded(&full[stage], phase, abort_flag, p.timeout_ns));
            if (!ok)
                break;
            tc_fence_after();
            const int nkb = min(KB, static_cast<int>(p.atoms_k) - ks * KB);
            const uint32_t sfa_s = sfa0 + stage * SF_BYTES, sfb_s = sfb0 + stage * SF_BYTES;
            const uint32_t a_s = a0 + stage * A_BYTES, b_s = b0 + stage * C::B_BYTES;
            if (elect_one()) {
                for (int kb = 0; kb < nkb; ++kb) {
                    tc_cp_32x128b_warpx4(sfa_t + kb * 4, make_smem_desc(sfa_s + kb * 512, 0, 128, 0));
                    tc_cp_32x128b_warpx4(sfb_t + kb * 4, make_smem_desc(sfb_s + kb * 512, 0, 128, 0));
                }
                for (int kb = 0; kb < nkb; ++kb)
                    tc_mma_nvfp4(tmem_base, make_smem_desc(a_s + kb * 32, 16, 1024, 2),
                                 make_smem_desc(b_s + kb * 32, 16, 1024, 2), idesc, sfa_t + kb * 4, sfb_t + kb * 4,
                                 (ks | kb) != 0);
                tc_commit(&empty[stage]);
            }
            __syncwarp();
            if (++stage == C::STAGES) {
                stage = 0;
                phase ^= 1u;
            }
        }
        if (elect_one()) {
            if (ok)
                tc_commit(acc_full);
            tc_commit(final_bar);
        }
        __syncwarp();
        volatile int no_abort = 0;
        if (!__all_sync(0xFFFFFFFFu, mbar_wait_bounded(final_bar, 0, &no_abort, DRAIN_TIMEOUT_NS)))
            *abort_flag = 1;
    } else {
        // ------------------------------------------------------------ epilogue
        const int quarter = warp & 3;
        const int nrow = w0 + quarter * 32 + lane;               // output column this lane owns
        pdl_wait_prerequisites();                               // s_x comes from the quantizer
        float alpha;
        {
            const float sx = *p.s_x;
            if (p.flags & FLAG_COLLAPSED) {
                float mx = p.s_w[0];
                for (int s = 1; s < p.nseg; ++s)
                    mx = fmaxf(mx, p.s_w[s]);
                alpha = sx * mx;
            } else {
                int seg = 0;
#pragma unroll
                for (int s = 0; s < 7; ++s)
                    seg += (s + 1 < p.nseg && nrow >= p.seg_end[s]) ? 1 : 0;
                alpha = sx * p.s_w[seg];
            }
        }
        // The four warps agree on the outcome of their bounded waits before any of
        // them reaches the named barrier below (a warp that gave up right at the
        // deadline must not strand the others there).
        const bool acc_ok = mbar_wait_bounded(acc_full, 0, abort_flag, p.timeout_ns);
        if (!bar_red_or(2, 128, acc_ok ? 0u : 1u)) {
            tc_fence_after();
            // Every stage has landed and every MMA has read its operands, so the
            // stage buffers are free: the tile is staged there as [token][128
            // columns] and leaves as 16-byte stores along each token's row.
            const bool f32 = (p.flags & FLAG_F32_OUT) != 0;
            uint8_t *stg = smem + C::OFF_A;
            constexpr int CH = (T < 32) ? T : 32;
#pragma unroll
            for (int c0 = 0; c0 < T; c0 += CH) {
                uint32_t r[CH];
                __syncwarp();
                tmem_ld_32x32b<CH>(tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + c0, r);
                tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < CH; ++i) {
                    const float v = __uint_as_float(r[i]) * alpha;
                    const int e = (c0 + i) * BW + quarter * 32 + lane;
                    if (f32)
                        reinterpret_cast<float *>(stg)[e] = v;
                    else
                        reinterpret_cast<__nv_bfloat16 *>(stg)[e] = __float2bfloat16_rn(v);
                }
            }
            bar_sync_named(1, 128);                              // the four epilogue warps
            const int esz = f32 ? 4 : 2;
            const int row_chunks = BW * esz / 16;                // 16-byte chunks per token row
            const int rows = min(T, p.m);
            uint8_t *y = static_cast<uint8_t *>(p.y);
            for (int idx = static_cast<int>(threadIdx.x) - 64; idx < rows * row_chunks; idx += 128) {
                const int t = idx / row_chunks, c = idx - t * row_chunks;
                const int col = w0 + c * (16 / esz);             // n % 8 == 0: a chunk is all in or all out
                if (col < p.n)
                    *reinterpret_cast<uint4 *>(y + (static_cast<int64_t>(t) * p.ldy + col) * esz) =
                        *reinterpret_cast<const uint4 *>(stg + (t * BW) * esz + c * 16);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 0 && *abort_flag)
        atomicCAS(&g_device_error, 0u, 6u /* NVFP4_ERR_TIMEOUT */);
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem_base, C::TMEM_COLS);
    }
}

}  // namespace decode
}  // namespace nvfp4
