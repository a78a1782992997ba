// gemm_decode_split.cuh -- the decode GEMM with K split over a cluster, for few
// weight tiles (small N), sm_100a.
//
// The swapped decode kernel (gemm_decode.cuh) gives each 128-row weight tile to
// one CTA for the whole K.  With few tiles (N = 5120 has 40) most SMs stay idle
// and each CTA streams a long row of stages on its own, far below the weight-
// bandwidth bound that "Why Gated DeltaNet Survives 4-Bit Quantization" puts on
// decode (§4).  Here a cluster of kSplit CTAs shares a tile:
//
//   * CTA r of the cluster streams K stages [r*S/kSplit, (r+1)*S/kSplit) of the
//     tile (weights and tokens, the same TMA and bulk copies as the decode
//     kernel) into its own tensor-memory accumulator.
//   * CTAs 1..kSplit-1 push their 128 x T fp32 partial sums into slots of CTA 0's
//     shared memory with st.async, counted on one mbarrier of CTA 0.
//   * CTA 0 adds them to its own in a fixed order (deterministic), scales by
//     alpha(n) and stores, as the decode epilogue does.
//
// Used for up to 32 tokens; the kernel is otherwise the decode kernel's
// (programmatic dependent launch, early weight stages behind the library's
// quantizer or with NVFP4_FLAG_STATIC_WEIGHTS, bounded waits, testing hooks).
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "gemm_decode.cuh"
#include "sm100_ptx.cuh"

namespace nvfp4 {
namespace decode {

constexpr int kSplit = 4;

template <int T>
struct SplitCfg {
    // Three ring stages up to 16 tokens; at 32 the three partial slots (16 KB
    // each) leave room for two beside them under two CTAs per SM.
    static constexpr int STAGES = T <= 16 ? 3 : 2;
    static constexpr int B_BYTES = T * BK / 2;
    static constexpr int STAGE = A_BYTES + B_BYTES + 2 * SF_BYTES;
    static constexpr int SLOT = BW * T * 4;                       // one CTA's fp32 partial sums
    static constexpr int OFF_A = 0;
    static constexpr int OFF_B = OFF_A + STAGES * A_BYTES;
    static constexpr int OFF_SFA = OFF_B + STAGES * B_BYTES;
    static constexpr int OFF_SFB = OFF_SFA + STAGES * SF_BYTES;
    static constexpr int OFF_SLOT = OFF_SFB + STAGES * SF_BYTES;
    static constexpr int OFF_BAR = OFF_SLOT + (kSplit - 1) * SLOT;
    static constexpr int OFF_MISC = OFF_BAR + (2 * STAGES + 3) * 8;
    static constexpr int SMEM_ALLOC = OFF_MISC + 64 + 1024;
    static constexpr int TMEM_SFA = T;
    static constexpr int TMEM_SFB = T + KB * 4;
    static constexpr int TMEM_COLS = (T + KB * 8 <= 32) ? 32 : 64;
    static_assert(T <= 32, "partials of more tokens do not fit beside the ring");
    static_assert(SMEM_ALLOC <= SMEM_LIMIT, "two CTAs per SM");
    static_assert(STAGES * A_BYTES >= T * BW * 4, "the epilogue stages a fp32 tile in the weight buffers");
    static_assert(TMEM_COLS >= T + KB * 8, "accumulator and scale columns");
    static_assert(SLOT % 16 == 0 && OFF_SLOT % 16 == 0, "16-byte partial pushes");
};

__device__ __forceinline__ void st_async_remote_v4(uint32_t cluster_addr, uint32_t a, uint32_t b, uint32_t c,
                                                   uint32_t d, uint32_t cluster_bar)
{
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.b32 [%0], {%1, %2, %3, %4}, [%5];" ::"r"(
                     cluster_addr),
                 "r"(a), "r"(b), "r"(c), "r"(d), "r"(cluster_bar)
                 : "memory");
}

template <int T>
__global__ void __cluster_dims__(kSplit, 1, 1) __launch_bounds__(THREADS, 2)
    nvfp4_gemm_decode_split_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_x,
                                   const Params p)
{
    using C = SplitCfg<T>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR);
    uint64_t *empty = full + C::STAGES;
    uint64_t *acc_full = full + 2 * C::STAGES;
    uint64_t *final_bar = acc_full + 1;
    uint64_t *slots_full = acc_full + 2;                          // CTA 0: every peer's partials landed
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const int tile = blockIdx.x / kSplit;
    const int w0 = tile * BW;
    const int ks_lo = static_cast<int>(rank) * p.k_stages / kSplit;
    const int nst = (static_cast<int>(rank) + 1) * p.k_stages / kSplit - ks_lo;   // >= 1: k_stages >= kSplit

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(acc_full, 1);
        mbar_init(final_bar, 1);
        mbar_init(slots_full, 1);
        *abort_flag = 0;
        fence_barrier_init();
        if (rank == 0)
            mbar_arrive_expect_tx(slots_full, (kSplit - 1) * C::SLOT);
        prefetch_tensormap(&tm_w);
        prefetch_tensormap(&tm_x);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();                                          // CTA 0's slot barrier exists before any push
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        const int pre = min(C::STAGES, nst);
        if (!p.early_weights)
            pdl_wait_prerequisites();
        for (int j = 0; j < pre; ++j) {
            const int ks = ks_lo + j;
            const int nkb = min(KB, static_cast<int>(p.atoms_k) - ks * KB);
            const uint8_t *sfw_src = p.sfw + (static_cast<int64_t>(tile) * p.atoms_k + ks * KB) * 512;
            if (j != p.stall_stage && elect_one()) {
                mbar_arrive_expect_tx(&full[j], A_BYTES + C::B_BYTES + 2 * nkb * 512);
                tma_load_2d(smem + C::OFF_A + j * A_BYTES, &tm_w, ks * (BK / 2), w0, &full[j]);
                bulk_load(smem + C::OFF_SFA + j * SF_BYTES, sfw_src, nkb * 512, &full[j]);
            }
            __syncwarp();
        }
        pdl_wait_prerequisites();
        for (int j = 0; j < pre; ++j) {
            const int ks = ks_lo + j;
            const int nkb = min(KB, static_cast<int>(p.atoms_k) - ks * KB);
            if (j != p.stall_stage && elect_one()) {
                tma_load_2d(smem + C::OFF_B + j * C::B_BYTES, &tm_x, ks * (BK / 2), 0, &full[j]);
                bulk_load(smem + C::OFF_SFB + j * SF_BYTES, p.sfx + static_cast<int64_t>(ks * KB) * 512, nkb * 512,
                          &full[j]);
            }
            __syncwarp();
        }
        int stage = pre % C::STAGES;
        uint32_t phase = (pre == C::STAGES) ? 1u : 0u;
        int issued = pre;
        for (int j = pre; j < nst; ++j) {
            if (!__all_sync(0xFFFFFFFFu, mbar_wait_bounded(&empty[stage], phase ^ 1u, abort_flag, p.timeout_ns)))
                break;
            const int ks = ks_lo + j;
            const int nkb = min(KB, static_cast<int>(p.atoms_k) - ks * KB);
            const uint8_t *sfw_src = p.sfw + (static_cast<int64_t>(tile) * p.atoms_k + ks * KB) * 512;
            if (j != p.stall_stage && elect_one()) {
                mbar_arrive_expect_tx(&full[stage], A_BYTES + C::B_BYTES + 2 * nkb * 512);
                tma_load_2d(smem + C::OFF_A + stage * A_BYTES, &tm_w, ks * (BK / 2), w0, &full[stage]);
                bulk_load(smem + C::OFF_SFA + stage * SF_BYTES, sfw_src, nkb * 512, &full[stage]);
                tma_load_2d(smem + C::OFF_B + stage * C::B_BYTES, &tm_x, ks * (BK / 2), 0, &full[stage]);
                bulk_load(smem + C::OFF_SFB + stage * SF_BYTES, p.sfx + static_cast<int64_t>(ks * KB) * 512,
                          nkb * 512, &full[stage]);
            }
            __syncwarp();
            issued = j + 1;
            if (++stage == C::STAGES) {
                stage = 0;
                phase ^= 1u;
            }
        }
        pdl_launch_dependents();
        for (int q = 0; q < min(C::STAGES, issued); ++q) {
            const int j = issued - 1 - q;
            if (j == p.stall_stage)
                continue;
            volatile int no_abort = 0;
            if (!__all_sync(0xFFFFFFFFu, mbar_wait_bounded(&full[j % C::STAGES],
                                                           static_cast<uint32_t>((j / C::STAGES) & 1), &no_abort,
                                                           DRAIN_TIMEOUT_NS)))
                *abort_flag = 1;
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        const uint32_t idesc = make_idesc_nvfp4(BW, T);
        const uint32_t sfa_t = tmem_base + C::TMEM_SFA;
        const uint32_t sfb_t = tmem_base + C::TMEM_SFB;
        const uint32_t a0 = smem_u32(smem + C::OFF_A), b0 = smem_u32(smem + C::OFF_B);
        const uint32_t sfa0 = smem_u32(smem + C::OFF_SFA), sfb0 = smem_u32(smem + C::OFF_SFB);
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        for (int j = 0; j < nst; ++j) {
            ok = __all_sync(0xFFFFFFFFu, mbar_wait_bounded(&full[stage], phase, abort_flag, p.timeout_ns));
            if (!ok)
                break;
            tc_fence_after();
            const int ks = ks_lo + j;
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
                                 (j | kb) != 0);
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
        const int row = quarter * 32 + lane;                    // accumulator lane = weight row in the tile
        const int nrow = w0 + row;
        const bool acc_ok = mbar_wait_bounded(acc_full, 0, abort_flag, p.timeout_ns);
        const bool any_fail = bar_red_or(2, 128, acc_ok ? 0u : 1u);
        uint32_t r[T];
        if (!any_fail) {
            tc_fence_after();
            __syncwarp();
            constexpr int CH = (T < 32) ? T : 32;
#pragma unroll
            for (int c0 = 0; c0 < T; c0 += CH)
                tmem_ld_32x32b<CH>(tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + c0, r + c0);
            tmem_ld_wait();
        } else {
#pragma unroll
            for (int i = 0; i < T; ++i)
                r[i] = 0u;
        }
        if (rank != 0) {
            // Always push, also after a failed wait, so that CTA 0's slot barrier
            // completes and no copy into it is outstanding when it leaves.
            const uint32_t dst =
                map_to_rank(smem_u32(smem + C::OFF_SLOT + (rank - 1) * C::SLOT + row * T * 4), 0);
            const uint32_t bar = map_to_rank(smem_u32(slots_full), 0);
#pragma unroll
            for (int i = 0; i < T; i += 4)
                st_async_remote_v4(dst + i * 4, r[i], r[i + 1], r[i + 2], r[i + 3], bar);
        } else {
            pdl_wait_prerequisites();                           // s_x comes from the quantizer
            float alpha;
            if (p.flags & FLAG_COLLAPSED) {
                float mx = p.s_w[0];
                for (int s = 1; s < p.nseg; ++s)
                    mx = fmaxf(mx, p.s_w[s]);
                alpha = *p.s_x * mx;
            } else {
                int seg = 0;
#pragma unroll
                for (int s = 0; s < 7; ++s)
                    seg += (s + 1 < p.nseg && nrow >= p.seg_end[s]) ? 1 : 0;
                alpha = *p.s_x * p.s_w[seg];
            }
            const bool slots_ok = mbar_wait_bounded(slots_full, 0, abort_flag, p.timeout_ns);
            if (!bar_red_or(3, 128, (slots_ok && !any_fail) ? 0u : 1u)) {
                // Partial sums in a fixed order: own K quarter, then CTAs 1, 2, 3.
                float v[T];
#pragma unroll
                for (int i = 0; i < T; ++i)
                    v[i] = __uint_as_float(r[i]);
#pragma unroll
                for (int s = 0; s < kSplit - 1; ++s) {
                    const float4 *slot =
                        reinterpret_cast<const float4 *>(smem + C::OFF_SLOT + s * C::SLOT + row * T * 4);
#pragma unroll
                    for (int i = 0; i < T; i += 4) {
                        const float4 q = slot[i / 4];
                        v[i] += q.x;
                        v[i + 1] += q.y;
                        v[i + 2] += q.z;
                        v[i + 3] += q.w;
                    }
                }
                const bool f32 = (p.flags & FLAG_F32_OUT) != 0;
                uint8_t *stg = smem + C::OFF_A;                   // every weight stage has been consumed
#pragma unroll
                for (int i = 0; i < T; ++i) {
                    const float o = v[i] * alpha;
                    const int e = i * BW + row;
                    if (f32)
                        reinterpret_cast<float *>(stg)[e] = o;
                    else
                        reinterpret_cast<__nv_bfloat16 *>(stg)[e] = __float2bfloat16_rn(o);
                }
                bar_sync_named(1, 128);
                const int esz = f32 ? 4 : 2;
                const int row_chunks = BW * esz / 16;
                const int rows = min(T, p.m);
                uint8_t *y = static_cast<uint8_t *>(p.y);
                for (int idx = static_cast<int>(threadIdx.x) - 64; idx < rows * row_chunks; idx += 128) {
                    const int t = idx / row_chunks, c = idx - t * row_chunks;
                    const int col = w0 + c * (16 / esz);
                    if (col < p.n)
                        *reinterpret_cast<uint4 *>(y + (static_cast<int64_t>(t) * p.ldy + col) * esz) =
                            *reinterpret_cast<const uint4 *>(stg + (t * BW) * esz + c * 16);
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 0) {
        if (rank == 0) {
            // The peers push unconditionally; after a failed wait above, wait
            // (bounded) for their bytes before this CTA's memory is released.
            volatile int no_abort = 0;
            mbar_wait_bounded(slots_full, 0, &no_abort, DRAIN_TIMEOUT_NS);
        }
        if (*abort_flag)
            atomicCAS(&g_device_error, 0u, 6u /* NVFP4_ERR_TIMEOUT */);
    }
    __syncwarp();
    cluster_sync_all();                                          // no push into CTA 0 is in flight
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem_base, C::TMEM_COLS);
    }
}

}  // namespace decode
}  // namespace nvfp4
