// mma_peak.cuh -- measurement of the dense block-scaled FP4 tensor-core rate on
// this device: the denominator against which the prefill GEMM is judged ("Why
// Gated DeltaNet Survives 4-Bit Quantization", §2 "NVFP4": the W4A4 GEMM runs on
// native 4-bit tensor cores).  Not part of the layer.
//
// Each CTA pair issues the GEMM's own instruction -- tcgen05.mma.cta_group::2
// .kind::mxf4nvf4.block_scale.block16, M = 256, N = 256, K = 64 -- back to back
// into one tensor-memory accumulator, from one 256-deep stage of operands (each
// CTA's 128 rows of A and of B, 16 KB each) and scale factors resident in shared
// memory.  Nothing touches global memory, so the rate is the tensor pipe's.
// With `copies` set, every four MMAs are preceded by the three tcgen05.cp scale
// copies the GEMM makes per stage, which share the tensor pipe.  The operands
// are arbitrary E2M1 codes with scale 1.0: the accumulator's value is never read.
// One CTA per SM (the shared-memory request makes sure of it), and as in the
// GEMM the issuing warp runs the loop as a whole warp and issues from one
// elected lane.
#pragma once

#include <cstdint>

#include "sm100_ptx.cuh"

namespace nvfp4 {
namespace peak {

constexpr int THREADS = 128;
constexpr int KB = 4;                      // MMAs per stage (256-deep)
constexpr int A_BYTES = 128 * 128;         // 128 rows x 256 K of E2M1 codes
constexpr int B_BYTES = 128 * 128;
constexpr int SFA_BYTES = KB * 512;
constexpr int SFB_BYTES = 2 * KB * 512;
constexpr int OFF_A = 0;
constexpr int OFF_B = OFF_A + A_BYTES;
constexpr int OFF_SFA = OFF_B + B_BYTES;
constexpr int OFF_SFB = OFF_SFA + SFA_BYTES;
constexpr int OFF_BAR = OFF_SFB + SFB_BYTES;
constexpr int OFF_MISC = OFF_BAR + 16;
constexpr int SMEM_ALLOC = 200 * 1024;     // more than half an SM's shared memory: one CTA per SM
constexpr int TMEM_COLS = 512;
constexpr int TMEM_SFA = 256;
constexpr int TMEM_SFB = 256 + KB * 4;
constexpr uint64_t DONE_TIMEOUT_NS = 10000000000ull;   // far above any launch the host makes
static_assert(OFF_MISC + 64 + 1024 <= SMEM_ALLOC, "layout fits");
static_assert(TMEM_SFB + KB * 8 <= TMEM_COLS, "tensor memory budget");

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(THREADS, 1) mma_peak_kernel(int64_t iters, int copies)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *done = reinterpret_cast<uint64_t *>(smem + OFF_BAR);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + OFF_MISC);
    const int warp = threadIdx.x >> 5;
    const uint32_t rank = cluster_ctarank();

    // Operands: E2M1 codes from a multiplicative hash of the word index (any
    // bits are valid codes); every scale byte 0x38 = 1.0.
    uint32_t *w = reinterpret_cast<uint32_t *>(smem);
    for (int i = threadIdx.x; i < (A_BYTES + B_BYTES) / 4; i += THREADS)
        w[i] = (static_cast<uint32_t>(i) + 0x9E3779B9u * (blockIdx.x + 1)) * 0x85EBCA6Bu;
    for (int i = threadIdx.x; i < (SFA_BYTES + SFB_BYTES) / 4; i += THREADS)
        w[OFF_SFA / 4 + i] = 0x38383838u;
    fence_async_shared();                     // generic-proxy writes -> tensor-core reads
    if (threadIdx.x == 0) {
        mbar_init(done, 1);
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_slot, TMEM_COLS);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();                       // both CTAs' operands, barriers and tensor memory are ready
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (rank == 0 && warp == 0) {
        const uint32_t idesc = make_idesc_nvfp4(256, 256);
        const uint32_t a_s = smem_u32(smem + OFF_A), b_s = smem_u32(smem + OFF_B);
        const uint32_t sfa_s = smem_u32(smem + OFF_SFA), sfb_s = smem_u32(smem + OFF_SFB);
        const uint32_t sfa_t = tmem_base + TMEM_SFA, sfb_t = tmem_base + TMEM_SFB;
        for (int64_t i = -1; i < iters; ++i) {
            if (elect_one()) {
                if (i < 0 || copies) {        // the scales once, or before every stage as in the GEMM
#pragma unroll
                    for (int kb = 0; kb < KB; ++kb) {
                        tc_cp_32x128b_warpx4_pair(sfa_t + kb * 4, make_smem_desc(sfa_s + kb * 512, 0, 128, 0));
                        tc_cp_32x128b_warpx4_pair(sfb_t + kb * 8, make_smem_desc(sfb_s + kb * 512, 0, 128, 0));
                        tc_cp_32x128b_warpx4_pair(sfb_t + kb * 8 + 4,
                                                  make_smem_desc(sfb_s + KB * 512 + kb * 512, 0, 128, 0));
                    }
                }
                if (i >= 0) {
#pragma unroll
                    for (int kb = 0; kb < KB; ++kb)
                        tc_mma_nvfp4_pair(tmem_base, make_smem_desc(a_s + kb * 32, 16, 1024, 2),
                                          make_smem_desc(b_s + kb * 32, 16, 1024, 2), idesc, sfa_t + kb * 4,
                                          sfb_t + kb * 8, (i | kb) != 0);
                }
            }
            __syncwarp();
        }
        if (elect_one())
            tc_commit_pair_multicast(done, 0x3);   // arrives in both CTAs once every MMA has completed
        __syncwarp();
    }
    if (warp == 0) {
        // Both CTAs stay until the MMAs (which read both CTAs' shared memory and
        // write both tensor memories) are done.
        volatile int no_abort = 0;
        if (!__all_sync(0xFFFFFFFFu, mbar_wait_bounded(done, 0, &no_abort, DONE_TIMEOUT_NS)) &&
            (threadIdx.x & 31) == 0)
            atomicCAS(&g_device_error, 0u, 6u /* NVFP4_ERR_TIMEOUT */);
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, TMEM_COLS);
    }
}

}  // namespace peak
}  // namespace nvfp4
