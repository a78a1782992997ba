// gemm_pair.cuh -- block-scaled FP4 GEMM on CTA pairs (tcgen05 cta_group::2), sm_100a.
//
// Computes Y[m, n] = alpha[n] * sum_k (e2m1(Qx[m,k]) * e4m3(SFx[m,k/16])) *
//                                     (e2m1(Qw[n,k]) * e4m3(SFw[n,k/16]))
// with FP32 accumulation in tensor memory and alpha[n] = s_x * s_w[segment(n)]:
// the W4A4 GEMM of "Why Gated DeltaNet Survives 4-Bit Quantization" (§2 "NVFP4":
// the GEMM runs on native 4-bit tensor cores) with the per-module global scales
// of a fused GEMM kept apart (§6 "Per-module calibration vs. fused-GEMM
// scaling").  Organised for the compute-bound prefill regime:
//
//   * Two CTAs on neighbouring SMs (a cluster of 2) own a 256 x 256 output tile.
//     The even CTA issues one M=256, N=256, K=64 block-scaled MMA per 64-deep K
//     block; each CTA contributes 128 activation rows and 128 weight rows from its
//     own shared memory and keeps its 128 x 256 half of the accumulator in its own
//     tensor memory.  Each SM therefore loads 32 KB of codes per 256-deep stage
//     for 128 x 256 x 256 MACs, a third less than a single-CTA 128 x 256 tile.
//   * Five 38 KB stages per CTA.  Both CTAs' TMA loads complete on the even CTA's
//     stage barrier; the even CTA's tcgen05.commit releases the stage in both.
//     Launched with programmatic stream serialization, the set-up overlaps the
//     preceding kernel; behind this library's activation quantizer the producers
//     also request the weight tiles and scales of their first five stages before
//     griddepcontrol.wait (otherwise nothing global is touched before it).
//   * Eight epilogue warps per CTA drain the accumulator into registers (128
//     columns each), hand the tensor memory back to the MMA issuer at once, and
//     only then scale and convert -- the next tile's MMAs overlap the rest of the
//     epilogue.  bf16 results leave through a 32 KB shared-memory staging tile
//     (two 128 x 64 sub-tiles, 128-byte swizzle: conflict-free 16-byte writes)
//     in two rounds, one per 128-column half, each ending in two TMA stores.
//   * Scale factors travel as 512-byte atoms through 3-D tensor maps; both CTAs
//     load the full 256-row weight-scale block (no multicast of any kind).
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "sm100_ptx.cuh"

namespace nvfp4 {
namespace pair {

constexpr int BM = 256;                 // output rows per pair (128 per CTA)
constexpr int BN = 256;                 // output columns per pair (MMA N)
constexpr int BK = 256;                 // K elements per stage
constexpr int KB = BK / 64;
constexpr int STAGES = 5;
constexpr int A_BYTES = 128 * BK / 2;   // this CTA's 128 activation rows
constexpr int B_BYTES = 128 * BK / 2;   // this CTA's 128 weight rows
constexpr int SFA_BYTES = KB * 512;     // this CTA's 128-row scale block
constexpr int SFB_BYTES = 2 * KB * 512; // all 256 weight rows' scales
constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
constexpr uint32_t TX_BYTES = 2 * STAGE_BYTES;   // both CTAs complete on the even CTA's barrier
constexpr int EPI_WARPS = 8;
constexpr int THREADS = 64 + 32 * EPI_WARPS;
constexpr int TMEM_COLS = 512;
constexpr int TMEM_SFA = BN;
constexpr int TMEM_SFB = BN + KB * 4;
constexpr uint64_t DRAIN_TIMEOUT_NS = 1000000000ull;

constexpr int OFF_A = 0;
constexpr int OFF_B = OFF_A + STAGES * A_BYTES;
constexpr int OFF_SFA = OFF_B + STAGES * B_BYTES;
constexpr int OFF_SFB = OFF_SFA + STAGES * SFA_BYTES;
constexpr int OFF_STG = OFF_SFB + STAGES * SFB_BYTES;   // bf16 output staging: 2 x [128 rows x 64 cols]
constexpr int STG_SUB = 128 * 64 * 2;
constexpr int OFF_BAR = OFF_STG + 2 * STG_SUB;
constexpr int NUM_BARS = 2 * STAGES + 3;
constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;   // +0 TMEM base, +4 abort flag, +8 peer's abort flag, +16 alpha[8]
constexpr int OFF_DRAIN = OFF_MISC + 64;            // copy records (struct Drain)
constexpr int SMEM_ALLOC = OFF_DRAIN + 128 + 1024;
static_assert(SMEM_ALLOC <= 232448, "shared memory budget");
static_assert(TMEM_SFB + KB * 8 <= TMEM_COLS, "tensor memory budget");

constexpr unsigned FLAG_F32_OUT = 1u;
constexpr unsigned FLAG_COLLAPSED = 2u;

struct Params {
    int m, n, k;
    int tiles_m, tiles_n, k_stages;
    int group_m;                 // tile order: groups of group_m M tiles, N-major inside a group
    void *y;
    int64_t ldy;
    const float *s_x;
    const float *s_w;
    int nseg;
    int seg_end[8];
    unsigned flags;
    uint64_t timeout_ns;
    int stall_tile;              // testing: a K stage of each pair's tile number stall_tile (0 = its first tile)
    int stall_stage;             //   has its loads withheld: stage stall_stage (-1: none)
    int early_weights;           // 1: the first weight stages are requested before griddepcontrol.wait
                                 //    (behind this library's quantizer); 0: no global access before it
};

// What a CTA's producer put in flight, per ring slot: the newest stage (by
// sequence number q = tile iteration * k_stages + ks; slot q % STAGES, barrier
// phase (q / STAGES) & 1) it issued copies for, the bytes of those copies, and,
// in the even CTA, whether that stage's barrier was armed with both CTAs'
// bytes.  Only a slot's newest stage can have copies in flight: a slot is
// reused only after the MMAs consumed its previous stage, i.e. after every byte
// of it landed.  At exit the odd CTA copies its records into peer_* of the even
// CTA, whose stage barriers count both CTAs' copies, so that after a timeout
// the even CTA can wait for exactly the copies still in flight.
struct Drain {
    int seq[STAGES];
    uint32_t bytes[STAGES];
    uint32_t armed[STAGES];
    int peer_seq[STAGES];
    uint32_t peer_bytes[STAGES];
};
static_assert(sizeof(Drain) <= 128, "copy records fit their slot");

// Records that this CTA issues `bytes` more for stage sequence number q.
__device__ __forceinline__ void note_issue(Drain *d, int q, uint32_t bytes, bool armed)
{
    const int s = q % STAGES;
    if (d->seq[s] != q) {
        d->seq[s] = q;
        d->bytes[s] = 0;
        d->armed[s] = 0;
    }
    d->bytes[s] += bytes;
    if (armed)
        d->armed[s] = 1;
}

// Segment (module) of output column `col`.
__device__ __forceinline__ int col_segment(const Params &p, int col)
{
    int seg = 0;
#pragma unroll
    for (int s = 0; s < 7; ++s)
        seg += (s + 1 < p.nseg && col >= p.seg_end[s]) ? 1 : 0;
    return seg;
}

// Scales 32 accumulator columns starting at output column nc by their segment's
// alpha (from the per-CTA table in shared memory).  Segment boundaries are
// multiples of 8 columns, so one alpha serves each group of 8.
__device__ __forceinline__ void scale32(const Params &p, const float *alpha, int nc, const uint32_t *r, float *v)
{
#pragma unroll
    for (int g = 0; g < 4; ++g) {
        const float a = alpha[col_segment(p, min(nc + 8 * g, p.n - 1))];
#pragma unroll
        for (int i = 0; i < 8; ++i)
            v[8 * g + i] = __uint_as_float(r[8 * g + i]) * a;
    }
}

// Output tile `tile` of the persistent schedule.  Tiles are visited in groups of
// group_m consecutive M tiles, N-major inside a group, so that the tiles in
// flight at once share fewer operand rows and more of them stay in L2.  The
// producer and the epilogue warps use the same order.
__device__ __forceinline__ void tile_coords(const Params &p, int tile, int &mb, int &nb)
{
    const int group_tiles = p.group_m * p.tiles_n;
    const int g = tile / group_tiles;
    const int first_m = g * p.group_m;
    const int rows = min(p.group_m, p.tiles_m - first_m);
    const int idx = tile - g * group_tiles;
    mb = first_m + idx % rows;
    nb = idx / rows;
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(THREADS, 1)
    nvfp4_gemm_pair_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                           const __grid_constant__ CUtensorMap tm_sfa, const __grid_constant__ CUtensorMap tm_sfb,
                           const __grid_constant__ CUtensorMap tm_y, const Params p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + OFF_BAR);
    uint64_t *empty = full + STAGES;
    uint64_t *acc_full = full + 2 * STAGES;
    uint64_t *acc_empty = acc_full + 1;
    uint64_t *final_bar = acc_full + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + OFF_MISC + 4);
    volatile int *peer_abort = reinterpret_cast<volatile int *>(smem + OFF_MISC + 8);
    Drain *drain = reinterpret_cast<Drain *>(smem + OFF_DRAIN);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();          // 0: issues the MMAs
    const int pair_id = blockIdx.x >> 1;
    const int npairs = gridDim.x >> 1;
    const int num_tiles = p.tiles_m * p.tiles_n;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(acc_full, 1);
        mbar_init(acc_empty, 2 * EPI_WARPS);
        mbar_init(final_bar, 1);
        *abort_flag = 0;
        *peer_abort = 0;
        for (int s = 0; s < STAGES; ++s) {
            drain->seq[s] = -1;
            drain->bytes[s] = 0;
            drain->armed[s] = 0;
            drain->peer_seq[s] = -1;
            drain->peer_bytes[s] = 0;
        }
        fence_barrier_init();
        prefetch_tensormap(&tm_a);
        prefetch_tensormap(&tm_b);
        prefetch_tensormap(&tm_sfa);
        prefetch_tensormap(&tm_sfb);
        prefetch_tensormap(&tm_y);
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_slot, TMEM_COLS);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    __syncthreads();
    __syncwarp();
    cluster_sync_all();                                // barriers of both CTAs are initialised
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------------ producer (both CTAs)
        // The whole warp walks the schedule (so every operand below is
        // warp-uniform); one elected lane issues the copies.
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        const uint32_t bar0 = map_to_rank(smem_u32(&full[0]), 0);
        const uint64_t keep = policy_evict_last();       // operand tiles are re-read by other pairs
        // The weight operand does not depend on the preceding kernel: the weight
        // tiles and scales of this pair's first `pre` stages are requested before
        // waiting for it (their slots are free; each stage's barrier expects the
        // bytes of all four copies of both CTAs).  Testing hook: withholding one
        // stage (no arrival, no copies) makes the MMA issuer's bounded wait on it
        // run out.
        const int pre = pair_id < num_tiles ? min(STAGES, p.k_stages) : 0;
        if (!p.early_weights)
            pdl_wait_prerequisites();                    // the predecessor may write any input
        {
            int mb0, nb;
            tile_coords(p, pair_id, mb0, nb);
            const int row_b = nb * BN + static_cast<int>(rank) * 128;
            for (int ks = 0; ks < pre; ++ks) {
                if (!(p.stall_tile == 0 && ks == p.stall_stage) && elect_one()) {
                    const uint32_t bar = bar0 + ks * 8;
                    note_issue(drain, ks, B_BYTES + SFB_BYTES, rank == 0);
                    if (rank == 0)
                        mbar_arrive_expect_tx(&full[ks], TX_BYTES);
                    tma_load_2d_pair_hint(smem + OFF_B + ks * B_BYTES, &tm_b, ks * (BK / 2), row_b, bar, keep);
                    tma_load_3d_pair(smem + OFF_SFB + ks * SFB_BYTES, &tm_sfb, 0, ks * KB, nb * 2, bar);
                }
                __syncwarp();
            }
        }
        pdl_wait_prerequisites();                        // the activation codes and scales are written
        int it = 0;                                      // this pair's tile iteration
        for (int tile = pair_id; tile < num_tiles && ok; tile += npairs, ++it) {
            int mb, nb;
            tile_coords(p, tile, mb, nb);
            const int row_a = mb * BM + static_cast<int>(rank) * 128;
            const int row_b = nb * BN + static_cast<int>(rank) * 128;
            for (int ks = 0; ks < p.k_stages; ++ks) {
                ok = __all_sync(0xFFFFFFFFu, mbar_wait_bounded(&empty[stage], phase ^ 1u, abort_flag, p.timeout_ns));
                if (!ok)
                    break;
                const uint32_t bar = bar0 + stage * 8;
                const bool withhold = it == p.stall_tile && ks == p.stall_stage;
                const bool weights_issued = it == 0 && ks < pre;
                if (!withhold && elect_one()) {
                    note_issue(drain, it * p.k_stages + ks, weights_issued ? A_BYTES + SFA_BYTES : STAGE_BYTES,
                               rank == 0 && !weights_issued);
                    if (rank == 0 && !weights_issued)
                        mbar_arrive_expect_tx(&full[stage], TX_BYTES);
                    tma_load_2d_pair_hint(smem + OFF_A + stage * A_BYTES, &tm_a, ks * (BK / 2), row_a, bar, keep);
                    tma_load_3d_pair(smem + OFF_SFA + stage * SFA_BYTES, &tm_sfa, 0, ks * KB,
                                     mb * 2 + static_cast<int>(rank), bar);
                    if (!weights_issued) {
                        tma_load_2d_pair_hint(smem + OFF_B + stage * B_BYTES, &tm_b, ks * (BK / 2), row_b, bar, keep);
                        tma_load_3d_pair(smem + OFF_SFB + stage * SFB_BYTES, &tm_sfb, 0, ks * KB, nb * 2, bar);
                    }
                }
                __syncwarp();
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
        // Nothing is left to issue: let the next kernel in the stream be scheduled
        // into the slots this grid frees (it waits for this grid's completion
        // before it reads anything this grid writes).
        pdl_launch_dependents();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer (even CTA)
        // The whole warp runs the loop; an elected lane issues the scale copies,
        // the MMAs and the commits (always the same lane, lane 0, since the warp
        // is converged there, so one thread's commits cover all its MMAs).
        if (rank == 0) {
            const uint32_t idesc = make_idesc_nvfp4(BM, BN);
            const uint32_t sfa_t = tmem_base + TMEM_SFA;
            const uint32_t sfb_t = tmem_base + TMEM_SFB;
            const uint32_t a0 = smem_u32(smem + OFF_A), b0 = smem_u32(smem + OFF_B);
            const uint32_t sfa0 = smem_u32(smem + OFF_SFA), sfb0 = smem_u32(smem + OFF_SFB);
            int stage = 0;
            uint32_t phase = 0, acc_phase = 0;
            bool ok = true;
            for (int tile = pair_id; tile < num_tiles && ok; tile += npairs) {
                ok = __all_sync(0xFFFFFFFFu, mbar_wait_bounded(acc_empty, acc_phase ^ 1u, abort_flag, p.timeout_ns));
                if (!ok)
                    break;
                tc_fence_after();
                for (int ks = 0; ks < p.k_stages; ++ks) {
                    ok = __all_sync(0xFFFFFFFFu, mbar_wait_bounded(&full[stage], phase, abort_flag, p.timeout_ns));
                    if (!ok)
                        break;
                    tc_fence_after();
                    const uint32_t sfa_s = sfa0 + stage * SFA_BYTES, sfb_s = sfb0 + stage * SFB_BYTES;
                    const uint32_t a_s = a0 + stage * A_BYTES, b_s = b0 + stage * B_BYTES;
                    if (elect_one()) {
#pragma unroll
                        for (int kb = 0; kb < KB; ++kb) {
                            tc_cp_32x128b_warpx4_pair(sfa_t + kb * 4, make_smem_desc(sfa_s + kb * 512, 0, 128, 0));
                            tc_cp_32x128b_warpx4_pair(sfb_t + kb * 8, make_smem_desc(sfb_s + kb * 512, 0, 128, 0));
                            tc_cp_32x128b_warpx4_pair(sfb_t + kb * 8 + 4,
                                                      make_smem_desc(sfb_s + KB * 512 + kb * 512, 0, 128, 0));
                        }
#pragma unroll
                        for (int kb = 0; kb < KB; ++kb)
                            tc_mma_nvfp4_pair(tmem_base, make_smem_desc(a_s + kb * 32, 16, 1024, 2),
                                              make_smem_desc(b_s + kb * 32, 16, 1024, 2), idesc, sfa_t + kb * 4,
                                              sfb_t + kb * 8, (ks | kb) != 0);
                        tc_commit_pair_multicast(&empty[stage], 0x3);
                    }
                    __syncwarp();
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok)
                    break;
                if (elect_one())
                    tc_commit_pair_multicast(acc_full, 0x3);
                __syncwarp();
                acc_phase ^= 1u;
            }
            if (elect_one())
                tc_commit_pair(final_bar);
            __syncwarp();
            // Wait for the last MMAs even when another role gave up (abort set):
            // the tensor memory is released only after they are done.
            volatile int no_abort = 0;
            if (!__all_sync(0xFFFFFFFFu, mbar_wait_bounded(final_bar, 0, &no_abort, DRAIN_TIMEOUT_NS)))
                *abort_flag = 1;
        }
    } else {
        // ------------------------------------------------------------ epilogue (both CTAs)
        const int ew = warp - 2;                        // 0..7
        const int quarter = warp & 3;                   // TMEM lanes this warp may read
        const int half = ew >> 2;                       // this warp's 128 accumulator columns
        const int col0 = half * 128;
        const int row = quarter * 32 + lane;            // row inside this CTA's 128-row half tile
        const bool issuer = (ew == 0 && lane == 0);     // issues the TMA stores
        pdl_wait_prerequisites();
        // alpha of each segment: s_x * s_w[segment] (or s_x * max s_w for the
        // collapsed negative control), computed once per CTA.
        float *alpha = reinterpret_cast<float *>(smem + OFF_MISC + 16);
        if (ew == 0 && lane == 0) {
            const float sx = *p.s_x;
            float swmax = p.s_w[0];
            for (int s = 1; s < p.nseg; ++s)
                swmax = fmaxf(swmax, p.s_w[s]);
            for (int s = 0; s < p.nseg; ++s)
                alpha[s] = (p.flags & FLAG_COLLAPSED) ? sx * swmax : sx * p.s_w[s];
        }
        bar_sync_named(2, 32 * EPI_WARPS);
        const bool f32_out = (p.flags & FLAG_F32_OUT) != 0;
        const uint32_t acc_empty_leader = map_to_rank(smem_u32(acc_empty), 0);
        uint8_t *stg = smem + OFF_STG;
        const uint64_t stream_out = policy_evict_first();  // output tiles are written once
        uint32_t acc_phase = 0;
        for (int tile = pair_id; tile < num_tiles; tile += npairs) {
            int mb, nb;
            tile_coords(p, tile, mb, nb);
            const bool ok = mbar_wait_bounded(acc_full, acc_phase, abort_flag, p.timeout_ns);
            // All eight warps take the same decision (each reaches this barrier after
            // its own bounded wait), so the named barriers below cannot strand one.
            if (bar_red_or(1, 32 * EPI_WARPS, ok ? 0u : 1u))
                break;
            tc_fence_after();
            uint32_t r[128];
            __syncwarp();
            const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + col0;
            tmem_ld_32x32b_x32(taddr + 0, *reinterpret_cast<uint32_t(*)[32]>(r + 0));
            tmem_ld_32x32b_x32(taddr + 32, *reinterpret_cast<uint32_t(*)[32]>(r + 32));
            tmem_ld_32x32b_x32(taddr + 64, *reinterpret_cast<uint32_t(*)[32]>(r + 64));
            tmem_ld_32x32b_x32(taddr + 96, *reinterpret_cast<uint32_t(*)[32]>(r + 96));
            tmem_ld_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive_remote(acc_empty_leader);    // the accumulator may be overwritten now
            acc_phase ^= 1u;

            const int m0 = mb * BM + static_cast<int>(rank) * 128;     // first row of this CTA's half tile
            const int n0 = nb * BN;
            if (!f32_out) {
                // Scale and round this warp's 128 columns to packed bf16 pairs.
                uint32_t pk[64];
#pragma unroll
                for (int c = 0; c < 128; c += 32) {
                    float v[32];
                    scale32(p, alpha, n0 + col0 + c, r + c, v);
#pragma unroll
                    for (int i = 0; i < 32; i += 2) {
                        __nv_bfloat162 h = __floats2bfloat162_rn(v[i], v[i + 1]);
                        pk[(c + i) >> 1] = *reinterpret_cast<uint32_t *>(&h);
                    }
                }
                // Two rounds, one per 128-column half: the half's four warps write
                // the staging tile, then one thread stores it.
#pragma unroll
                for (int round = 0; round < 2; ++round) {
                    // The previous stores must have finished reading the staging tile.
                    if (issuer)
                        bulk_wait_group_read0();
                    bar_sync_named(2, 32 * EPI_WARPS);
                    if (half == round) {
#pragma unroll
                        for (int chunk16 = 0; chunk16 < 16; ++chunk16) {       // 16 chunks of 8 columns
                            const int sub = chunk16 >> 3, chunk = chunk16 & 7;
                            uint8_t *base = stg + sub * STG_SUB + row * 128;
                            *reinterpret_cast<uint4 *>(base + ((chunk ^ (row & 7)) << 4)) =
                                make_uint4(pk[chunk16 * 4 + 0], pk[chunk16 * 4 + 1], pk[chunk16 * 4 + 2],
                                           pk[chunk16 * 4 + 3]);
                        }
                        fence_async_shared();
                    }
                    bar_sync_named(2, 32 * EPI_WARPS);
                    if (issuer && m0 < p.m) {
#pragma unroll
                        for (int sub = 0; sub < 2; ++sub) {
                            const int col = n0 + round * 128 + sub * 64;
                            if (col < p.n)
                                tma_store_2d_hint(&tm_y, col, m0, stg + sub * STG_SUB, stream_out);
                        }
                        bulk_commit_group();
                    }
                }
            } else {
                const int m = m0 + row;
                if (m < p.m) {
#pragma unroll
                    for (int c = 0; c < 128; c += 32) {
                        const int nc = n0 + col0 + c;
                        if (nc >= p.n)
                            break;
                        float v[32];
                        scale32(p, alpha, nc, r + c, v);
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
            }
        }
        if (issuer)
            bulk_wait_group0();                         // every output store has completed
    }

    tc_fence_before();
    __syncthreads();
    // Every role of this CTA is done.  Each CTA tells the other whether it gave
    // up, and the odd CTA hands its copy records to the even one.
    if (threadIdx.x == 0) {
        st_cluster_u32(map_to_rank(smem_u32(const_cast<int *>(peer_abort)), rank ^ 1u), *abort_flag ? 1u : 0u);
        if (rank == 1) {
            for (int s = 0; s < STAGES; ++s) {
                st_cluster_u32(map_to_rank(smem_u32(&drain->peer_seq[s]), 0), static_cast<uint32_t>(drain->seq[s]));
                st_cluster_u32(map_to_rank(smem_u32(&drain->peer_bytes[s]), 0), drain->bytes[s]);
            }
        }
    }
    __syncwarp();
    cluster_sync_all();                                 // the peer's MMAs are finished; the records are visible
    if (*abort_flag || *peer_abort) {
        // A role gave up, so some stage barriers were left unobserved and copies
        // issued by either CTA may still be landing in its shared memory.  Both
        // CTAs' copies complete on the even CTA's stage barriers: for each ring
        // slot's newest stage the even CTA accounts for the bytes that were
        // expected but never sent (or arms the stage with the bytes the odd CTA
        // sent without it), then waits, bounded, until the phase completes --
        // that is, until every copy of that stage has landed.  The odd CTA waits
        // at the cluster barrier meanwhile.
        if (rank == 0 && threadIdx.x == 0) {
            for (int s = 0; s < STAGES; ++s) {
                const int q0 = drain->seq[s], q1 = drain->peer_seq[s];
                const int q = max(q0, q1);
                if (q < 0)
                    continue;
                const uint32_t b = (q0 == q ? drain->bytes[s] : 0u) + (q1 == q ? drain->peer_bytes[s] : 0u);
                if (q0 == q && drain->armed[s] != 0) {
                    if (b < TX_BYTES)
                        mbar_complete_tx(&full[s], TX_BYTES - b);
                } else if (b != 0) {
                    mbar_arrive_expect_tx(&full[s], b);
                } else {
                    continue;
                }
                volatile int no_abort = 0;
                mbar_wait_bounded(&full[s], static_cast<uint32_t>((q / STAGES) & 1), &no_abort, DRAIN_TIMEOUT_NS);
            }
        }
        __syncwarp();
        cluster_sync_all();                             // no copy is in flight into either CTA
    }
    if (threadIdx.x == 0 && *abort_flag)
        atomicCAS(&g_device_error, 0u, 6u /* NVFP4_ERR_TIMEOUT */);
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, TMEM_COLS);
    }
}

}  // namespace pair
}  // namespace nvfp4
