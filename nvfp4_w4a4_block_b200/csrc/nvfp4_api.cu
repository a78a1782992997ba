// nvfp4_api.cu -- the C ABI declared in include/nvfp4.h: host-side validation,
// workspace layout, TMA descriptor construction and kernel launches.
//
// Workspace layout (caller-owned device memory, no initialisation needed):
//   [0, 32 KB)            amax partials: up to 8 segments x 1024 CTAs x 4 bytes
//   [32 KB, +m*k/2)       activation codes Qx (nvfp4_linear*)
//   [.., +sf_bytes(m,k))  activation block scales SFx (nvfp4_linear*)
//   +16 bytes             activation global scale s_x (nvfp4_linear*)
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <cstdint>
#include <utility>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "nvfp4.h"
#include "convert.cuh"
#include "gemm_decode.cuh"
#include "gemm_decode_split.cuh"
#include "gemm_pair.cuh"
#include "mma_peak.cuh"
#include "quantize.cuh"

// Device scratch of nvfp4_linear_fused_noalloc (see include/nvfp4.h).  In host
// code this name is only a stand-in for the device array: its device address is
// looked up per device with cudaGetSymbolAddress before any kernel gets it.
static __device__ __align__(256) uint8_t g_noalloc_scratch[NVFP4_NOALLOC_SCRATCH_BYTES];

namespace {

using namespace nvfp4;

constexpr size_t kPartialBytes = 32 * 1024;
constexpr int kMaxPartials = 1024;
constexpr size_t kAlign = 256;

std::atomic<uint64_t> g_timeout_ns{2000000000ull};
std::atomic<uint64_t> g_launches{0};       // kernel launches enqueued by this library (process-wide)

struct DeviceInfo {
    bool ready = false;
    unsigned long long ctx_id = 0;  // context the set-up below was made in
    nvfp4_status status = NVFP4_OK;
    int sms = 0;
    int tile_quant_ctas_per_sm = 1;
    int expand_ctas_per_sm = 1;
    bool cluster_quant = false;     // a 16-CTA cluster of the decode quantizer can be resident
    bool cluster_quant_mid = false;     // ... of its 1024-thread instance
    bool cluster_quant_large = false;   // ... of its 12-unit instance
};

std::mutex g_mu;
DeviceInfo g_dev[64];
thread_local int g_tile_quant_ctas = 148;   // resident tile-quantize CTAs on the current device
thread_local int g_expand_ctas = 148;       // resident expansion CTAs on the current device
thread_local bool g_cluster_quant = false;  // decode quantizer cluster available on the current device
thread_local bool g_cluster_quant_mid = false;    // its 1024-thread instance too
thread_local bool g_cluster_quant_large = false;  // its 12-unit instance too
constexpr int64_t kSmallQuantElems = int64_t(1) << 20;   // per-unit encoder below, tiled encoder above
// Decode-sized activations: one cluster launch holds the whole tensor in
// registers (quantize_cluster_kernel) up to these many elements (5 units x 512
// threads, 5 x 1024, 12 x 512 per CTA).
#define NVFP4_CLUSTER_SMALL quantize_cluster_kernel<5, 512>
#define NVFP4_CLUSTER_MID quantize_cluster_kernel<5, 1024>
#define NVFP4_CLUSTER_LARGE quantize_cluster_kernel<12, 512>
constexpr int64_t kClusterQuantElems = int64_t(kClusterCtas) * 512 * 5 * 8;
constexpr int64_t kClusterQuantElemsMid = int64_t(kClusterCtas) * 1024 * 5 * 8;
constexpr int64_t kClusterQuantElemsLarge = int64_t(kClusterCtas) * 512 * 12 * 8;
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
PFN_cuCtxGetCurrent_v4000 g_ctx_current = nullptr;
PFN_cuCtxGetId_v12000 g_ctx_get_id = nullptr;

// Unique id of the calling thread's current CUDA context on device `dev`,
// initialising the device's primary context first if no context is current.
// Per-device state (kernel attributes, the scratch address) is keyed by it: a
// cudaDeviceReset replaces the primary context, and everything set up in the
// old one is gone, so a new id means the set-up is made again.  Called with
// g_mu held.
nvfp4_status current_context_id(int dev, unsigned long long *id)
{
    if (g_ctx_current == nullptr || g_ctx_get_id == nullptr) {
        cudaDriverEntryPointQueryResult q1, q2;
        void *f1 = nullptr, *f2 = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f1, cudaEnableDefault, &q1) != cudaSuccess ||
            q1 != cudaDriverEntryPointSuccess || f1 == nullptr ||
            cudaGetDriverEntryPoint("cuCtxGetId", &f2, cudaEnableDefault, &q2) != cudaSuccess ||
            q2 != cudaDriverEntryPointSuccess || f2 == nullptr)
            return NVFP4_ERR_CUDA;
        g_ctx_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(f1);
        g_ctx_get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(f2);
    }
    CUcontext ctx = nullptr;
    if (g_ctx_current(&ctx) != CUDA_SUCCESS)
        return NVFP4_ERR_CUDA;
    if (ctx == nullptr) {
        if (cudaSetDevice(dev) != cudaSuccess || g_ctx_current(&ctx) != CUDA_SUCCESS || ctx == nullptr)
            return NVFP4_ERR_CUDA;
    }
    return g_ctx_get_id(ctx, id) == CUDA_SUCCESS ? NVFP4_OK : NVFP4_ERR_CUDA;
}

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

nvfp4_status cuda_status(cudaError_t e) { return e == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA; }

// Kernel launch; with `pdl` the kernel may start before the previous kernel in
// the stream finishes (programmatic stream serialization) and must call
// griddepcontrol.wait before it touches that kernel's results.
template <typename... KArgs, typename... Args>
cudaError_t launch(void (*kernel)(KArgs...), int grid, int block, size_t smem, cudaStream_t stream, bool pdl,
                   Args &&...args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(static_cast<unsigned>(block));
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
    if (e == cudaSuccess)
        g_launches.fetch_add(1, std::memory_order_relaxed);
    return e;
}

// One-time per-device (per-context) set-up: capability check, SM count, kernel
// attributes, driver entry point for tensor-map encoding.
nvfp4_status device_setup(int *sms)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return NVFP4_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mu);
    DeviceInfo &d = g_dev[dev];
    unsigned long long ctx_id = 0;
    if (current_context_id(dev, &ctx_id) != NVFP4_OK)
        return NVFP4_ERR_CUDA;
    if (d.ready && d.ctx_id != ctx_id)
        d.ready = false;                 // the context was replaced (cudaDeviceReset): set up again
    if (!d.ready) {
        d.ctx_id = ctx_id;
        int major = 0, minor = 0, sm = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return NVFP4_ERR_CUDA;
        if (major != 10 || minor != 0) {
            d.ready = true;
            d.status = NVFP4_ERR_UNSUPPORTED_DEVICE;
            return d.status;
        }
        if (cudaFuncSetAttribute(pair::nvfp4_gemm_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 pair::SMEM_ALLOC) != cudaSuccess ||
            cudaFuncSetAttribute(decode::nvfp4_gemm_decode_kernel<8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 decode::Cfg<8>::SMEM_ALLOC) != cudaSuccess ||
            cudaFuncSetAttribute(decode::nvfp4_gemm_decode_kernel<16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 decode::Cfg<16>::SMEM_ALLOC) != cudaSuccess ||
            cudaFuncSetAttribute(decode::nvfp4_gemm_decode_kernel<32>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 decode::Cfg<32>::SMEM_ALLOC) != cudaSuccess ||
            cudaFuncSetAttribute(decode::nvfp4_gemm_decode_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 decode::Cfg<64>::SMEM_ALLOC) != cudaSuccess ||
            cudaFuncSetAttribute(decode::nvfp4_gemm_decode_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 decode::Cfg<128>::SMEM_ALLOC) != cudaSuccess ||
            cudaFuncSetAttribute(decode::nvfp4_gemm_decode_split_kernel<8>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, decode::SplitCfg<8>::SMEM_ALLOC) !=
                cudaSuccess ||
            cudaFuncSetAttribute(decode::nvfp4_gemm_decode_split_kernel<16>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, decode::SplitCfg<16>::SMEM_ALLOC) !=
                cudaSuccess ||
            cudaFuncSetAttribute(decode::nvfp4_gemm_decode_split_kernel<32>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, decode::SplitCfg<32>::SMEM_ALLOC) !=
                cudaSuccess ||
            cudaFuncSetAttribute(peak::mma_peak_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 peak::SMEM_ALLOC) != cudaSuccess)
            return NVFP4_ERR_CUDA;
        if (g_encode == nullptr) {
            cudaDriverEntryPointQueryResult q;
            void *fn = nullptr;
            if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
                q != cudaDriverEntryPointSuccess || fn == nullptr)
                return NVFP4_ERR_CUDA;
            g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
        }
        // The decode-size quantizer runs as one cluster of 16 CTAs (beyond the
        // portable 8, which sm_100 allows once the kernel opts in).
        if (cudaFuncSetAttribute(NVFP4_CLUSTER_SMALL, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) !=
                cudaSuccess ||
            cudaFuncSetAttribute(NVFP4_CLUSTER_MID, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess ||
            cudaFuncSetAttribute(NVFP4_CLUSTER_LARGE, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) !=
                cudaSuccess)
            return NVFP4_ERR_CUDA;
        {
            // A device (or partition) that cannot hold one such cluster takes the
            // amax pass + per-unit encoder instead.
            auto resident = [](auto kernel, int threads) {
                cudaLaunchConfig_t cc = {};
                cc.gridDim = dim3(kClusterCtas);
                cc.blockDim = dim3(static_cast<unsigned>(threads));
                int nclusters = 0;
                const bool ok = cudaOccupancyMaxActiveClusters(&nclusters, kernel, &cc) == cudaSuccess && nclusters >= 1;
                cudaGetLastError();     // a refused query leaves no sticky error behind
                return ok;
            };
            d.cluster_quant = resident(NVFP4_CLUSTER_SMALL, 512);
            d.cluster_quant_mid = d.cluster_quant && resident(NVFP4_CLUSTER_MID, 1024);
            d.cluster_quant_large = d.cluster_quant && resident(NVFP4_CLUSTER_LARGE, 512);
            // NVFP4_NO_CLUSTER_QUANTIZER=1 takes the same fallback on any device
            // (it is how the fallback is tested on parts where the cluster fits).
            const char *no_cluster = std::getenv("NVFP4_NO_CLUSTER_QUANTIZER");
            if (no_cluster != nullptr && no_cluster[0] == '1')
                d.cluster_quant = d.cluster_quant_mid = d.cluster_quant_large = false;
        }
        int occ = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, quantize_tile_kernel, kQuantThreads, 0) !=
            cudaSuccess)
            return NVFP4_ERR_CUDA;
        d.tile_quant_ctas_per_sm = occ > 0 ? occ : 1;
        occ = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, convert::expand_kernel, convert::kThreads, 0) !=
            cudaSuccess)
            return NVFP4_ERR_CUDA;
        d.expand_ctas_per_sm = occ > 0 ? occ : 1;
        d.sms = sm;
        d.status = NVFP4_OK;
        d.ready = true;
    }
    *sms = d.sms;
    g_tile_quant_ctas = d.sms * d.tile_quant_ctas_per_sm;
    g_expand_ctas = d.sms * d.expand_ctas_per_sm;
    g_cluster_quant = d.cluster_quant;
    g_cluster_quant_mid = d.cluster_quant_mid;
    g_cluster_quant_large = d.cluster_quant_large;
    return d.status;
}

// Shared argument checks for an operand [rows, k] in bf16 with row stride ld.
nvfp4_status check_bf16_operand(const void *x, int64_t rows, int64_t k, int64_t ld)
{
    if (rows < 0 || k <= 0 || ld < k)
        return NVFP4_ERR_INVALID_ARG;
    if (k % 64 != 0)
        return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (rows > (int64_t(1) << 31) || k > (int64_t(1) << 30))
        return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (rows > 0 && x == nullptr)
        return NVFP4_ERR_INVALID_ARG;
    if (!aligned16(x) || (ld * 2) % 16 != 0)
        return NVFP4_ERR_MISALIGNED;
    return NVFP4_OK;
}

// Validates a segment table over `total` rows/columns and copies its ends.
nvfp4_status read_segments(const int64_t *offsets, int nseg, int64_t total, int64_t *ends)
{
    if (nseg < 1 || nseg > NVFP4_MAX_SEGMENTS)
        return nseg > NVFP4_MAX_SEGMENTS ? NVFP4_ERR_UNSUPPORTED_SHAPE : NVFP4_ERR_INVALID_ARG;
    if (offsets == nullptr) {
        if (nseg != 1)
            return NVFP4_ERR_INVALID_ARG;
        ends[0] = total;
        return NVFP4_OK;
    }
    if (offsets[0] != 0 || offsets[nseg] != total)
        return NVFP4_ERR_INVALID_ARG;
    for (int i = 0; i < nseg; ++i)
        if (offsets[i + 1] <= offsets[i])
            return NVFP4_ERR_INVALID_ARG;
    for (int i = 0; i < nseg; ++i) {
        if (i + 1 < nseg && offsets[i + 1] % 8 != 0)      // interior boundaries; the total has its own limits
            return NVFP4_ERR_UNSUPPORTED_SHAPE;
        ends[i] = offsets[i + 1];
    }
    return NVFP4_OK;
}

int amax_grid(int sms, int64_t rows, int64_t k)
{
    const int64_t units = rows * (k / 8);
    int64_t g = (units + kQuantThreads * 4 - 1) / (kQuantThreads * 4);
    if (g > 4 * sms)
        g = 4 * sms;
    if (g > kMaxPartials)
        g = kMaxPartials;
    return static_cast<int>(g < 1 ? 1 : g);
}

int quant_grid(int sms, int64_t rows, int64_t k)
{
    const int64_t units = rows * (k / 8) + (int64_t(128) * (k / 64));   // + pad words
    int64_t g = (units + kQuantThreads - 1) / kQuantThreads;
    if (g > 8 * sms)
        g = 8 * sms;
    return static_cast<int>(g < 1 ? 1 : g);
}

// Quantization of [rows, k] (rows split into segments).  One segment, at most
// 786432 elements (decode, up to 153 tokens at K = 5120): one cluster launch
// reduces the amax (dynamic scale) and encodes: 512 threads x 5 units per CTA up
// to 327680 elements, 1024 x 5 up to 655360 (measured 0.3-0.9 us faster per call
// than 512 x 12 at 65-128 tokens), 512 x 12 above.  Up to 2^20 elements: the per-unit encoder,
// after an amax pass in dynamic mode.  Larger (or several segments): amax passes
// and the tiled encoder.
nvfp4_status launch_quantize(const void *x, int64_t rows, int64_t k, int64_t ldx, const int64_t *seg_ends, int nseg,
                             const float *static_scale, float *scale_out, uint8_t *q, uint8_t *sf,
                             uint32_t *partials, int sms, cudaStream_t stream)
{
    const int ga = amax_grid(sms, rows, k);
    if (nseg == 1 && rows * k <= kSmallQuantElems) {
        const int64_t elems = rows * k;
        const bool cluster_small = g_cluster_quant && elems <= kClusterQuantElems;
        const bool cluster_mid = !cluster_small && g_cluster_quant_mid && elems <= kClusterQuantElemsMid;
        const bool cluster_large = !cluster_small && !cluster_mid && g_cluster_quant_large &&
                                   elems <= kClusterQuantElemsLarge;
        const bool cluster = cluster_small || cluster_mid || cluster_large;
        if (static_scale == nullptr && !cluster) {
            AmaxParams ap;
            ap.x = static_cast<const uint16_t *>(x);
            ap.row_begin = 0;
            ap.row_end = rows;
            ap.k = k;
            ap.ldx = ldx;
            ap.partial = partials;
            if (launch(amax_partial_kernel, ga, kQuantThreads, 0, stream, false, ap) != cudaSuccess)
                return NVFP4_ERR_CUDA;
        }
        QuantParams qp;
        memset(&qp, 0, sizeof qp);
        qp.x = static_cast<const uint16_t *>(x);
        qp.rows = rows;
        qp.k = k;
        qp.ldx = ldx;
        qp.q = reinterpret_cast<uint32_t *>(q);
        qp.sf = sf;
        qp.rows_pad = (rows + 127) / 128 * 128;
        qp.kb_pad = ((k / 16) + 3) / 4 * 4;
        qp.nseg = 1;
        qp.seg_end[0] = rows;
        qp.static_scale = static_scale;
        qp.partial = partials;
        qp.npartial = ga;
        qp.scale_out = scale_out;
        qp.timeout_ns = g_timeout_ns.load();
        if (cluster_small)
            return cuda_status(launch(NVFP4_CLUSTER_SMALL, kClusterCtas, 512, 0, stream, true, qp));
        if (cluster_mid)
            return cuda_status(launch(NVFP4_CLUSTER_MID, kClusterCtas, 1024, 0, stream, true, qp));
        if (cluster_large)
            return cuda_status(launch(NVFP4_CLUSTER_LARGE, kClusterCtas, 512, 0, stream, true, qp));
        const int grid = quant_grid(sms, rows, k);
        return cuda_status(launch(quantize_kernel, grid, kQuantThreads, 0, stream, true, qp));
    }
    if (static_scale == nullptr) {
        int64_t begin = 0;
        for (int s = 0; s < nseg; ++s) {
            AmaxParams ap;
            ap.x = static_cast<const uint16_t *>(x);
            ap.row_begin = begin;
            ap.row_end = seg_ends[s];
            ap.k = k;
            ap.ldx = ldx;
            ap.partial = partials + s * ga;
            if (launch(amax_partial_kernel, ga, kQuantThreads, 0, stream, false, ap) != cudaSuccess)
                return NVFP4_ERR_CUDA;
            begin = seg_ends[s];
        }
    }
    TileQuantParams tp;
    memset(&tp, 0, sizeof tp);
    tp.x = static_cast<const uint16_t *>(x);
    tp.rows = rows;
    tp.k = k;
    tp.ldx = ldx;
    tp.q = q;
    tp.sf = sf;
    tp.row_tiles = (rows + 127) / 128;
    tp.col_tiles = k / 64;
    tp.nseg = nseg;
    for (int s = 0; s < nseg; ++s)
        tp.seg_end[s] = seg_ends[s];
    tp.static_scale = static_scale;
    tp.partial = partials;
    tp.npartial = ga;
    tp.scale_out = scale_out;
    const int64_t tiles = tp.row_tiles * tp.col_tiles;
    const int grid = static_cast<int>(tiles < g_tile_quant_ctas ? tiles : g_tile_quant_ctas);
    return cuda_status(launch(quantize_tile_kernel, grid, kQuantThreads, 0, stream, true, tp));
}

nvfp4_status make_map(CUtensorMap *map, const void *base, uint64_t inner_bytes, uint64_t rows, uint32_t box_rows)
{
    cuuint64_t dims[2] = {inner_bytes, rows};
    cuuint64_t strides[1] = {inner_bytes};
    cuuint32_t box[2] = {128, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? NVFP4_OK : NVFP4_ERR_CUDA;
}

// Scale atoms as a 3-D tensor: 512-byte atoms (128 x 32-bit), atoms along K,
// 128-row blocks; a box is 4 atoms (one 256-deep stage) of box_rb row blocks.
nvfp4_status make_sf_map(CUtensorMap *map, const void *base, uint64_t atoms_k, uint64_t row_blocks, uint32_t box_rb)
{
    cuuint64_t dims[3] = {128, atoms_k, row_blocks};
    cuuint64_t strides[2] = {512, atoms_k * 512};
    cuuint32_t box[3] = {128, 4, box_rb};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, const_cast<void *>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? NVFP4_OK : NVFP4_ERR_CUDA;
}

// bf16 output as a TMA store target: [m, n] with row stride ldy elements, boxes
// of 64 columns x 128 rows with 128-byte swizzle (the epilogue's staging layout).
nvfp4_status make_out_map(CUtensorMap *map, void *y, uint64_t m, uint64_t n, uint64_t ldy)
{
    cuuint64_t dims[2] = {n, m};
    cuuint64_t strides[1] = {ldy * 2};
    cuuint32_t box[2] = {64, 128};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, y, dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? NVFP4_OK : NVFP4_ERR_CUDA;
}

nvfp4_status launch_pair(const uint8_t *qx, const uint8_t *sfx, const float *s_x, int64_t m, const uint8_t *qw,
                         const uint8_t *sfw, int64_t n, int64_t k, const int64_t *seg_ends, int nseg,
                         const float *seg_gscales, void *y, int64_t ldy, unsigned flags, int sms,
                         bool early_weights, cudaStream_t stream)
{
    CUtensorMap ta, tb, tsa, tsb, ty;
    memset(&ty, 0, sizeof ty);
    nvfp4_status st = make_map(&ta, qx, static_cast<uint64_t>(k / 2), static_cast<uint64_t>(m), 128);
    if (st == NVFP4_OK && !(flags & NVFP4_FLAG_F32_OUT))
        st = make_out_map(&ty, y, static_cast<uint64_t>(m), static_cast<uint64_t>(n), static_cast<uint64_t>(ldy));
    if (st == NVFP4_OK)
        st = make_map(&tb, qw, static_cast<uint64_t>(k / 2), static_cast<uint64_t>(n), 128);
    if (st == NVFP4_OK)
        st = make_sf_map(&tsa, sfx, static_cast<uint64_t>(k / 64), static_cast<uint64_t>((m + 127) / 128), 1);
    if (st == NVFP4_OK)
        st = make_sf_map(&tsb, sfw, static_cast<uint64_t>(k / 64), static_cast<uint64_t>((n + 127) / 128), 2);
    if (st != NVFP4_OK)
        return st;
    pair::Params p;
    memset(&p, 0, sizeof p);
    p.m = static_cast<int>(m);
    p.n = static_cast<int>(n);
    p.k = static_cast<int>(k);
    p.tiles_m = static_cast<int>((m + pair::BM - 1) / pair::BM);
    p.tiles_n = static_cast<int>((n + pair::BN - 1) / pair::BN);
    // Groups of 16 M tiles once there are at least two such groups (measured:
    // -5% on 8192 x 17408 x 5120; smaller M keeps the plain M-major order).
    p.group_m = p.tiles_m >= 32 ? 16 : 1;
    p.k_stages = static_cast<int>((k + pair::BK - 1) / pair::BK);
    p.y = y;
    p.ldy = ldy;
    p.s_x = s_x;
    p.s_w = seg_gscales;
    p.nseg = nseg;
    for (int s = 0; s < nseg; ++s)
        p.seg_end[s] = static_cast<int>(seg_ends[s]);
    p.flags = flags;
    p.timeout_ns = g_timeout_ns.load();
    p.early_weights = early_weights ? 1 : 0;
    // Testing hooks: withhold the second K stage of each pair's first tile, or
    // the last K stage of each pair's second tile.
    p.stall_tile = -1;
    p.stall_stage = -1;
    if (flags & NVFP4_FLAG_TEST_STALL) {
        p.stall_tile = 0;
        p.stall_stage = 1;
    } else if (flags & NVFP4_FLAG_TEST_STALL_LATE) {
        p.stall_tile = 1;
        p.stall_stage = p.k_stages - 1;
    }
    const int64_t tiles = static_cast<int64_t>(p.tiles_m) * p.tiles_n;
    const int64_t pairs = tiles < sms / 2 ? tiles : sms / 2;
    return cuda_status(launch(pair::nvfp4_gemm_pair_kernel, static_cast<int>(2 * pairs), pair::THREADS,
                              pair::SMEM_ALLOC, stream, true, ta, tb, tsa, tsb, ty, p));
}

// The split decode kernel serves up to this many weight tiles times two (one
// tile per two SMs of a B200's 148).
constexpr int kSplitMaxTilesTimes2 = 148;

template <int T>
nvfp4_status launch_decode(const uint8_t *qx, const uint8_t *sfx, const float *s_x, int64_t m, const uint8_t *qw,
                           const uint8_t *sfw, int64_t n, int64_t k, const int64_t *seg_ends, int nseg,
                           const float *seg_gscales, void *y, int64_t ldy, unsigned flags, bool early_weights,
                           cudaStream_t stream)
{
    CUtensorMap tw, tx;
    nvfp4_status st = make_map(&tw, qw, static_cast<uint64_t>(k / 2), static_cast<uint64_t>(n), decode::BW);
    if (st != NVFP4_OK)
        return st;
    st = make_map(&tx, qx, static_cast<uint64_t>(k / 2), static_cast<uint64_t>(m), T);
    if (st != NVFP4_OK)
        return st;
    decode::Params p;
    memset(&p, 0, sizeof p);
    p.sfw = sfw;
    p.sfx = sfx;
    p.m = static_cast<int>(m);
    p.n = static_cast<int>(n);
    p.k = static_cast<int>(k);
    p.atoms_k = k / 64;
    p.k_stages = static_cast<int>((k + decode::BK - 1) / decode::BK);
    p.y = y;
    p.ldy = ldy;
    p.s_x = s_x;
    p.s_w = seg_gscales;
    p.nseg = nseg;
    for (int s = 0; s < nseg; ++s)
        p.seg_end[s] = static_cast<int>(seg_ends[s]);
    p.flags = flags;
    p.timeout_ns = g_timeout_ns.load();
    // Testing hooks (one tile per CTA): withhold the second or the last K stage.
    p.stall_stage = (flags & NVFP4_FLAG_TEST_STALL) ? 1 : (flags & NVFP4_FLAG_TEST_STALL_LATE) ? p.k_stages - 1 : -1;
    p.early_weights = early_weights ? 1 : 0;
    const int grid = static_cast<int>((n + decode::BW - 1) / decode::BW);
    if constexpr (T <= 32) {
        // Up to 32 tokens, few weight tiles (at most one per two SMs) and a K
        // of at least 8 stages: each tile runs on a cluster of decode::kSplit
        // CTAs, one K range each (gemm_decode_split.cuh).
        if (grid * 2 <= kSplitMaxTilesTimes2 && p.k_stages >= 2 * decode::kSplit) {
            if (flags & NVFP4_FLAG_TEST_STALL_LATE)          // the last stage of each CTA's K range
                p.stall_stage = p.k_stages / decode::kSplit - 1;
            return cuda_status(launch(decode::nvfp4_gemm_decode_split_kernel<T>, grid * decode::kSplit,
                                      decode::THREADS, decode::SplitCfg<T>::SMEM_ALLOC, stream, true, tw, tx, p));
        }
    }
    return cuda_status(launch(decode::nvfp4_gemm_decode_kernel<T>, grid, decode::THREADS, decode::Cfg<T>::SMEM_ALLOC,
                              stream, true, tw, tx, p));
}

// GEMM + epilogue.  Up to 128 tokens take the swapped decode kernel, more take
// the persistent CTA-pair kernel (256 x 256 tiles).  Both are launched with
// programmatic stream serialization and touch no global memory before
// griddepcontrol.wait, except that `early_weights` lets them request their
// first weight stages before it.  It is set when the preceding kernel in the
// stream is this library's quantizer (whose early trigger comes after all
// earlier work has completed), or when the caller passed
// NVFP4_FLAG_STATIC_WEIGHTS (no pending work writes the weights).
nvfp4_status launch_gemm(const uint8_t *qx, const uint8_t *sfx, const float *s_x, int64_t m, const uint8_t *qw,
                         const uint8_t *sfw, int64_t n, int64_t k, const int64_t *seg_ends, int nseg,
                         const float *seg_gscales, void *y, int64_t ldy, unsigned flags, int sms, bool early_weights,
                         cudaStream_t stream)
{
    const bool ew = early_weights;
    if (m <= 8)
        return launch_decode<8>(qx, sfx, s_x, m, qw, sfw, n, k, seg_ends, nseg, seg_gscales, y, ldy, flags, ew, stream);
    if (m <= 16)
        return launch_decode<16>(qx, sfx, s_x, m, qw, sfw, n, k, seg_ends, nseg, seg_gscales, y, ldy, flags, ew, stream);
    if (m <= 32)
        return launch_decode<32>(qx, sfx, s_x, m, qw, sfw, n, k, seg_ends, nseg, seg_gscales, y, ldy, flags, ew, stream);
    if (m <= 64)
        return launch_decode<64>(qx, sfx, s_x, m, qw, sfw, n, k, seg_ends, nseg, seg_gscales, y, ldy, flags, ew, stream);
    // 65..128 tokens: the weight stream still bounds the GEMM, which the swapped
    // kernel serves better than 256-row pair tiles (N = 34816, K = 5120: M = 128
    // measured 25.3 us on the pair kernel).
    if (m <= 128)
        return launch_decode<128>(qx, sfx, s_x, m, qw, sfw, n, k, seg_ends, nseg, seg_gscales, y, ldy, flags, ew,
                                  stream);
    return launch_pair(qx, sfx, s_x, m, qw, sfw, n, k, seg_ends, nseg, seg_gscales, y, ldy, flags, sms, ew, stream);
}

struct WorkspaceLayout {
    size_t q_off, sf_off, scale_off, total;
};

WorkspaceLayout workspace_layout(int64_t m, int64_t k)
{
    WorkspaceLayout w;
    w.q_off = kPartialBytes;
    w.sf_off = align_up(w.q_off + static_cast<size_t>(m) * static_cast<size_t>(k / 2), kAlign);
    w.scale_off = align_up(w.sf_off + nvfp4_sf_bytes(m, k), kAlign);
    w.total = w.scale_off + kAlign;
    return w;
}

nvfp4_status check_gemm_args(const uint8_t *qx, const uint8_t *sfx, const float *s_x, int64_t m, const uint8_t *qw,
                             const uint8_t *sfw, int64_t n, int64_t k, const float *seg_gscales, const void *y,
                             int64_t ldy, unsigned flags)
{
    if (m < 0 || n <= 0 || k <= 0)
        return NVFP4_ERR_INVALID_ARG;
    if (flags & ~(NVFP4_FLAG_F32_OUT | NVFP4_FLAG_COLLAPSED_MAX_SCALE | NVFP4_FLAG_STATIC_WEIGHTS |
                  NVFP4_FLAG_TEST_STALL | NVFP4_FLAG_TEST_STALL_LATE))
        return NVFP4_ERR_INVALID_ARG;
    if (k % 64 != 0 || n % 8 != 0)
        return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (m > (int64_t(1) << 31) - 256 || n > (int64_t(1) << 31) - 256 || k > (int64_t(1) << 30))
        return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (qw == nullptr || sfw == nullptr || seg_gscales == nullptr)
        return NVFP4_ERR_INVALID_ARG;
    if (m > 0 && (qx == nullptr || sfx == nullptr || s_x == nullptr || y == nullptr))
        return NVFP4_ERR_INVALID_ARG;
    if (ldy < n)
        return NVFP4_ERR_INVALID_ARG;
    const int64_t esz = (flags & NVFP4_FLAG_F32_OUT) ? 4 : 2;
    if (!aligned16(qx) || !aligned16(sfx) || !aligned16(qw) || !aligned16(sfw) || !aligned16(y) ||
        (ldy * esz) % 16 != 0)
        return NVFP4_ERR_MISALIGNED;
    return NVFP4_OK;
}

}  // namespace

extern "C" {

const char *nvfp4_status_string(nvfp4_status st)
{
    switch (st) {
    case NVFP4_OK: return "ok";
    case NVFP4_ERR_INVALID_ARG: return "invalid argument";
    case NVFP4_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case NVFP4_ERR_MISALIGNED: return "misaligned pointer or stride";
    case NVFP4_ERR_NONFINITE: return "non-finite global scale";
    case NVFP4_ERR_CUDA: return "CUDA error";
    case NVFP4_ERR_TIMEOUT: return "pipeline wait timed out";
    case NVFP4_ERR_WORKSPACE: return "workspace missing or too small";
    case NVFP4_ERR_UNSUPPORTED_DEVICE: return "device is not sm_100";
    case NVFP4_ERR_SCRATCH_LIMIT: return "problem exceeds the static scratch of nvfp4_linear_fused_noalloc";
    }
    return "unknown status";
}

const char *nvfp4_version(void) { return "nvfp4-b200 0.1"; }

size_t nvfp4_sf_bytes(int64_t rows, int64_t k)
{
    if (rows < 0 || k <= 0 || k % 16 != 0)
        return 0;
    const size_t rows_pad = static_cast<size_t>((rows + 127) / 128 * 128);
    const size_t cols_pad = static_cast<size_t>(((k / 16) + 3) / 4 * 4);
    return rows_pad * cols_pad;
}

size_t nvfp4_workspace_bytes(int64_t m, int64_t n, int64_t k)
{
    (void)n;
    if (m < 0 || k <= 0 || k % 16 != 0)
        return 0;
    return workspace_layout(m, k).total;
}

void nvfp4_set_wait_timeout_ns(uint64_t ns) { g_timeout_ns.store(ns < 1000 ? 1000 : ns); }

uint64_t nvfp4_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

nvfp4_status nvfp4_quantize_act(const void *x, int64_t m, int64_t k, int64_t ldx, const float *gscale_in,
                                float *gscale_out, uint8_t *q, uint8_t *sf, void *workspace, size_t ws_bytes,
                                nvfp4_stream_t stream)
{
    nvfp4_status st = check_bf16_operand(x, m, k, ldx);
    if (st != NVFP4_OK)
        return st;
    if (gscale_out == nullptr || (m > 0 && (q == nullptr || sf == nullptr)))
        return NVFP4_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(sf))
        return NVFP4_ERR_MISALIGNED;
    if (gscale_in == nullptr && (workspace == nullptr || ws_bytes < kPartialBytes))
        return NVFP4_ERR_WORKSPACE;
    if (m == 0)
        return NVFP4_OK;
    int sms = 0;
    if ((st = device_setup(&sms)) != NVFP4_OK)
        return st;
    int64_t end = m;
    return launch_quantize(x, m, k, ldx, &end, 1, gscale_in, gscale_out, q, sf, static_cast<uint32_t *>(workspace),
                           sms, reinterpret_cast<cudaStream_t>(stream));
}

nvfp4_status nvfp4_pack_weight(const void *w, int64_t n, int64_t k, int64_t ldw, const int64_t *seg_offsets,
                               int nseg, const float *gscale_in, float *gscale_out, uint8_t *q, uint8_t *sf,
                               void *workspace, size_t ws_bytes, nvfp4_stream_t stream)
{
    nvfp4_status st = check_bf16_operand(w, n, k, ldw);
    if (st != NVFP4_OK)
        return st;
    if (n <= 0)
        return NVFP4_ERR_INVALID_ARG;
    int64_t ends[NVFP4_MAX_SEGMENTS];
    if ((st = read_segments(seg_offsets, nseg, n, ends)) != NVFP4_OK)
        return st;
    if (gscale_out == nullptr || q == nullptr || sf == nullptr)
        return NVFP4_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(sf))
        return NVFP4_ERR_MISALIGNED;
    if (gscale_in == nullptr && (workspace == nullptr || ws_bytes < kPartialBytes))
        return NVFP4_ERR_WORKSPACE;
    int sms = 0;
    if ((st = device_setup(&sms)) != NVFP4_OK)
        return st;
    return launch_quantize(w, n, k, ldw, ends, nseg, gscale_in, gscale_out, q, sf,
                           static_cast<uint32_t *>(workspace), sms, reinterpret_cast<cudaStream_t>(stream));
}

nvfp4_status nvfp4_gemm(const uint8_t *qx, const uint8_t *sfx, const float *s_x, int64_t m, const uint8_t *qw,
                        const uint8_t *sfw, int64_t n, int64_t k, const int64_t *seg_offsets,
                        const float *seg_gscales, int nseg, void *y, int64_t ldy, unsigned flags,
                        nvfp4_stream_t stream)
{
    nvfp4_status st = check_gemm_args(qx, sfx, s_x, m, qw, sfw, n, k, seg_gscales, y, ldy, flags);
    if (st != NVFP4_OK)
        return st;
    int64_t ends[NVFP4_MAX_SEGMENTS];
    if ((st = read_segments(seg_offsets, nseg, n, ends)) != NVFP4_OK)
        return st;
    if (m == 0)
        return NVFP4_OK;
    int sms = 0;
    if ((st = device_setup(&sms)) != NVFP4_OK)
        return st;
    return launch_gemm(qx, sfx, s_x, m, qw, sfw, n, k, ends, nseg, seg_gscales, y, ldy, flags, sms,
                       (flags & NVFP4_FLAG_STATIC_WEIGHTS) != 0, reinterpret_cast<cudaStream_t>(stream));
}

nvfp4_status nvfp4_linear_fused(const void *x, int64_t m, int64_t k, int64_t ldx, const float *act_gscale,
                                const uint8_t *qw, const uint8_t *sfw, int64_t n, const int64_t *seg_offsets,
                                const float *seg_gscales, int nseg, void *y, int64_t ldy, unsigned flags,
                                void *workspace, size_t ws_bytes, nvfp4_stream_t stream)
{
    nvfp4_status st = check_bf16_operand(x, m, k, ldx);
    if (st != NVFP4_OK)
        return st;
    const WorkspaceLayout wl = workspace_layout(m, k);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    // The GEMM's activation operands come from the workspace (the scale slot
    // stands in for s_x: a NULL act_gscale selects the dynamic scale).
    st = check_gemm_args(ws + wl.q_off, ws + wl.sf_off, reinterpret_cast<const float *>(ws + wl.scale_off), m, qw,
                         sfw, n, k, seg_gscales, y, ldy, flags);
    if (st != NVFP4_OK)
        return st;
    int64_t ends[NVFP4_MAX_SEGMENTS];
    if ((st = read_segments(seg_offsets, nseg, n, ends)) != NVFP4_OK)
        return st;
    if (m == 0)
        return NVFP4_OK;
    if (workspace == nullptr || ws_bytes < wl.total || !aligned16(workspace))
        return NVFP4_ERR_WORKSPACE;
    int sms = 0;
    if ((st = device_setup(&sms)) != NVFP4_OK)
        return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    float *sx = reinterpret_cast<float *>(ws + wl.scale_off);
    int64_t end = m;
    st = launch_quantize(x, m, k, ldx, &end, 1, act_gscale, sx, ws + wl.q_off, ws + wl.sf_off,
                         reinterpret_cast<uint32_t *>(ws), sms, s);
    if (st != NVFP4_OK)
        return st;
    return launch_gemm(ws + wl.q_off, ws + wl.sf_off, sx, m, qw, sfw, n, k, ends, nseg, seg_gscales, y, ldy, flags,
                       sms, true, s);
}

nvfp4_status nvfp4_linear(const void *x, int64_t m, int64_t k, int64_t ldx, const float *act_gscale,
                          const uint8_t *qw, const uint8_t *sfw, const float *w_gscale, int64_t n, void *y,
                          int64_t ldy, unsigned flags, void *workspace, size_t ws_bytes, nvfp4_stream_t stream)
{
    return nvfp4_linear_fused(x, m, k, ldx, act_gscale, qw, sfw, n, nullptr, w_gscale, 1, y, ldy, flags, workspace,
                              ws_bytes, stream);
}

nvfp4_status nvfp4_linear_fused_noalloc(const void *x, int64_t m, int64_t k, int64_t ldx, const float *act_gscale,
                                        const uint8_t *qw, const uint8_t *sfw, int64_t n,
                                        const int64_t *seg_offsets, const float *seg_gscales, int nseg,
                                        void *y, int64_t ldy, unsigned flags, nvfp4_stream_t stream)
{
    // The shape is validated first, so a malformed call gets the same status as
    // from nvfp4_linear_fused; only a well-formed problem too large for the
    // scratch array gets NVFP4_ERR_SCRATCH_LIMIT.
    nvfp4_status st = check_bf16_operand(x, m, k, ldx);
    if (st != NVFP4_OK)
        return st;
    if (workspace_layout(m, k).total > NVFP4_NOALLOC_SCRATCH_BYTES)
        return NVFP4_ERR_SCRATCH_LIMIT;
    // Per-device look-up of the scratch array's device address, made with that
    // device current, once per context (again after a cudaDeviceReset).
    static void *scratch[64] = {};
    static unsigned long long scratch_ctx[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return NVFP4_ERR_CUDA;
    void *ptr = nullptr;
    {
        std::lock_guard<std::mutex> lock(g_mu);
        unsigned long long ctx_id = 0;
        if (current_context_id(dev, &ctx_id) != NVFP4_OK)
            return NVFP4_ERR_CUDA;
        if (scratch[dev] == nullptr || scratch_ctx[dev] != ctx_id) {
            void *p = nullptr;
            if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
                return NVFP4_ERR_CUDA;
            scratch[dev] = p;
            scratch_ctx[dev] = ctx_id;
        }
        ptr = scratch[dev];
    }
    return nvfp4_linear_fused(x, m, k, ldx, act_gscale, qw, sfw, n, seg_offsets, seg_gscales, nseg, y, ldy, flags,
                              ptr, NVFP4_NOALLOC_SCRATCH_BYTES, stream);
}

nvfp4_status nvfp4_dequantize(const uint8_t *q, const uint8_t *sf, int64_t rows, int64_t k,
                              const int64_t *seg_offsets, const float *seg_gscales, int nseg, void *y, int64_t ldy,
                              nvfp4_stream_t stream)
{
    if (rows < 0 || k <= 0 || ldy < k)
        return NVFP4_ERR_INVALID_ARG;
    if (k % 64 != 0 || rows > (int64_t(1) << 31) || k > (int64_t(1) << 30))
        return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (rows == 0)
        return seg_offsets == nullptr && nseg == 1 ? NVFP4_OK : NVFP4_ERR_INVALID_ARG;
    int64_t ends[NVFP4_MAX_SEGMENTS];
    nvfp4_status st = read_segments(seg_offsets, nseg, rows, ends);
    if (st != NVFP4_OK)
        return st;
    if (q == nullptr || sf == nullptr || seg_gscales == nullptr || y == nullptr)
        return NVFP4_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(sf) || !aligned16(y) || (ldy * 2) % 16 != 0)
        return NVFP4_ERR_MISALIGNED;
    int sms = 0;
    if ((st = device_setup(&sms)) != NVFP4_OK)
        return st;
    convert::ExpandParams ep;
    memset(&ep, 0, sizeof ep);
    ep.q = q;
    ep.sf = sf;
    ep.y = static_cast<uint16_t *>(y);
    ep.rows = rows;
    ep.k = k;
    ep.ldy = ldy;
    ep.row_tiles = (rows + 127) / 128;
    ep.col_tiles = k / 64;
    ep.nseg = nseg;
    for (int i = 0; i < nseg; ++i)
        ep.seg_end[i] = ends[i];
    ep.gscale = seg_gscales;
    const int64_t tiles = ep.row_tiles * ep.col_tiles;
    const int grid = static_cast<int>(tiles < g_expand_ctas ? tiles : g_expand_ctas);
    return cuda_status(launch(convert::expand_kernel, grid, convert::kThreads, 0,
                              reinterpret_cast<cudaStream_t>(stream), false, ep));
}

nvfp4_status nvfp4_import_weight_scales(const uint8_t *sf_linear, int64_t n, int64_t k, int64_t ld_sf,
                                        uint8_t *sf_out, nvfp4_stream_t stream)
{
    if (n < 0 || k <= 0 || ld_sf < k / 16)
        return NVFP4_ERR_INVALID_ARG;
    if (k % 64 != 0 || n > (int64_t(1) << 31) || k > (int64_t(1) << 30))
        return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (n == 0)
        return NVFP4_OK;
    if (sf_linear == nullptr || sf_out == nullptr)
        return NVFP4_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(sf_linear) & 3u) != 0 || ld_sf % 4 != 0 || !aligned16(sf_out))
        return NVFP4_ERR_MISALIGNED;
    const uintptr_t in0 = reinterpret_cast<uintptr_t>(sf_linear);
    const uintptr_t in1 = in0 + static_cast<uintptr_t>((n - 1) * ld_sf + k / 16);
    const uintptr_t out0 = reinterpret_cast<uintptr_t>(sf_out);
    const uintptr_t out1 = out0 + nvfp4_sf_bytes(n, k);
    if (in0 < out1 && out0 < in1)
        return NVFP4_ERR_INVALID_ARG;        // the layouts differ, so no in-place import
    int sms = 0;
    nvfp4_status st = device_setup(&sms);
    if (st != NVFP4_OK)
        return st;
    convert::ImportParams ip;
    memset(&ip, 0, sizeof ip);
    ip.lin = sf_linear;
    ip.sf = sf_out;
    ip.rows = n;
    ip.ld = ld_sf;
    ip.row_tiles = (n + 127) / 128;
    ip.atoms_k = k / 64;
    ip.col_groups = (ip.atoms_k + 15) / 16;
    const int64_t tiles = ip.row_tiles * ip.col_groups;
    const int64_t cap = static_cast<int64_t>(sms) * 8;
    const int grid = static_cast<int>(tiles < cap ? tiles : cap);
    return cuda_status(launch(convert::import_scales_kernel, grid, convert::kThreads, 0,
                              reinterpret_cast<cudaStream_t>(stream), false, ip));
}

nvfp4_status nvfp4_harmonize_scales(const uint8_t *sf_in, uint8_t *sf_out, int64_t n, int64_t k,
                                    const int64_t *seg_offsets, const float *seg_gscales, int nseg,
                                    float *shared_gscale_out, nvfp4_stream_t stream)
{
    if (n <= 0 || k <= 0)
        return NVFP4_ERR_INVALID_ARG;
    if (k % 64 != 0 || n > (int64_t(1) << 31) || k > (int64_t(1) << 30))
        return NVFP4_ERR_UNSUPPORTED_SHAPE;
    int64_t ends[NVFP4_MAX_SEGMENTS];
    nvfp4_status st = read_segments(seg_offsets, nseg, n, ends);
    if (st != NVFP4_OK)
        return st;
    if (sf_in == nullptr || sf_out == nullptr || seg_gscales == nullptr || shared_gscale_out == nullptr)
        return NVFP4_ERR_INVALID_ARG;
    if (!aligned16(sf_in) || !aligned16(sf_out))
        return NVFP4_ERR_MISALIGNED;
    const size_t bytes = nvfp4_sf_bytes(n, k);
    const uintptr_t a = reinterpret_cast<uintptr_t>(sf_in), b = reinterpret_cast<uintptr_t>(sf_out);
    if (a != b && a < b + bytes && b < a + bytes)
        return NVFP4_ERR_INVALID_ARG;        // partial overlap
    int sms = 0;
    if ((st = device_setup(&sms)) != NVFP4_OK)
        return st;
    convert::HarmonizeParams hp;
    memset(&hp, 0, sizeof hp);
    hp.sf_in = sf_in;
    hp.sf_out = sf_out;
    hp.rows = n;
    hp.atoms_k = k / 64;
    hp.units = static_cast<int64_t>(bytes / 16);
    hp.nseg = nseg;
    for (int i = 0; i < nseg; ++i)
        hp.seg_end[i] = ends[i];
    hp.gscale = seg_gscales;
    hp.shared_out = shared_gscale_out;
    const int64_t blocks = (hp.units + convert::kThreads - 1) / convert::kThreads;
    const int64_t cap = static_cast<int64_t>(sms) * 8;
    const int grid = static_cast<int>(blocks < cap ? blocks : cap);
    return cuda_status(launch(convert::harmonize_kernel, grid, convert::kThreads, 0,
                              reinterpret_cast<cudaStream_t>(stream), false, hp));
}

nvfp4_status nvfp4_mma_peak_probe(int pairs, int64_t iters, int with_scale_copies, double *flops,
                                  nvfp4_stream_t stream)
{
    if (pairs < 1 || iters < 1 || iters > (int64_t(1) << 40) || flops == nullptr)
        return NVFP4_ERR_INVALID_ARG;
    int sms = 0;
    nvfp4_status st = device_setup(&sms);
    if (st != NVFP4_OK)
        return st;
    if (pairs > sms / 2)
        return NVFP4_ERR_UNSUPPORTED_SHAPE;
    st = cuda_status(launch(peak::mma_peak_kernel, 2 * pairs, peak::THREADS, peak::SMEM_ALLOC,
                            reinterpret_cast<cudaStream_t>(stream), false, iters, with_scale_copies ? 1 : 0));
    if (st == NVFP4_OK)
        *flops = 2.0 * 256.0 * 256.0 * 64.0 * peak::KB * static_cast<double>(iters) * pairs;
    return st;
}

nvfp4_status nvfp4_get_device_error(nvfp4_stream_t stream)
{
    if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
        return NVFP4_ERR_CUDA;
    unsigned int v = 0;
    if (cudaMemcpyFromSymbol(&v, nvfp4::g_device_error, sizeof v) != cudaSuccess)
        return NVFP4_ERR_CUDA;
    if (v != 0) {
        const unsigned int zero = 0;
        if (cudaMemcpyToSymbol(nvfp4::g_device_error, &zero, sizeof zero) != cudaSuccess)
            return NVFP4_ERR_CUDA;
    }
    return static_cast<nvfp4_status>(v);
}

}  // extern "C"
