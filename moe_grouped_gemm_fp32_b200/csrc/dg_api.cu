// dg_api.cu -- host side of the C ABI declared in include/dg.h: argument
// validation, TMA descriptor encoding, tile-configuration choice and kernel
// launch.  Nothing here synchronises the host (except dg_get_device_status)
// or allocates memory.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdio>
#include <cstdlib>
#include <atomic>
#include <cstring>
#include <mutex>

#include "dg.h"
#include "api_common.h"
#include "gemm_kernel.cuh"

namespace {
__device__ unsigned g_dg_status = 0u;
thread_local char t_last_cuda_error[256] = "";
int g_debug_flags = 0;
}  // namespace

namespace dg_host {

dg_status_t cuda_fail(cudaError_t e, const char *what) {
    std::snprintf(t_last_cuda_error, sizeof(t_last_cuda_error), "%s: %s", what,
                  cudaGetErrorString(e));
    return DG_ERR_CUDA;
}

int debug_flags() { return g_debug_flags; }

bool verbose() {
    static bool v = [] {
        const char *s = std::getenv("DG_VERBOSE");
        return s && s[0] == '1';
    }();
    return v;
}

// ------------------------------------------------------------------ device info
namespace {
DeviceInfo g_devices[kMaxDevices];
std::mutex g_mutex;
}  // namespace

dg_status_t device_info(const DeviceInfo **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return DG_ERR_UNSUPPORTED_DEVICE;
    }
    if (dev < 0 || dev >= kMaxDevices) return DG_ERR_UNSUPPORTED_DEVICE;
    std::lock_guard<std::mutex> lock(g_mutex);
    DeviceInfo &info = g_devices[dev];
    if (!info.ready) {
        int major = 0, minor = 0, sms = 0;
        if ((e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess ||
            (e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess ||
            (e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
            return cuda_fail(e, "cudaDeviceGetAttribute");
        info.supported = (major == 10 && minor == 0);
        info.num_sms = sms;
        if (info.supported) {
            void *addr = nullptr;
            if ((e = cudaGetSymbolAddress(&addr, g_dg_status)) != cudaSuccess)
                return cuda_fail(e, "cudaGetSymbolAddress(status)");
            info.status = static_cast<unsigned *>(addr);
        }
        info.ready = true;
    }
    if (!info.supported) return DG_ERR_UNSUPPORTED_DEVICE;
    *out = &info;
    return DG_SUCCESS;
}

}  // namespace dg_host

namespace {
using namespace dg_host;

// ------------------------------------------------------------------ tensor maps
using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
        else
            cudaGetLastError();
    });
    return fn;
}

}  // namespace

namespace dg_host {

dg_status_t make_kmajor_map(CUtensorMap *m, const void *base, int elem_bytes, long long K,
                            long long rows, long long groups, int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) {
        std::snprintf(t_last_cuda_error, sizeof(t_last_cuda_error),
                      "cuTensorMapEncodeTiled entry point unavailable");
        return DG_ERR_CUDA;
    }
    const cuuint64_t eb = static_cast<cuuint64_t>(elem_bytes);
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(rows),
                          static_cast<cuuint64_t>(groups)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(K) * eb, static_cast<cuuint64_t>(K * rows) * eb};
    cuuint32_t box[3] = {static_cast<cuuint32_t>(128 / elem_bytes), static_cast<cuuint32_t>(box_rows), 1};
    cuuint32_t estr[3] = {1, 1, 1};
    const CUtensorMapDataType dt = elem_bytes == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                   : CU_TENSOR_MAP_DATA_TYPE_UINT8;
    CUresult r = fn(m, dt, 3, const_cast<void *>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        std::snprintf(t_last_cuda_error, sizeof(t_last_cuda_error),
                      "cuTensorMapEncodeTiled failed (CUresult %d)", static_cast<int>(r));
        return DG_ERR_CUDA;
    }
    return DG_SUCCESS;
}

long long timeout_cycles() {
    static long long v = [] {
        const char *s = std::getenv("DG_WAIT_TIMEOUT_CYCLES");
        long long x = s ? std::atoll(s) : 0;
        return x > 0 ? x : (1LL << 32);   // ~2 s at 2 GHz; legitimate waits are micro- to milliseconds
    }();
    return v;
}

}  // namespace dg_host

namespace {
using namespace dg_host;

// D as a 2-D BF16 tensor {N, rows} (masked / K-grouped: all groups' rows
// stacked), box {32 columns, box_rows rows} with 64-byte swizzle: the TMA-store
// epilogue's box (32 rows per warp; CTA pairs store 128-row boxes of a staged tile).  A null d (no BF16 output) gives an all-zero map the kernel
// never uses.
dg_status_t make_d_map(CUtensorMap *m, void *d, long long N, long long rows, int box_rows = 32) {
    std::memset(m, 0, sizeof(*m));
    if (!d || rows <= 0) return DG_SUCCESS;
    EncodeTiledFn fn = encode_fn();
    if (!fn) {
        std::snprintf(t_last_cuda_error, sizeof(t_last_cuda_error),
                      "cuTensorMapEncodeTiled entry point unavailable");
        return DG_ERR_CUDA;
    }
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(N) * 2};
    cuuint32_t box[2] = {32, static_cast<cuuint32_t>(box_rows)};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, d, dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                    CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        std::snprintf(t_last_cuda_error, sizeof(t_last_cuda_error),
                      "cuTensorMapEncodeTiled (D) failed (CUresult %d)", static_cast<int>(r));
        return DG_ERR_CUDA;
    }
    return DG_SUCCESS;
}

// 3-D uint8 tensor {K, rows, groups} (K innermost), box {128, box_rows, 1},
// 128-byte swizzle, zero fill out of bounds.
dg_status_t make_map(CUtensorMap *m, const void *base, long long K, long long rows,
                     long long groups, int box_rows) {
    return make_kmajor_map(m, base, 1, K, rows, groups, box_rows);
}

// Row count of the D map's TMA-store box for a kernel instantiation: CTA-pair
// kernels that stage the whole tile store 128-row boxes, the others 32 rows per warp.
template <int kBN, int kStages, int kCtaGroup>
constexpr int d_box_rows() {
    return dg::SmemLayout<kBN, false, kStages, kCtaGroup>::kTileStaging ? dg::kTileX : 32;
}

// ------------------------------------------------------------------ validation
dg_status_t check_common(const void *a, const float *sfa, int ld_sfa, const void *b,
                         const float *sfb, const void *d, int rows, int N, int K) {
    if (!a || !sfa || !b || !sfb || !d) return DG_ERR_INVALID_VALUE;
    if (rows < 0 || N <= 0 || K <= 0) return DG_ERR_INVALID_VALUE;
    if (K % dg::kBlockK != 0 || N % 16 != 0) return DG_ERR_UNSUPPORTED_SHAPE;
    if (ld_sfa < rows || ld_sfa <= 0) return DG_ERR_INVALID_VALUE;
    if (ld_sfa % 4 != 0) return DG_ERR_MISALIGNED;
    if (!aligned16(a) || !aligned16(b) || !aligned16(d) || !aligned16(sfa) || !aligned16(sfb))
        return DG_ERR_MISALIGNED;
    // TMA coordinates and element offsets stay within 32-bit ranges
    if (static_cast<long long>(K) > (1LL << 30) || N > (1 << 30)) return DG_ERR_UNSUPPORTED_SHAPE;
    return DG_SUCCESS;
}

// ------------------------------------------------------------------ launch
template <int kBN, bool kSwap, int kStages, int kLayout, int kCtaGroup = 1, bool kSwiGLU = false>
dg_status_t launch(const CUtensorMap &ma, const CUtensorMap &mb, const CUtensorMap &md, const dg::Params &p,
                   int grid_x, int grid_y, int cluster_x, cudaStream_t stream) {
    using L = dg::SmemLayout<kBN, kSwap, kStages, kCtaGroup, kSwap && kLayout == dg::kDense && kBN <= 128>;
    auto kernel = dg::fp8_gemm_kernel<kBN, kSwap, kStages, kLayout, kCtaGroup, kSwiGLU>;
    // one-time per-device set-up; it is idempotent, so two threads that race on
    // the first call both do it and the atomic flag keeps the access defined
    static std::atomic<bool> attr_done[kMaxDevices] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (!attr_done[dev].load(std::memory_order_acquire)) {
        cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             L::kAlloc);
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
        if (!kSwap) {
            // The register rebalancing inside the kernel (setmaxnreg) is sized for
            // exactly kRegsLaunch registers per thread at launch; with any other
            // count the promotion warps' request could never be granted.  Refuse.
            cudaFuncAttributes fa;
            if ((e = cudaFuncGetAttributes(&fa, kernel)) != cudaSuccess)
                return cuda_fail(e, "cudaFuncGetAttributes");
            if (fa.numRegs != dg::kRegsLaunch) {
                std::snprintf(t_last_cuda_error, sizeof(t_last_cuda_error),
                              "kernel built with %d registers per thread, expected %d", fa.numRegs,
                              dg::kRegsLaunch);
                return DG_ERR_CUDA;
            }
        }
        attr_done[dev].store(true, std::memory_order_release);
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid_x, grid_y, 1);
    cfg.blockDim = dim3(dg::num_threads(kSwap), 1, 1);
    cfg.dynamicSmemBytes = L::kAlloc;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    cfg.attrs = attr;
    cfg.numAttrs = 0;
    if (cluster_x > 1) {
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = cluster_x;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.numAttrs = 1;
    }
    if (verbose())
        std::fprintf(stderr,
                     "[dg] layout=%d M=%d N=%d K=%d G=%d tile_n=%d swap=%d stages=%d ctas/mma=%d "
                     "split=%d grid=%dx%d cluster=%d smem=%d\n",
                     kLayout, p.M, p.N, p.K, p.G, kBN, int(kSwap), kStages, kCtaGroup, p.split, grid_x,
                     grid_y, cluster_x, L::kAlloc);
    cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, ma, mb, md, p);
    if (e != cudaSuccess) return cuda_fail(e, "cudaLaunchKernelEx");
    return DG_SUCCESS;
}

// How many clusters of `cluster_x` CTAs of this kernel can be resident at once
// (cached per device and cluster size).  0 if the query fails.
template <int kBN, bool kSwap, int kStages, int kLayout, int kCtaGroup = 1>
int max_active_clusters(int cluster_x) {
    using L = dg::SmemLayout<kBN, kSwap, kStages, kCtaGroup, kSwap && kLayout == dg::kDense && kBN <= 128>;
    auto kernel = dg::fp8_gemm_kernel<kBN, kSwap, kStages, kLayout, kCtaGroup>;
    // per-device cache of an idempotent query (atomic: concurrent first calls are defined)
    static std::atomic<int> cache[kMaxDevices][9] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (cluster_x < 1 || cluster_x > 8) return 0;
    if (const int c = cache[dev][cluster_x].load(std::memory_order_relaxed)) return c;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc) !=
        cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(cluster_x, 1, 1);
    cfg.blockDim = dim3(dg::num_threads(kSwap), 1, 1);
    cfg.dynamicSmemBytes = L::kAlloc;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = cluster_x;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kernel, &cfg) != cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    cache[dev][cluster_x].store(n, std::memory_order_relaxed);
    return n;
}

// Split-K factor for swap-mode tiles: the largest split <= 8 such that every
// cluster of the grid is resident at once (one wave), each CTA keeps at least
// four K-blocks, and the CTAs fit on the SMs.  The cluster exchange costs about
// 3 us, more than streaming a few K-blocks saves: 128 x 256 x 512 ran 7.9 us
// per call unsplit against 9.1 us split in two.  DG_SPLIT_K overrides it (tuning).
template <int kBN, int kStages, int kLayout>
int choose_split(int tiles, int num_kb, int num_sms) {
    static int forced = [] {
        const char *s = std::getenv("DG_SPLIT_K");
        return s ? std::atoi(s) : 0;
    }();
    if (forced >= 1 && forced <= 8) return num_kb >= 2 * forced ? forced : 1;
    for (int split = 8; split >= 2; --split) {
        if (tiles * split > num_sms || num_kb < 4 * split) continue;
        if (max_active_clusters<kBN, true, kStages, kLayout>(split) >= tiles) return split;
    }
    return 1;
}

// Efficiency of a pair-tile width: the share of the tiles' columns that are
// real (N tail) times how full the waves of resident pairs are.
double pair_efficiency(long long rows_pairs, int N, int bn, int pairs_max) {
    if (pairs_max <= 0) return 0.0;
    const long long nt = (N + bn - 1) / bn;
    const long long tiles = rows_pairs * nt;
    const long long waves = (tiles + pairs_max - 1) / pairs_max;
    return (static_cast<double>(N) / (nt * bn)) * (static_cast<double>(tiles) / (waves * pairs_max));
}

dg::Params base_params(const float *sfa, int ld_sfa, const float *sfb, void *d, int rows, int N,
                       int K, int G, const DeviceInfo *info) {
    dg::Params p = {};
    p.sfa = sfa;
    p.sfb = sfb;
    p.d = static_cast<__nv_bfloat16 *>(d);
    p.status = info->status;
    p.timeout_cycles = timeout_cycles();
    p.ld_sfa = ld_sfa;
    p.M = rows;
    p.N = N;
    p.K = K;
    p.G = G;
    p.num_kb = K / dg::kBlockK;
    p.num_nb = (N + 127) / 128;
    p.split = 1;
    p.debug_flags = g_debug_flags;
    return p;
}



}  // namespace

// ==================================================================== C ABI
extern "C" {

dg_status_t dg_fp8_gemm_nt(const uint8_t *a, const float *sfa, int ld_sfa, const uint8_t *b,
                           const float *sfb, void *d, int M, int N, int K, void *stream) {
    dg_status_t st = check_common(a, sfa, ld_sfa, b, sfb, d, M, N, K);
    if (st != DG_SUCCESS) return st;
    const DeviceInfo *info = nullptr;
    if ((st = device_info(&info)) != DG_SUCCESS) return st;
    if (M == 0) return DG_SUCCESS;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    dg::Params p = base_params(sfa, ld_sfa, sfb, d, M, N, K, 1, info);
    CUtensorMap ma, mb;
    CUtensorMap md;
    if ((st = make_d_map(&md, d, N, M)) != DG_SUCCESS) return st;
    if (M <= 256) {
        // swap-AB: weights on the 128 TMEM lanes, the few tokens on the MMA's N side
        const int bn = M <= 64 ? 64 : (M <= 128 ? 128 : 256);
        const int tiles = ((N + 127) / 128) * ((M + bn - 1) / bn);
        p.split = bn == 64    ? choose_split<64, 7, dg::kDense>(tiles, p.num_kb, info->num_sms)
                  : bn == 128 ? choose_split<128, 4, dg::kDense>(tiles, p.num_kb, info->num_sms)
                              : 1;   // 256-token tiles run persistent (no split-K buffer)
        if ((st = make_map(&mb, b, K, N, 1, 128)) != DG_SUCCESS) return st;
        if ((st = make_map(&ma, a, K, M, 1, 32)) != DG_SUCCESS) return st;   // 32-token boxes
        const int gx = p.split > 1 ? p.split : (tiles < info->num_sms ? tiles : info->num_sms);
        const int gy = p.split > 1 ? tiles : 1;
        if (bn == 64) return launch<64, true, 7, dg::kDense>(ma, mb, md, p, gx, gy, p.split, s);
        if (bn == 128) return launch<128, true, 4, dg::kDense>(ma, mb, md, p, gx, gy, p.split, s);
        return launch<256, true, 4, dg::kDense>(ma, mb, md, p, gx, gy, p.split, s);
    }
    if (N <= 128) {
        const int tiles = ((M + 127) / 128) * ((N + 127) / 128);
        const int grid = tiles < info->num_sms ? tiles : info->num_sms;
        if ((st = make_map(&ma, a, K, M, 1, 128)) != DG_SUCCESS) return st;
        if ((st = make_map(&mb, b, K, N, 1, 128)) != DG_SUCCESS) return st;
        return launch<128, false, 6, dg::kDense>(ma, mb, md, p, grid, 1, 1, s);
    }
    // CTA pairs: 256 x bn tiles with tcgen05.mma.cta_group::2 (DG_PAIR_N =
    // 128 / 160 / 224 / 256 overrides bn for tuning sweeps)
    static const int forced_bn = [] {
        const char *e = std::getenv("DG_PAIR_N");
        return e ? std::atoi(e) : 0;
    }();
    const long long row_pairs = (M + 255) / 256;
    const int pm224 = max_active_clusters<224, false, 5, dg::kDense, 2>(2);
    const int pm256 = max_active_clusters<256, false, 6, dg::kDense, 2>(2);
    int bn = pair_efficiency(row_pairs, N, 224, pm224) > pair_efficiency(row_pairs, N, 256, pm256) + 1e-9
                 ? 224 : 256;
    if (forced_bn == 128 || forced_bn == 160 || forced_bn == 224 || forced_bn == 256) bn = forced_bn;
    const int pairs_max = bn == 128   ? max_active_clusters<128, false, 7, dg::kDense, 2>(2)
                          : bn == 160 ? max_active_clusters<160, false, 6, dg::kDense, 2>(2)
                          : bn == 224 ? pm224 : pm256;
    if (pairs_max <= 0) return cuda_fail(cudaErrorInvalidConfiguration, "no resident CTA pair");
    const int tiles = ((M + 255) / 256) * ((N + bn - 1) / bn);
    const int pairs = tiles < pairs_max ? tiles : pairs_max;
    {
        const int box = bn == 128 ? d_box_rows<128, 7, 2>() : bn == 160 ? d_box_rows<160, 6, 2>()
                        : bn == 224 ? d_box_rows<224, 5, 2>() : d_box_rows<256, 6, 2>();
        if ((st = make_d_map(&md, d, N, M, box)) != DG_SUCCESS) return st;
    }
    if ((st = make_map(&ma, a, K, M, 1, 128)) != DG_SUCCESS) return st;
    if ((st = make_map(&mb, b, K, N, 1, bn / 2)) != DG_SUCCESS) return st;
    if (bn == 128) return launch<128, false, 7, dg::kDense, 2>(ma, mb, md, p, 2 * pairs, 1, 2, s);
    if (bn == 160) return launch<160, false, 6, dg::kDense, 2>(ma, mb, md, p, 2 * pairs, 1, 2, s);
    if (bn == 224) return launch<224, false, 5, dg::kDense, 2>(ma, mb, md, p, 2 * pairs, 1, 2, s);
    return launch<256, false, 6, dg::kDense, 2>(ma, mb, md, p, 2 * pairs, 1, 2, s);
}

dg_status_t dg_m_grouped_fp8_gemm_nt_contiguous(const uint8_t *a, const float *sfa, int ld_sfa,
                                                const uint8_t *b, const float *sfb, void *d,
                                                const int32_t *m_indices, int M_total, int N,
                                                int K, int G, void *stream) {
    dg_status_t st = check_common(a, sfa, ld_sfa, b, sfb, d, M_total, N, K);
    if (st != DG_SUCCESS) return st;
    if (!m_indices || G <= 0) return DG_ERR_INVALID_VALUE;
    if (M_total % 128 != 0) return DG_ERR_UNSUPPORTED_SHAPE;
    const DeviceInfo *info = nullptr;
    if ((st = device_info(&info)) != DG_SUCCESS) return st;
    if (M_total == 0) return DG_SUCCESS;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    dg::Params p = base_params(sfa, ld_sfa, sfb, d, M_total, N, K, G, info);
    p.m_indices = m_indices;
    CUtensorMap ma, mb;
    CUtensorMap md;
    if ((st = make_d_map(&md, d, N, M_total)) != DG_SUCCESS) return st;
    // CTA pairs (256-row tiles) by default for N > 128 and K >= 4096: with the
    // TMA-store epilogue they measured 997 us against 1018 us for 128 x 256
    // single-CTA tiles on 4 groups x 32768 tokens x N 4096 x K 7168, but were
    // slower with short K (the FFN's down projection, K 2048: fewer K-blocks
    // per tile to amortise the pair's tile switch).  DG_CONTIG_PAIRS=0 / =1
    // forces single-CTA tiles / pairs.
    static const int contig_pairs_env = [] {
        const char *e = std::getenv("DG_CONTIG_PAIRS");
        return e ? (e[0] == '1' ? 1 : 0) : -1;
    }();
    const bool contig_pairs = contig_pairs_env >= 0 ? contig_pairs_env == 1 : K >= 4096;
    if (contig_pairs && N > 128 && G < dg::kMaxGroups) {
        // CTA pairs with 256-row tiles; pairs straddling a group boundary run
        // a second pass (the tile count grows by at most (G-1) x N-tiles)
        const long long row_pairs = (M_total / 128 + 1) / 2;
        const int pm224 = max_active_clusters<224, false, 5, dg::kContiguous, 2>(2);
        const int pm256 = max_active_clusters<256, false, 6, dg::kContiguous, 2>(2);
        const int bn = pair_efficiency(row_pairs, N, 224, pm224) > pair_efficiency(row_pairs, N, 256, pm256) + 1e-9
                           ? 224 : 256;
        const int pairs_max = bn == 224 ? pm224 : pm256;
        if (pairs_max > 0) {
            const long long tiles = row_pairs * ((N + bn - 1) / bn);
            const int pairs = tiles < pairs_max ? static_cast<int>(tiles) : pairs_max;
            const int box = bn == 224 ? d_box_rows<224, 5, 2>() : d_box_rows<256, 6, 2>();
            if ((st = make_d_map(&md, d, N, M_total, box)) != DG_SUCCESS) return st;
            if ((st = make_map(&ma, a, K, M_total, 1, 128)) != DG_SUCCESS) return st;
            if ((st = make_map(&mb, b, K, N, G, bn / 2)) != DG_SUCCESS) return st;
            if (bn == 224) return launch<224, false, 5, dg::kContiguous, 2>(ma, mb, md, p, 2 * pairs, 1, 2, s);
            return launch<256, false, 6, dg::kContiguous, 2>(ma, mb, md, p, 2 * pairs, 1, 2, s);
        }
    }
    const int bn = N <= 128 ? 128 : 256;
    const int tiles = (M_total / 128) * ((N + bn - 1) / bn);
    const int grid = tiles < info->num_sms ? tiles : info->num_sms;
    if ((st = make_map(&ma, a, K, M_total, 1, 128)) != DG_SUCCESS) return st;
    if ((st = make_map(&mb, b, K, N, G, bn)) != DG_SUCCESS) return st;
    if (bn == 128) return launch<128, false, 6, dg::kContiguous>(ma, mb, md, p, grid, 1, 1, s);
    return launch<256, false, 4, dg::kContiguous>(ma, mb, md, p, grid, 1, 1, s);
}

dg_status_t dg_m_grouped_fp8_gemm_nt_masked(const uint8_t *a, const float *sfa, int ld_sfa,
                                            const uint8_t *b, const float *sfb, void *d,
                                            const int32_t *masked_m, int G, int Mmax, int N,
                                            int K, void *stream) {
    dg_status_t st = check_common(a, sfa, ld_sfa, b, sfb, d, Mmax, N, K);
    if (st != DG_SUCCESS) return st;
    if (!masked_m || G <= 0) return DG_ERR_INVALID_VALUE;
    if (G > dg::kMaxGroups) return DG_ERR_UNSUPPORTED_SHAPE;
    // the stacked [G * Mmax] rows of d are addressed by 32-bit tensor-map coordinates
    if (static_cast<long long>(G) * Mmax > (1LL << 31) - 1) return DG_ERR_UNSUPPORTED_SHAPE;
    const DeviceInfo *info = nullptr;
    if ((st = device_info(&info)) != DG_SUCCESS) return st;
    if (Mmax == 0) return DG_SUCCESS;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    dg::Params p = base_params(sfa, ld_sfa, sfb, d, Mmax, N, K, G, info);
    p.masked_m = masked_m;
    CUtensorMap ma, mb;
    CUtensorMap md;
    if ((st = make_d_map(&md, d, N, static_cast<long long>(G) * Mmax)) != DG_SUCCESS) return st;
    const int grid = info->num_sms;   // the tile count lives on the device
    static const bool force_swap = [] {
        const char *e = std::getenv("DG_MASKED_SWAP");
        return e && e[0] == '1';
    }();
    if (force_swap) {
        // swap-AB tiles: 128 weight rows x up to 128 tokens (DG_MASKED_SWAP=1, comparisons)
        const int bn = Mmax <= 64 ? 64 : 128;
        if ((st = make_map(&mb, b, K, N, G, 128)) != DG_SUCCESS) return st;
        if ((st = make_map(&ma, a, K, Mmax, G, 32)) != DG_SUCCESS) return st;   // 32-token boxes
        if (bn == 64) return launch<64, true, 8, dg::kMasked>(ma, mb, md, p, grid, 1, 1, s);
        return launch<128, true, 6, dg::kMasked>(ma, mb, md, p, grid, 1, 1, s);
    }
    // Normal mode: 128 token rows on the TMEM lanes, so each promotion thread's
    // token scale is one register and the weight scale is uniform per 128
    // columns (one FMA per element, no per-column scale traffic).  Groups with
    // fewer than 128 valid rows leave the other lanes idle; the weight stream,
    // which bounds this layout, is read once per token block.
    // DG_MASKED_BN=64|128|256 overrides the tile width (tuning sweeps)
    static const int forced_bn = [] {
        const char *e = std::getenv("DG_MASKED_BN");
        return e ? std::atoi(e) : 0;
    }();
    // 128-wide tiles by default: with a mean of 128 valid rows per group the
    // 256-wide grid ends in a long partial wave (measured 123 us vs 112 us on
    // 16 groups x N 4096); the weight stream is read once either way
    int bn = 128;
    if (forced_bn == 64 || forced_bn == 128 || forced_bn == 256) bn = forced_bn;
    if ((st = make_map(&ma, a, K, Mmax, G, 128)) != DG_SUCCESS) return st;
    if ((st = make_map(&mb, b, K, N, G, bn)) != DG_SUCCESS) return st;
    if (bn == 64) return launch<64, false, 8, dg::kMasked>(ma, mb, md, p, grid, 1, 1, s);
    if (bn == 128) return launch<128, false, 6, dg::kMasked>(ma, mb, md, p, grid, 1, 1, s);
    return launch<256, false, 4, dg::kMasked>(ma, mb, md, p, grid, 1, 1, s);
}

dg_status_t dg_k_grouped_fp8_gemm_nt_contiguous(const uint8_t *a, const float *sfa, int ld_sfa,
                                                const uint8_t *b, const float *sfb, void *d,
                                                const int32_t *ks, int G, int M, int N, int K,
                                                void *stream) {
    dg_status_t st = check_common(a, sfa, ld_sfa, b, sfb, d, M, N, K);
    if (st != DG_SUCCESS) return st;
    if (!ks || G <= 0) return DG_ERR_INVALID_VALUE;
    if (G > dg::kMaxGroups) return DG_ERR_UNSUPPORTED_SHAPE;
    // the stacked [G * M] rows of d are addressed by 32-bit tensor-map coordinates
    if (static_cast<long long>(G) * M > (1LL << 31) - 1) return DG_ERR_UNSUPPORTED_SHAPE;
    const DeviceInfo *info = nullptr;
    if ((st = device_info(&info)) != DG_SUCCESS) return st;
    if (M == 0) return DG_SUCCESS;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    dg::Params p = base_params(sfa, ld_sfa, sfb, d, M, N, K, G, info);
    p.ks = ks;
    CUtensorMap ma, mb;
    CUtensorMap md;
    if ((st = make_d_map(&md, d, N, static_cast<long long>(G) * M)) != DG_SUCCESS) return st;
    if ((st = make_map(&ma, a, K, M, 1, 128)) != DG_SUCCESS) return st;
    // The tile grid does not depend on the group sizes (they only set each
    // tile's K range, read on the device): G x token blocks x weight blocks.
    if (N <= 128 || M <= 128) {
        const int bn = N <= 128 ? 128 : 256;
        const long long tiles = static_cast<long long>(G) * ((M + 127) / 128) * ((N + bn - 1) / bn);
        const int grid = tiles < info->num_sms ? static_cast<int>(tiles) : info->num_sms;
        if ((st = make_map(&mb, b, K, N, 1, bn)) != DG_SUCCESS) return st;
        if (bn == 128) return launch<128, false, 6, dg::kKGrouped>(ma, mb, md, p, grid, 1, 1, s);
        return launch<256, false, 4, dg::kKGrouped>(ma, mb, md, p, grid, 1, 1, s);
    }
    // CTA pairs: 256 x bn tiles (tcgen05.mma.cta_group::2), as for large dense GEMMs
    const long long row_pairs = static_cast<long long>(G) * ((M + 255) / 256);
    const int pm224 = max_active_clusters<224, false, 5, dg::kKGrouped, 2>(2);
    const int pm256 = max_active_clusters<256, false, 6, dg::kKGrouped, 2>(2);
    const int bn = pair_efficiency(row_pairs, N, 224, pm224) > pair_efficiency(row_pairs, N, 256, pm256) + 1e-9
                       ? 224 : 256;
    const int pairs_max = bn == 224 ? pm224 : pm256;
    if (pairs_max <= 0) return cuda_fail(cudaErrorInvalidConfiguration, "no resident CTA pair");
    const long long tiles = row_pairs * ((N + bn - 1) / bn);
    const int pairs = tiles < pairs_max ? static_cast<int>(tiles) : pairs_max;
    const int box = bn == 224 ? d_box_rows<224, 5, 2>() : d_box_rows<256, 6, 2>();
    if ((st = make_d_map(&md, d, N, static_cast<long long>(G) * M, box)) != DG_SUCCESS) return st;
    if ((st = make_map(&mb, b, K, N, 1, bn / 2)) != DG_SUCCESS) return st;
    if (bn == 224) return launch<224, false, 5, dg::kKGrouped, 2>(ma, mb, md, p, 2 * pairs, 1, 2, s);
    return launch<256, false, 6, dg::kKGrouped, 2>(ma, mb, md, p, 2 * pairs, 1, 2, s);
}

dg_status_t dg_m_grouped_fp8_gemm_swiglu_quant_contiguous(
    const uint8_t *a, const float *sfa, int ld_sfa, const uint8_t *b, const float *sfb,
    uint8_t *q_out, float *s_out, int ld_s_out, const int32_t *m_indices, int M_total, int N, int K,
    int G, void *stream) {
    // d is not written in this mode; pass q_out to the common checks in its place
    dg_status_t st = check_common(a, sfa, ld_sfa, b, sfb, q_out, M_total, N, K);
    if (st != DG_SUCCESS) return st;
    if (!m_indices || !s_out || G <= 0) return DG_ERR_INVALID_VALUE;
    if (M_total % 128 != 0 || N % 256 != 0) return DG_ERR_UNSUPPORTED_SHAPE;
    if (ld_s_out < M_total || ld_s_out <= 0) return DG_ERR_INVALID_VALUE;
    if (ld_s_out % 4 != 0 || !aligned16(s_out)) return DG_ERR_MISALIGNED;
    const DeviceInfo *info = nullptr;
    if ((st = device_info(&info)) != DG_SUCCESS) return st;
    if (M_total == 0) return DG_SUCCESS;
    dg::Params p = base_params(sfa, ld_sfa, sfb, nullptr, M_total, N, K, G, info);
    p.m_indices = m_indices;
    p.q_out = q_out;
    p.s_out = s_out;
    p.ld_s_out = ld_s_out;
    CUtensorMap ma, mb;
    CUtensorMap md;
    if ((st = make_d_map(&md, nullptr, N, 0)) != DG_SUCCESS) return st;
    if ((st = make_map(&ma, a, K, M_total, 1, 128)) != DG_SUCCESS) return st;
    if ((st = make_map(&mb, b, K, N, G, 256)) != DG_SUCCESS) return st;
    const int tiles = (M_total / 128) * (N / 256);
    const int grid = tiles < info->num_sms ? tiles : info->num_sms;
    return launch<256, false, 4, dg::kContiguous, 1, true>(ma, mb, md, p, grid, 1, 1, static_cast<cudaStream_t>(stream));
}

dg_status_t dg_m_grouped_fp8_ffn_contiguous(const uint8_t *a, const float *sfa, int ld_sfa,
                                            const uint8_t *w1, const float *sfb1, const uint8_t *w2,
                                            const float *sfb2, uint8_t *q_mid, float *s_mid,
                                            int ld_mid, void *y, const int32_t *m_indices,
                                            int M_total, int H, int I, int G, void *stream) {
    if (I <= 0 || I % 128 != 0) return DG_ERR_UNSUPPORTED_SHAPE;
    if (!y) return DG_ERR_INVALID_VALUE;
    dg_status_t st = dg_m_grouped_fp8_gemm_swiglu_quant_contiguous(a, sfa, ld_sfa, w1, sfb1, q_mid, s_mid, ld_mid,
                                                                   m_indices, M_total, 2 * I, H, G, stream);
    if (st != DG_SUCCESS) return st;
    return dg_m_grouped_fp8_gemm_nt_contiguous(q_mid, s_mid, ld_mid, w2, sfb2, y, m_indices, M_total, H, I, G,
                                               stream);
}

}  // extern "C"

// ------------------------------------------------------------ no-allocation FFN
namespace {
// The intermediate of dg_m_grouped_fp8_ffn_contiguous_noalloc (E4M3 codes, then
// their scales) lives in this file-scope device array, for callers that cannot
// allocate device memory.  Every GPU that loads the library holds it until exit.
__device__ __align__(256) unsigned char g_noalloc_scratch[DG_NOALLOC_SCRATCH_BYTES];

// The array's device address on each device.  In host code the name
// g_noalloc_scratch is only a host-side stand-in, not a device address (a kernel
// given it would fault, or silently use host memory where the GPU can reach it),
// so the address is looked up once per device, with that device current.
std::atomic<void *> g_noalloc_addr[kMaxDevices];

dg_status_t noalloc_scratch(void **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices) return DG_ERR_UNSUPPORTED_DEVICE;
    void *p = g_noalloc_addr[dev].load(std::memory_order_acquire);
    if (!p) {
        if ((e = cudaGetSymbolAddress(&p, g_noalloc_scratch)) != cudaSuccess)
            return cuda_fail(e, "cudaGetSymbolAddress(no-allocation scratch)");
        g_noalloc_addr[dev].store(p, std::memory_order_release);
    }
    *out = p;
    return DG_SUCCESS;
}
}  // namespace

extern "C" {

dg_status_t dg_m_grouped_fp8_ffn_contiguous_noalloc(const uint8_t *a, const float *sfa, int ld_sfa,
                                                    const uint8_t *w1, const float *sfb1,
                                                    const uint8_t *w2, const float *sfb2, void *y,
                                                    const int32_t *m_indices, int M_total, int H,
                                                    int I, int G, void *stream) {
    if (M_total < 0) return DG_ERR_INVALID_VALUE;
    if (I <= 0 || I % 128 != 0) return DG_ERR_UNSUPPORTED_SHAPE;
    // intermediate: codes [M_total][I], then scales [I/128][ld_mid] at a 256-byte offset
    const long long ld_mid = M_total < 4 ? 4 : (static_cast<long long>(M_total) + 3) / 4 * 4;
    const long long s_offset = (static_cast<long long>(M_total) * I + 255) / 256 * 256;
    const long long need = s_offset + static_cast<long long>(I / 128) * ld_mid * 4;
    if (need > static_cast<long long>(DG_NOALLOC_SCRATCH_BYTES)) return DG_ERR_UNSUPPORTED_SHAPE;
    const DeviceInfo *info = nullptr;
    dg_status_t st = device_info(&info);
    if (st != DG_SUCCESS) return st;
    void *scratch = nullptr;
    if ((st = noalloc_scratch(&scratch)) != DG_SUCCESS) return st;
    uint8_t *q_mid = static_cast<uint8_t *>(scratch);
    float *s_mid = reinterpret_cast<float *>(static_cast<unsigned char *>(scratch) + s_offset);
    return dg_m_grouped_fp8_ffn_contiguous(a, sfa, ld_sfa, w1, sfb1, w2, sfb2, q_mid, s_mid,
                                           static_cast<int>(ld_mid), y, m_indices, M_total, H, I, G,
                                           stream);
}

int dg_get_m_alignment_for_contiguous_layout(void) { return 128; }

size_t dg_get_tma_aligned_size(size_t n, size_t elem_bytes) {
    if (elem_bytes == 0 || elem_bytes > 16 || 16 % elem_bytes != 0) return 0;
    const size_t q = 16 / elem_bytes;
    return (n + q - 1) / q * q;
}

dg_status_t dg_get_device_status(int *code, int clear) {
    if (!code) return DG_ERR_INVALID_VALUE;
    const DeviceInfo *info = nullptr;
    dg_status_t st = device_info(&info);
    if (st != DG_SUCCESS) return st;
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceSynchronize");
    unsigned v = 0;
    if ((e = cudaMemcpyFromSymbol(&v, g_dg_status, sizeof(v))) != cudaSuccess)
        return cuda_fail(e, "cudaMemcpyFromSymbol(status)");
    *code = static_cast<int>(v);
    if (clear) {
        const unsigned zero = 0;
        if ((e = cudaMemcpyToSymbol(g_dg_status, &zero, sizeof(zero))) != cudaSuccess)
            return cuda_fail(e, "cudaMemcpyToSymbol(status)");
    }
    return DG_SUCCESS;
}

const char *dg_status_string(dg_status_t status) {
    switch (status) {
        case DG_SUCCESS: return "success";
        case DG_ERR_INVALID_VALUE: return "invalid value";
        case DG_ERR_MISALIGNED: return "pointer or leading dimension not 16-byte aligned";
        case DG_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
        case DG_ERR_UNSUPPORTED_DEVICE: return "unsupported device (needs compute capability 10.0)";
        case DG_ERR_CUDA: return "CUDA error";
        case DG_ERR_TIMEOUT: return "a kernel wait timed out";
    }
    return "unknown status";
}

const char *dg_last_cuda_error(void) { return t_last_cuda_error; }

// Test hook (not part of the GEMM contract): kernels launched afterwards on
// this process run with the given debug flags.  Flag 1 makes the producer warp
// issue no loads, so the consumers' bounded waits run out and the kernel
// reports DG_ERR_TIMEOUT through the status word instead of hanging.  Flag 2
// makes the quantiser take the IEEE division for every element (its results
// are identical; tests compare the two paths).
void dg_debug_set_flags(int flags) { g_debug_flags = flags; }

}  // extern "C"
