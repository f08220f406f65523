// bf16_api.cu -- host side of the BF16 GEMM entry points declared in
// include/dg.h (dg_bf16_gemm_nt, dg_m_grouped_bf16_gemm_nt_contiguous,
// dg_m_grouped_bf16_gemm_nt_masked): argument validation, TMA descriptors,
// tile width by wave efficiency, launch.  Nothing here synchronises the host
// or allocates memory.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdio>
#include <cstdlib>

#include "dg.h"
#include "api_common.h"
#include "bf16_kernel.cuh"

namespace {
using namespace dg_host;

dg_status_t check_bf16(const void *a, const void *b, const void *d, int rows, int N, int K) {
    if (!a || !b || !d) return DG_ERR_INVALID_VALUE;
    if (rows < 0 || N <= 0 || K <= 0) return DG_ERR_INVALID_VALUE;
    // 16-byte row strides for TMA (K) and 16-byte output stores (N)
    if (K % 8 != 0 || N % 8 != 0) return DG_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(a) || !aligned16(b) || !aligned16(d)) return DG_ERR_MISALIGNED;
    if (static_cast<long long>(K) > (1LL << 30) || N > (1 << 30)) return DG_ERR_UNSUPPORTED_SHAPE;
    return DG_SUCCESS;
}

dg::Params bf16_params(void *d, int rows, int N, int K, int G, const DeviceInfo *info) {
    dg::Params p = {};
    p.d = static_cast<__nv_bfloat16 *>(d);
    p.status = info->status;
    p.timeout_cycles = timeout_cycles();
    p.M = rows;
    p.N = N;
    p.K = K;
    p.G = G;
    p.num_kb = (K + dg::kBf16BlockK - 1) / dg::kBf16BlockK;
    p.num_nb = (N + 127) / 128;
    p.split = 1;
    p.debug_flags = debug_flags();
    return p;
}

template <int kBN, int kStages, int kLayout, bool kSplitK = false, int kCtaGroup = 1>
dg_status_t launch_bf16(const CUtensorMap &ma, const CUtensorMap &mb, const dg::Params &p, int grid,
                        cudaStream_t stream, int grid_y = 1, int cluster_x = 1) {
    using L = dg::Bf16Smem<kBN, kStages, kSplitK, kCtaGroup>;
    auto kernel = dg::bf16_gemm_kernel<kBN, kStages, kLayout, kSplitK, kCtaGroup>;
    // one-time per-device set-up (idempotent; the atomic flag keeps racing first calls defined)
    static std::atomic<bool> configured[kMaxDevices] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (!configured[dev].load(std::memory_order_acquire)) {
        cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc);
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(bf16 smem)");
        configured[dev].store(true, std::memory_order_release);
    }
    if (verbose())
        std::fprintf(stderr, "[dg] bf16_gemm layout=%d bn=%d stages=%d ctas/mma=%d grid=%dx%d cluster=%d split=%d smem=%d\n",
                     kLayout, kBN, kStages, kCtaGroup, grid, grid_y, cluster_x, p.split, L::kAlloc);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid, grid_y, 1);
    cfg.blockDim = dim3(dg::kBf16Threads, 1, 1);
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
    cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, ma, mb, p);
    return e == cudaSuccess ? DG_SUCCESS : cuda_fail(e, "bf16_gemm_kernel launch");
}

// tile width: N <= 128 -> 128; otherwise 224 or 256, whichever wastes less of
// the last wave and of the last weight-tile's columns
int pick_bn(long long token_blocks, int N, int num_sms) {
    if (N <= 128) return 128;
    auto eff = [&](int bn) {
        const long long nt = (N + bn - 1) / bn;
        const long long tiles = token_blocks * nt;
        const long long waves = (tiles + num_sms - 1) / num_sms;
        return (static_cast<double>(N) / (nt * bn)) * (static_cast<double>(tiles) / (waves * num_sms));
    };
    return eff(224) > eff(256) + 1e-9 ? 224 : 256;
}

// Resident clusters of `split` CTAs of the split-K kernel, or of CTA pairs of
// the pair kernel (0 if the query fails).
template <int kBN, int kStages, int kLayout = dg::kDense, bool kSplitK = true, int kCtaGroup = 1>
int bf16_max_clusters(int split) {
    using L = dg::Bf16Smem<kBN, kStages, kSplitK, kCtaGroup>;
    auto kernel = dg::bf16_gemm_kernel<kBN, kStages, kLayout, kSplitK, kCtaGroup>;
    // per-device cache of an idempotent query (atomic: concurrent first calls are defined)
    static std::atomic<int> cache[kMaxDevices][9] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (split < 2 || split > 8) return 0;
    if (const int c = cache[dev][split].load(std::memory_order_relaxed)) return c;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc) != cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(split, 1, 1);
    cfg.blockDim = dim3(dg::kBf16Threads, 1, 1);
    cfg.dynamicSmemBytes = L::kAlloc;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = split;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kernel, &cfg) != cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    cache[dev][split].store(n, std::memory_order_relaxed);
    return n;
}

// CTA pairs (256-row tiles, tcgen05.mma.cta_group::2) for the dense and
// contiguous layouts with N > 128 and at least two 128-row blocks: each SM then
// reads half of the weight tile per K-block.  DG_BF16_PAIRS=0 / =1 forces
// single-CTA tiles / pairs (comparisons and tests).
int bf16_pairs_env() {
    static const int v = [] {
        const char *e = std::getenv("DG_BF16_PAIRS");
        return e ? (e[0] == '1' ? 1 : 0) : -1;
    }();
    return v;
}

template <int kLayout>
dg_status_t dispatch_pairs(const CUtensorMap &ma, const void *b, int N, int K, int G, const dg::Params &p,
                           long long row_pairs, cudaStream_t s, bool *done) {
    *done = false;
    const int pm224 = bf16_max_clusters<224, 6, kLayout, false, 2>(2);
    const int pm256 = bf16_max_clusters<256, 6, kLayout, false, 2>(2);
    auto eff = [&](int bn, int pairs_max) {
        if (pairs_max <= 0) return 0.0;
        const long long nt = (N + bn - 1) / bn;
        const long long tiles = row_pairs * nt;
        const long long waves = (tiles + pairs_max - 1) / pairs_max;
        return (static_cast<double>(N) / (nt * bn)) * (static_cast<double>(tiles) / (waves * pairs_max));
    };
    const int bn = eff(224, pm224) > eff(256, pm256) + 1e-9 ? 224 : 256;
    const int pairs_max = bn == 224 ? pm224 : pm256;
    if (pairs_max <= 0) return DG_SUCCESS;   // no resident pair: the caller takes single-CTA tiles
    CUtensorMap mb;
    dg_status_t st = make_kmajor_map(&mb, b, 2, K, N, G, bn / 2);
    if (st != DG_SUCCESS) return st;
    const long long tiles = row_pairs * ((N + bn - 1) / bn);
    const int pairs = tiles < pairs_max ? static_cast<int>(tiles) : pairs_max;
    *done = true;
    if (bn == 224) return launch_bf16<224, 6, kLayout, false, 2>(ma, mb, p, 2 * pairs, s, 1, 2);
    return launch_bf16<256, 6, kLayout, false, 2>(ma, mb, p, 2 * pairs, s, 1, 2);
}

template <int kLayout>
dg_status_t dispatch(const CUtensorMap &ma, const void *b, int N, int K, int G, const dg::Params &p,
                     long long tiles_hint_blocks, int grid_cap, cudaStream_t s) {
    if constexpr (kLayout != dg::kMasked) {
        if (N > 128 && bf16_pairs_env() != 0 && (tiles_hint_blocks >= 2 || bf16_pairs_env() == 1) &&
            (kLayout != dg::kContiguous || G < dg::kMaxGroups)) {
            bool done = false;
            const dg_status_t st = dispatch_pairs<kLayout>(ma, b, N, K, G, p, (tiles_hint_blocks + 1) / 2, s, &done);
            if (st != DG_SUCCESS || done) return st;
        }
    }
    const int bn = pick_bn(tiles_hint_blocks, N, grid_cap);
    CUtensorMap mb;
    dg_status_t st = make_kmajor_map(&mb, b, 2, K, N, G, bn);
    if (st != DG_SUCCESS) return st;
    const long long tiles = tiles_hint_blocks * ((N + bn - 1) / bn);
    const int grid = tiles < grid_cap ? static_cast<int>(tiles > 0 ? tiles : 1) : grid_cap;
    if (bn == 128) return launch_bf16<128, 6, kLayout>(ma, mb, p, grid, s);
    if (bn == 224) return launch_bf16<224, 4, kLayout>(ma, mb, p, grid, s);
    return launch_bf16<256, 4, kLayout>(ma, mb, p, grid, s);
}

}  // namespace

extern "C" {

dg_status_t dg_bf16_gemm_nt(const void *a, const void *b, void *d, int M, int N, int K, void *stream) {
    dg_status_t st = check_bf16(a, b, d, M, N, K);
    if (st != DG_SUCCESS) return st;
    const DeviceInfo *info = nullptr;
    if ((st = device_info(&info)) != DG_SUCCESS) return st;
    if (M == 0) return DG_SUCCESS;
    dg::Params p = bf16_params(d, M, N, K, 1, info);
    CUtensorMap ma;
    if ((st = make_kmajor_map(&ma, a, 2, K, M, 1, 128)) != DG_SUCCESS) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // one token block and few weight tiles (decode shapes): split K over a
    // cluster of CTAs per 128-wide tile, the largest split <= 8 whose clusters
    // are all resident (DG_SPLIT_K overrides)
    if (M <= 128) {
        static const int forced = [] {
            const char *e = std::getenv("DG_SPLIT_K");
            return e ? std::atoi(e) : 0;
        }();
        const int tiles = (N + 127) / 128;
        int split = 1;
        if (forced >= 2 && forced <= 8) {
            split = p.num_kb >= 2 * forced ? forced : 1;
        } else {
            for (int c = 8; c >= 2; --c) {
                if (tiles * c > info->num_sms || p.num_kb < 2 * c) continue;
                if (bf16_max_clusters<128, 4>(c) >= tiles) { split = c; break; }
            }
        }
        if (split > 1) {
            CUtensorMap mb;
            if ((st = make_kmajor_map(&mb, b, 2, K, N, 1, 128)) != DG_SUCCESS) return st;
            p.split = split;
            return launch_bf16<128, 4, dg::kDense, true>(ma, mb, p, split, s, tiles, split);
        }
    }
    return dispatch<dg::kDense>(ma, b, N, K, 1, p, (M + 127) / 128, info->num_sms, s);
}

dg_status_t dg_m_grouped_bf16_gemm_nt_contiguous(const void *a, const void *b, void *d,
                                                 const int32_t *m_indices, int M_total, int N, int K,
                                                 int G, void *stream) {
    dg_status_t st = check_bf16(a, b, d, M_total, N, K);
    if (st != DG_SUCCESS) return st;
    if (!m_indices || G <= 0) return DG_ERR_INVALID_VALUE;
    if (M_total % 128 != 0) return DG_ERR_UNSUPPORTED_SHAPE;
    const DeviceInfo *info = nullptr;
    if ((st = device_info(&info)) != DG_SUCCESS) return st;
    if (M_total == 0) return DG_SUCCESS;
    dg::Params p = bf16_params(d, M_total, N, K, G, info);
    p.m_indices = m_indices;
    CUtensorMap ma;
    if ((st = make_kmajor_map(&ma, a, 2, K, M_total, 1, 128)) != DG_SUCCESS) return st;
    return dispatch<dg::kContiguous>(ma, b, N, K, G, p, M_total / 128, info->num_sms,
                                     static_cast<cudaStream_t>(stream));
}

dg_status_t dg_m_grouped_bf16_gemm_nt_masked(const void *a, const void *b, void *d,
                                             const int32_t *masked_m, int G, int Mmax, int N, int K,
                                             void *stream) {
    dg_status_t st = check_bf16(a, b, d, Mmax, N, K);
    if (st != DG_SUCCESS) return st;
    if (!masked_m || G <= 0) return DG_ERR_INVALID_VALUE;
    if (G > dg::kMaxGroups) return DG_ERR_UNSUPPORTED_SHAPE;
    if (static_cast<long long>(G) * Mmax > (1LL << 31) - 1) return DG_ERR_UNSUPPORTED_SHAPE;
    const DeviceInfo *info = nullptr;
    if ((st = device_info(&info)) != DG_SUCCESS) return st;
    if (Mmax == 0) return DG_SUCCESS;
    dg::Params p = bf16_params(d, Mmax, N, K, G, info);
    p.masked_m = masked_m;
    CUtensorMap ma;
    if ((st = make_kmajor_map(&ma, a, 2, K, Mmax, G, 128)) != DG_SUCCESS) return st;
    // the tile count lives on the device: a persistent grid of one CTA per SM;
    // the tile width assumes every group full (the workload's upper bound)
    return dispatch<dg::kMasked>(ma, b, N, K, G, p, static_cast<long long>(G) * ((Mmax + 127) / 128),
                                 info->num_sms, static_cast<cudaStream_t>(stream)) ;
}

}  // extern "C"
