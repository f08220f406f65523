// quant_api.cu -- host side of the quantiser entry points declared in
// include/dg.h (dg_per_token_cast_to_fp8, dg_per_token_cast_to_fp8_masked):
// argument validation, grid sizing from the kernel's occupancy, launch.
// Nothing here synchronises the host or allocates memory.
#include <cuda_runtime.h>

#include <atomic>
#include <cstdio>

#include "dg.h"
#include "api_common.h"
#include "quant_kernel.cuh"

namespace {
using namespace dg_host;

constexpr int kBlockK = 128;
constexpr int kDebugQuantExactDiv = 2;   // quantiser: IEEE division on every element

template <bool kMasked, bool kFastDiv>
dg_status_t launch_quant(const dg::QuantParams &p, long long max_items, const DeviceInfo *info,
                         cudaStream_t stream) {
    auto kernel = dg::quant_1x128_kernel<kMasked, kFastDiv>;
    // per-device cache of an idempotent query (atomic: concurrent first calls are defined)
    static std::atomic<int> occ[kMaxDevices] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    int resident = occ[dev].load(std::memory_order_relaxed);
    if (!resident) {
        int n = 0;
        cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, dg::kQuantThreads, 0);
        if (e != cudaSuccess) return cuda_fail(e, "cudaOccupancyMaxActiveBlocksPerMultiprocessor");
        resident = n > 0 ? n : 1;
        occ[dev].store(resident, std::memory_order_relaxed);
    }
    const long long want = (max_items + dg::kQuantWarps - 1) / dg::kQuantWarps;
    const long long full = static_cast<long long>(info->num_sms) * resident;
    const int grid = static_cast<int>(want < full ? (want > 0 ? want : 1) : full);
    if (verbose())
        std::fprintf(stderr, "[dg] quant_1x128 masked=%d fast_div=%d grid=%d occ=%d\n", kMasked ? 1 : 0,
                     kFastDiv ? 1 : 0, grid, resident);
    kernel<<<grid, dg::kQuantThreads, 0, stream>>>(p);
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? DG_SUCCESS : cuda_fail(e, "quant_1x128_kernel launch");
}

dg_status_t check_quant(const void *x, const uint8_t *q, const float *sfa, int ld_sfa, int rows,
                        int K) {
    if (!x || !q || !sfa) return DG_ERR_INVALID_VALUE;
    if (rows < 0 || K <= 0) return DG_ERR_INVALID_VALUE;
    if (K % kBlockK != 0) return DG_ERR_UNSUPPORTED_SHAPE;
    if (ld_sfa < rows || ld_sfa <= 0) return DG_ERR_INVALID_VALUE;
    if (ld_sfa % 4 != 0) return DG_ERR_MISALIGNED;
    if (!aligned16(x) || !aligned16(q) || !aligned16(sfa)) return DG_ERR_MISALIGNED;
    if (static_cast<long long>(K) > (1LL << 30)) return DG_ERR_UNSUPPORTED_SHAPE;
    return DG_SUCCESS;
}

}  // namespace

extern "C" {

dg_status_t dg_per_token_cast_to_fp8(const void *x, uint8_t *q, float *sfa, int ld_sfa, int M,
                                     int K, void *stream) {
    dg_status_t st = check_quant(x, q, sfa, ld_sfa, M, K);
    if (st != DG_SUCCESS) return st;
    const DeviceInfo *info = nullptr;
    if ((st = device_info(&info)) != DG_SUCCESS) return st;
    if (M == 0) return DG_SUCCESS;
    dg::QuantParams p = {};
    p.x = static_cast<const uint4 *>(x);
    p.q = reinterpret_cast<uint2 *>(q);
    p.sfa = sfa;
    p.status = info->status;
    p.rows = M;
    p.num_kb = K / kBlockK;
    p.ld_sfa = ld_sfa;
    p.G = 1;
    const long long items = static_cast<long long>(M) *
                            ((p.num_kb + dg::kQuantBlocksPerWarp - 1) / dg::kQuantBlocksPerWarp);
    if (items > (1LL << 31) - 1) return DG_ERR_UNSUPPORTED_SHAPE;   // 32-bit item walk
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (debug_flags() & kDebugQuantExactDiv) return launch_quant<false, false>(p, items, info, s);
    return launch_quant<false, true>(p, items, info, s);
}

dg_status_t dg_per_token_cast_to_fp8_masked(const void *x, uint8_t *q, float *sfa, int ld_sfa,
                                            const int32_t *masked_m, int G, int Mmax, int K,
                                            void *stream) {
    dg_status_t st = check_quant(x, q, sfa, ld_sfa, Mmax, K);
    if (st != DG_SUCCESS) return st;
    if (!masked_m || G <= 0) return DG_ERR_INVALID_VALUE;
    if (G > dg::kQuantMaxGroups) return DG_ERR_UNSUPPORTED_SHAPE;
    if (static_cast<long long>(G) * Mmax > (1LL << 31) - 1) return DG_ERR_UNSUPPORTED_SHAPE;
    const DeviceInfo *info = nullptr;
    if ((st = device_info(&info)) != DG_SUCCESS) return st;
    if (Mmax == 0) return DG_SUCCESS;
    dg::QuantParams p = {};
    p.x = static_cast<const uint4 *>(x);
    p.q = reinterpret_cast<uint2 *>(q);
    p.sfa = sfa;
    p.masked_m = masked_m;
    p.status = info->status;
    p.rows = Mmax;
    p.num_kb = K / kBlockK;
    p.ld_sfa = ld_sfa;
    p.G = G;
    // the valid-row count lives on the device: size the grid for every row
    const long long items = static_cast<long long>(G) * Mmax *
                            ((p.num_kb + dg::kQuantBlocksPerWarp - 1) / dg::kQuantBlocksPerWarp);
    if (items > (1LL << 31) - 1) return DG_ERR_UNSUPPORTED_SHAPE;   // 32-bit item walk
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (debug_flags() & kDebugQuantExactDiv) return launch_quant<true, false>(p, items, info, s);
    return launch_quant<true, true>(p, items, info, s);
}

}  // extern "C"
