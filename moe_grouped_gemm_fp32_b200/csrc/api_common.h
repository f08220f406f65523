// api_common.h -- host-side helpers shared by the library's translation units
// (GEMMs in dg_api.cu, quantisers in quant_api.cu): device capability cache,
// CUDA error capture, alignment check, debug flags and DG_VERBOSE.  Internal:
// nothing here is exported from the shared library.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "dg.h"

namespace dg_host {

constexpr int kMaxDevices = 64;

struct DeviceInfo {
    bool ready = false;
    bool supported = false;
    int num_sms = 0;
    unsigned *status = nullptr;   // device address of the library's status word
};

// Capabilities of the current device (cached); DG_ERR_UNSUPPORTED_DEVICE
// unless it is compute capability 10.0.
dg_status_t device_info(const DeviceInfo **out);

// Records "what: CUDA error text" for dg_last_cuda_error() and returns DG_ERR_CUDA.
dg_status_t cuda_fail(cudaError_t e, const char *what);

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Flags set by dg_debug_set_flags().
int debug_flags();

// DG_VERBOSE=1 prints each launch's configuration to stderr.
bool verbose();

// Bounded-wait limit in clock cycles for kernels (DG_WAIT_TIMEOUT_CYCLES, read once).
long long timeout_cycles();

// 3-D tensor map {K, rows, groups} of elem_bytes-wide elements (1: uint8 E4M3,
// 2: BF16), K innermost with a row stride of K elements; box {128 bytes of K,
// box_rows, 1}; 128-byte swizzle; out-of-bounds elements read as zero.
dg_status_t make_kmajor_map(CUtensorMap *m, const void *base, int elem_bytes, long long K,
                            long long rows, long long groups, int box_rows);

}  // namespace dg_host
