// quant_kernel.cuh -- the per-token 1x128 activation quantiser (BF16 -> E4M3
// codes + FP32 block scales), the step that produces the GEMM's A operand and
// its scales at run time (DeepGEMM pages: page 2 "技术特性" -- fine-grained
// dynamic scaling; page 3 "核心功能" -- block-wise scaling instead of one
// factor per tensor).
//
// For every row m and 128-wide K-block kb:
//   amax = max_k |x[m,k]|,  s = amax / 448 (FP32, IEEE division; 1 when amax == 0)
//   q[m,k] = E4M3_RNE(clamp(x[m,k] / s, -448, 448)),  sfa[kb][m] = s
// The quotient x / s is the correctly rounded FP32 division, so the codes are
// reproducible bit for bit on any IEEE machine.
//
// The work is pure streaming (2 bytes in, 1 byte + 4/128 bytes out per
// element), so the kernel is laid out for HBM: a warp owns one row segment of
// up to 8 K-blocks; each half-warp covers one 256-byte block with one 16-byte
// load per lane, four blocks in flight per half-warp, consecutive half-warps
// on consecutive blocks (512 contiguous bytes per warp load, 128 per store).
// The block's amax is an exact BF16 max (packed max.bf16x2 and four xor
// shuffles inside the half-warp).
//
// Division.  The scale is shared by the block's 128 elements, so the kernel
// multiplies by r = RN(1/s) instead of dividing, and proves per element that
// the product gives the code the correctly rounded quotient would: y = RN(x*r)
// lies within 2.5 units in the last place of RN(x/s), so both lie between
// y * (1 - 2^-21) and y * (1 + 2^-21); when those two ends quantise to the
// same code (E4M3 rounding is monotone), that code is the answer.  Only ends
// that disagree -- x/s within about 2^-21 (relative) of an E4M3 rounding
// midpoint -- or an infinite reciprocal (s below 2^-128) take __fdiv_rn.  The
// check is packed FP32 multiplies and conversions, not integer bit tests,
// which would load the half-rate integer pipe.  The all-division
// instantiation exists so tests can check that both give the same codes.
//
// The four blocks' scales are computed together: lane j of a half-warp does
// the one IEEE division amax / 448 and the reciprocal for block j % 4, and the
// results are broadcast with shuffles.  Each warp prefetches its next item's
// loads before working on the current one.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace dg {

struct QuantParams {
    const uint4 *x;             // BF16 rows, as 16-byte chunks of 8 values
    uint2 *q;                   // E4M3 rows, as 8-byte chunks
    float *sfa;                 // [G][KB][ld_sfa]
    const int32_t *masked_m;    // masked layout: valid rows per group (device)
    unsigned *status;           // device status word
    int rows;                   // dense: M; masked: Mmax (rows per group)
    int num_kb;                 // K / 128
    int ld_sfa;
    int G;                      // 1 for the dense layout
};

constexpr int kQuantThreads = 256;
constexpr int kQuantWarps = kQuantThreads / 32;
constexpr int kQuantBlocksPerWarp = 8;   // K-blocks per warp work item (2 half-warps x 4)
constexpr int kQuantMaxGroups = 1024;
constexpr unsigned kQuantSiteBadMask = 9;

namespace quant {

__device__ __forceinline__ uint4 ld_stream(const uint4 *p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// max(|a|, |b|) per BF16 half; the sign bits come out as the xor of the
// inputs' signs and are cleared by the caller
__device__ __forceinline__ uint32_t absmax_bf16x2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// (a0 * b0, a1 * b1), each rounded to nearest even (packed FP32 pipe op)
__device__ __forceinline__ void mul2(float &d0, float &d1, float a0, float a1, float b0, float b1) {
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\t"
        "mov.b64 rb, {%4, %5};\n\t"
        "mul.rn.f32x2 rd, ra, rb;\n\t"
        "mov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d0), "=f"(d1)
        : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

// two FP32 values -> two E4M3 codes (RNE, finite values saturate to +-448);
// lo lands in the low byte
__device__ __forceinline__ uint32_t cvt_e4m3x2(float lo, float hi) {
    uint16_t d;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(d) : "f"(hi), "f"(lo));
    return d;
}

__device__ __forceinline__ void unpack8(const uint32_t (&w)[4], float (&x)[8]) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        x[2 * j] = __uint_as_float(w[j] << 16);
        x[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
    }
}

// Codes of 8 values x_j (BF16 pairs w) by the reciprocal: y = RN(x * r) is
// within 2.5 units in the last place of RN(x/s) (both normal, r = RN(1/s)),
// so both lie inside [y (1 - 2^-21), y (1 + 2^-21)], whose ends are at least 3
// units from y.  E4M3 rounding is monotone, so when the two ends give the same
// code every point between them does too -- RN(x/s) included -- and that code
// is returned.  The bytes of (d0, d1) are non-zero where the ends disagree:
// x/s lies within about 2^-21 (relative) of an E4M3 rounding midpoint, and
// code_near_midpoint settles the element.  The sign of a zero is kept
// (y = x * r keeps x's).
__device__ __forceinline__ uint2 codes8_fast(const uint32_t (&w)[4], float r, uint32_t &d0,
                                             uint32_t &d1) {
    float x[8], y[8], a[8], b[8];
    unpack8(w, x);
#pragma unroll
    for (int j = 0; j < 8; j += 2) {
        mul2(y[j], y[j + 1], x[j], x[j + 1], r, r);
        mul2(a[j], a[j + 1], y[j], y[j + 1], 1.0f - 0x1p-21f, 1.0f - 0x1p-21f);
        mul2(b[j], b[j + 1], y[j], y[j + 1], 1.0f + 0x1p-21f, 1.0f + 0x1p-21f);
    }
    uint32_t lo[2], hi[2];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        lo[j] = cvt_e4m3x2(a[4 * j], a[4 * j + 1]) | (cvt_e4m3x2(a[4 * j + 2], a[4 * j + 3]) << 16);
        hi[j] = cvt_e4m3x2(b[4 * j], b[4 * j + 1]) | (cvt_e4m3x2(b[4 * j + 2], b[4 * j + 3]) << 16);
    }
    d0 = lo[0] ^ hi[0];
    d1 = lo[1] ^ hi[1];
    return make_uint2(hi[0], hi[1]);
}

// E4M3 code (low byte) of RN(x / s) by the IEEE division.
__device__ __noinline__ uint32_t code_div(float x, float s) {
    return cvt_e4m3x2(__fdiv_rn(x, s), 0.0f) & 0xFFu;
}

// E4M3 code of RN(x / s) for an element whose ends disagreed.  Such ties are
// common, not rare: BF16 values have 8-bit significands, so x/s often lands
// exactly on an E4M3 midpoint (a 5-bit significand).  In the E4M3 normal range
// the midpoint M near y = RN(x * r) has y's sign, exponent and top three
// mantissa bits followed by the bit pattern 0x80000 (y is within 4 units of M,
// which never sits at a binade edge).  RN(x/s) == M exactly when
// |x/s - M| <= half an FP32 unit of M, i.e. |x - M s| <= h = s * 2^(e_M - 24);
// x - M s is computed exactly by one FMA (it is a multiple of
// 2^(e_M + e_s - 27) below 2^8 of those), h exactly by a power-of-two scaling,
// and x/s is never itself an FP32 midpoint (a BF16 value cannot equal a 25-bit
// odd significand times s), so the comparison decides.  The code is then
// produced by converting M itself (a tie: round-half-even, like the quotient),
// or M nudged by one unit towards the quotient's side.  E4M3 subnormals,
// scales below 2^-90 and an infinite reciprocal take the IEEE division.
__device__ __forceinline__ uint32_t code_near_midpoint(float x, float s, float r) {
    const float y = __fmul_rn(x, r);
    const uint32_t yb = __float_as_uint(y);
    const uint32_t mag = yb & 0x7FFFFFFFu;
    if (mag < 0x3C800000u || mag >= 0x44000000u || !(s >= 0x1p-90f) || !(r < INFINITY))
        return code_div(x, s);
    const uint32_t mb = (yb & 0xFFF00000u) | 0x80000u;
    const float rm = fmaf(-__uint_as_float(mb), s, x);
    const float h = __uint_as_float((mb & 0x7F800000u) - (24u << 23)) * s;
    const float beyond = (yb >> 31) ? -rm : rm;   // > 0: |x/s| above |M|
    uint32_t zb = mb;
    if (beyond > h) zb += 1u;
    else if (beyond < -h) zb -= 1u;
    return cvt_e4m3x2(__uint_as_float(zb), 0.0f) & 0xFFu;
}

// Codes of 8 values by the IEEE division RN(x / s).  Kept out of line: it is
// the rare path, and inlined its eight division sequences would be predicated
// into every block's instruction stream.
__device__ __noinline__ uint2 codes8_div(uint32_t w0, uint32_t w1, uint32_t w2, uint32_t w3, float s) {
    const uint32_t w[4] = {w0, w1, w2, w3};
    float x[8], t[8];
    unpack8(w, x);
#pragma unroll
    for (int j = 0; j < 8; ++j) t[j] = __fdiv_rn(x[j], s);
    uint32_t c[2];
#pragma unroll
    for (int j = 0; j < 2; ++j)
        c[j] = cvt_e4m3x2(t[4 * j], t[4 * j + 1]) | (cvt_e4m3x2(t[4 * j + 2], t[4 * j + 3]) << 16);
    return make_uint2(c[0], c[1]);
}

}  // namespace quant

template <bool kMaskedLayout, bool kFastDiv>
__global__ void __launch_bounds__(kQuantThreads) quant_1x128_kernel(QuantParams p) {
    __shared__ int prefix[kQuantMaxGroups + 1];   // masked: exclusive prefix of valid rows
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int half = lane >> 4;
    const int l16 = lane & 15;

    int total_rows = p.rows;
    if (kMaskedLayout) {
        if (warp == 0) {
            int carry = 0;
            for (int base = 0; base < p.G; base += 32) {
                const int g = base + lane;
                int mm = 0;
                if (g < p.G) {
                    mm = __ldg(p.masked_m + g);
                    if (mm < 0 || mm > p.rows) {
                        if (blockIdx.x == 0)
                            atomicCAS(p.status, 0u, 1u | (kQuantSiteBadMask << 8));
                        mm = mm < 0 ? 0 : p.rows;
                    }
                }
                int incl = mm;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int t = __shfl_up_sync(0xffffffffu, incl, o);
                    if (lane >= o) incl += t;
                }
                if (g < p.G) prefix[g] = carry + incl - mm;
                carry += __shfl_sync(0xffffffffu, incl, 31);
            }
            if (lane == 0) prefix[p.G] = carry;
        }
        __syncthreads();
        total_rows = prefix[p.G];
    }

    // work items: (valid row, chunk of 8 K-blocks); a warp walks items with a
    // fixed stride, carrying (row, chunk) instead of dividing
    const int nchunk = (p.num_kb + kQuantBlocksPerWarp - 1) / kQuantBlocksPerWarp;
    const unsigned items = static_cast<unsigned>(total_rows) * static_cast<unsigned>(nchunk);
    const unsigned stride = gridDim.x * kQuantWarps;
    const int stride_rows = static_cast<int>(stride / nchunk);
    const int stride_chunks = static_cast<int>(stride - static_cast<unsigned>(stride_rows) * nchunk);
    unsigned it = blockIdx.x * kQuantWarps + warp;
    int vr = static_cast<int>(it / nchunk);
    int chunk = static_cast<int>(it - static_cast<unsigned>(vr) * nchunk);
    const size_t row_chunks = static_cast<size_t>(p.num_kb) * 16;   // 16-byte x chunks per row

    // the loads of one item: 4 blocks of this half-warp (blocks past K read nothing)
    auto locate = [&](int vrow, int& g, int& row) {
        g = 0;
        row = vrow;
        if (kMaskedLayout) {
            int lo = 0, hi = p.G - 1;   // last group whose prefix is <= vrow
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (prefix[mid] <= vrow) lo = mid; else hi = mid - 1;
            }
            g = lo;
            row = vrow - prefix[g];
        }
    };
    auto load = [&](int vrow, int ch, uint4 (&v)[4]) {
        int g, row;
        locate(vrow, g, row);
        const uint4 *xr = p.x + (static_cast<size_t>(g) * p.rows + row) * row_chunks;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int kb = ch * kQuantBlocksPerWarp + 2 * i + half;
            v[i] = kb < p.num_kb ? quant::ld_stream(xr + static_cast<size_t>(kb) * 16 + l16)
                                 : make_uint4(0u, 0u, 0u, 0u);
        }
    };

    uint4 v[4];
    if (it < items) load(vr, chunk, v);
    while (it < items) {
        // prefetch the next item before working on this one
        const unsigned it_next = it + stride;
        int vr_next = vr + stride_rows, chunk_next = chunk + stride_chunks;
        if (chunk_next >= nchunk) {
            chunk_next -= nchunk;
            ++vr_next;
        }
        uint4 vn[4];
        if (it_next < items) load(vr_next, chunk_next, vn);

        // block amax: exact BF16 max over the lane's 8 values (both halves), two
        // blocks per packed word, then over the half-warp
        uint32_t pm[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            pm[i] = quant::absmax_bf16x2(quant::absmax_bf16x2(v[i].x, v[i].y),
                                         quant::absmax_bf16x2(v[i].z, v[i].w));
            pm[i] = quant::absmax_bf16x2(pm[i], __byte_perm(pm[i], 0u, 0x1032));
        }
        uint32_t p01 = __byte_perm(pm[0], pm[1], 0x5410);
        uint32_t p23 = __byte_perm(pm[2], pm[3], 0x5410);
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) {
            p01 = quant::absmax_bf16x2(p01, __shfl_xor_sync(0xffffffffu, p01, o));
            p23 = quant::absmax_bf16x2(p23, __shfl_xor_sync(0xffffffffu, p23, o));
        }
        // scales: lane j of each half-warp divides for block j % 4 (one IEEE
        // division and one reciprocal per lane instead of four), then broadcasts
        const int own = lane & 3;
        const uint32_t pw = own < 2 ? p01 : p23;
        const uint32_t abits = ((own & 1) ? (pw >> 16) : pw) & 0x7FFFu;
        const float amax = __uint_as_float(abits << 16);
        const float s_own = amax == 0.0f ? 1.0f : __fdiv_rn(amax, 448.0f);
        const float r_own = kFastDiv ? __frcp_rn(s_own) : 0.0f;

        int g, row;
        locate(vr, g, row);
        uint2 *qr = p.q + (static_cast<size_t>(g) * p.rows + row) * row_chunks;   // 8-byte chunks
        float *sr = p.sfa + static_cast<size_t>(g) * p.num_kb * p.ld_sfa + row;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float s = __shfl_sync(0xffffffffu, s_own, (lane & 16) | i);
            const float r = kFastDiv ? __shfl_sync(0xffffffffu, r_own, (lane & 16) | i) : 0.0f;
            const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
            // the reciprocal path unless it is infinite (s below 2^-128) or the
            // all-division instantiation; a warp-uniform branch to the division
            const bool bad = !kFastDiv || !(r < INFINITY);
            uint2 c = make_uint2(0u, 0u);
            uint32_t d0 = 0u, d1 = 0u;   // bytes of elements next to an E4M3 midpoint
            if (kFastDiv) c = quant::codes8_fast(w, r, d0, d1);
            if (__any_sync(0xffffffffu, bad) && bad) {
                c = quant::codes8_div(w[0], w[1], w[2], w[3], s);
                d0 = d1 = 0u;
            }
            const int kb = chunk * kQuantBlocksPerWarp + 2 * i + half;
            if (kb < p.num_kb) {
                qr[static_cast<size_t>(kb) * 16 + l16] = c;
                if (l16 == 0) sr[static_cast<size_t>(kb) * p.ld_sfa] = s;
            }
            // elements next to an E4M3 midpoint (about 0.5% of BF16 data, so
            // most blocks have one somewhere in the warp): each lane settles
            // its own and rewrites their bytes after the 8-byte store
            if (kFastDiv && __any_sync(0xffffffffu, (d0 | d1) != 0u)) {
                uint64_t dw = (static_cast<uint64_t>(d1) << 32) | d0;
                uint8_t *qb = reinterpret_cast<uint8_t *>(qr + static_cast<size_t>(kb) * 16 + l16);
                while (dw != 0ull) {
                    const int j = (__ffsll(static_cast<long long>(dw)) - 1) >> 3;   // element 0..7
                    dw &= ~(0xFFull << (8 * j));
                    const uint32_t word = j < 2 ? w[0] : j < 4 ? w[1] : j < 6 ? w[2] : w[3];
                    const float xj = (j & 1) ? __uint_as_float(word & 0xFFFF0000u)
                                             : __uint_as_float(word << 16);
                    if (kb < p.num_kb) qb[j] = static_cast<uint8_t>(quant::code_near_midpoint(xj, s, r));
                }
            }
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) v[i] = vn[i];
        it = it_next;
        vr = vr_next;
        chunk = chunk_next;
    }
}

}  // namespace dg
