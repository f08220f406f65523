// gemm_kernel.cuh -- the sm_100a kernel of the FP8 block-scaled NT GEMM.
//
// One warp-specialised kernel template covers the three layouts (DeepGEMM
// pages: page 2 "六大核心技术突破" items 1, 4 and 5 -- TMA loads, persistent
// warp specialisation overlapping data movement, tensor-core MMA and CUDA-core
// promotion, one block scheduler for dense and grouped GEMMs; page 5 "03" --
// swapAB on Blackwell for skinny token matrices):
//
//   warp 0      producer: one thread issues TMA tile loads of both operands
//               for one 128-wide K-block per pipeline stage (128B swizzle).
//   warp 1      TMEM allocator + MMA issuer: one thread issues 4 x
//               tcgen05.mma.kind::f8f6f4 (K = 32 each) per K-block into a
//               fresh FP32 partial in TMEM (two partial buffers, ping-pong).
//   warps 2..9  promotion + epilogue (two warpgroups, each owning half of the
//               tile's columns): tcgen05.ld the partial, acc += (sA*sB)*P in
//               FP32 registers, release the partial; after the last K-block
//               convert to BF16 and store.
//
// Operand roles.  The MMA's "M" side is 128 TMEM lanes; its "N" side is kBN
// columns.  Normal mode puts 128 token rows of A on lanes and kBN weight rows
// of B on columns.  Swap-AB mode (small token counts) computes D^T = B * A^T:
// 128 weight rows on lanes, kBN token rows on columns, so a 64-token decode
// batch does not waste half of a 128-lane MMA.  Both operands stay K-major.
//
// Split-K (swap mode only): a cluster of `split` CTAs shares one output tile,
// each CTA takes a contiguous range of K-blocks, and the FP32 partial tiles
// are summed in a fixed order through distributed shared memory -- no global
// workspace.  This fills the 148 SMs at decode shapes (17 tiles at N = 2112).
//
// Every wait is bounded (BoundedWait): after `timeout_cycles` the waiting
// thread records DG_ERR_TIMEOUT in the device status word, raises a CTA-wide
// abort flag and the kernel winds down (waiting, again bounded, for its own
// TMA loads and MMAs in flight, then freeing TMEM) instead of hanging.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"

namespace dg {

enum Layout : int { kDense = 0, kContiguous = 1, kMasked = 2 };

constexpr int kBlockK = 128;         // K-block (one 128-byte swizzled row of FP8)
constexpr int kTileX = 128;          // MMA M (TMEM lanes)
constexpr int kMaxGroups = 1024;     // masked layout, group prefix table in smem
constexpr int kNumThreads = 320;     // 10 warps
constexpr int kMinSmem = 120 * 1024; // > half an SM: one CTA per SM (TMEM is never contended)

// status word layout: low 8 bits = dg_status_t code, bits 8..15 = site, bits 16..31 = CTA
enum StatusCode : unsigned { kStatusInvalid = 1u, kStatusTimeout = 6u };
enum Site : unsigned {
    kSiteProducerEmpty = 1, kSiteMmaTmemEmpty = 2, kSiteMmaFull = 3, kSitePromoFull = 4,
    kSiteTeardownLoads = 5, kSiteTeardownMma = 6, kSiteBadGroup = 7, kSiteBadMask = 8
};

struct Params {
    const float *sfa;
    const float *sfb;
    __nv_bfloat16 *d;
    const int32_t *m_indices;   // contiguous
    const int32_t *masked_m;    // masked
    unsigned *status;           // device status word
    long long timeout_cycles;
    int ld_sfa;
    int M;      // dense: M; contiguous: M_total; masked: Mmax
    int N, K, G;
    int num_kb, num_nb;
    int split;  // CTAs per cluster along K (swap mode); 1 = persistent
    int debug_flags;
};

constexpr int kDebugProducerIdle = 1;   // fault injection: the producer never loads

__device__ __forceinline__ void record_status(unsigned *status, unsigned code, unsigned site) {
    unsigned v = code | (site << 8) | ((blockIdx.x + gridDim.x * blockIdx.y) << 16);
    atomicCAS(status, 0u, v);
}

struct BoundedWait {
    volatile int *abort_flag;
    unsigned *status;
    long long limit;

    // Returns true when the phase completed; false on timeout or abort.
    __device__ __forceinline__ bool operator()(uint32_t bar, uint32_t parity, unsigned site) const {
        if (ptx::mbar_try_wait(bar, parity)) return true;
        const long long start = clock64();
        while (true) {
            if (ptx::mbar_try_wait(bar, parity)) return true;
            if (*abort_flag) return false;
            if (clock64() - start > limit) {
                record_status(status, kStatusTimeout, site);
                *abort_flag = 1;
                return false;
            }
        }
    }
};

// K-major, 128-byte swizzle smem matrix descriptor (tcgen05 format): start
// address, leading offset 16 B (unused for this swizzle), 1024 B between
// 8-row core groups, version 1, layout SWIZZLE_128B.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr & 0x3FFFF) >> 4);
    d |= static_cast<uint64_t>(16 >> 4) << 16;
    d |= static_cast<uint64_t>(1024 >> 4) << 32;
    d |= static_cast<uint64_t>(1) << 46;
    d |= static_cast<uint64_t>(2) << 61;
    return d;
}

// Instruction descriptor: D = F32, A = B = E4M3, both K-major, M = 128, N = n.
__host__ __device__ constexpr uint32_t f8_idesc(int n) {
    return (1u << 4) | (static_cast<uint32_t>(n >> 3) << 17) |
           (static_cast<uint32_t>(kTileX >> 4) << 24);
}

struct Tile {
    int g;       // group: B and sfb index
    int a_row;   // A tensor-map row coordinate of the tile's first token
    int a_grp;   // A tensor-map outer coordinate (masked: g, else 0)
    int tok0;    // first token row (within the group's rows)
    int tok_end; // exclusive bound of valid token rows
    int n0;      // first weight row
    int ntok;    // token rows of this tile that exist: min(rows per tile, tok_end - tok0)
};

template <int kBN, bool kSwap, int kLayout>
struct TileMap {
    static constexpr int kTokRows = kSwap ? kBN : kTileX;     // token rows per tile
    static constexpr int kWRows = kSwap ? kTileX : kBN;       // weight rows per tile
    static constexpr int kRasterM = 16;                       // L2 raster band (token blocks)

    // Number of tiles (masked: from the smem prefix table).
    __device__ static int count(const Params &p, const int *prefix) {
        const int nw = (p.N + kWRows - 1) / kWRows;
        if (kLayout == kMasked) return prefix[p.G];
        const int nt = (p.M + kTokRows - 1) / kTokRows;
        return nt * nw;
    }

    // Decode tile t; false means the tile has no work (contiguous padding block).
    __device__ static bool decode(int t, const Params &p, const int *prefix, Tile &tl) {
        const int nw = (p.N + kWRows - 1) / kWRows;
        int tb, wb;
        if (kLayout == kMasked) {
            int lo = 0, hi = p.G - 1;                // last g with prefix[g] <= t
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (prefix[mid] <= t) lo = mid; else hi = mid - 1;
            }
            const int g = lo, local = t - prefix[g];
            tb = local / nw;
            wb = local - tb * nw;
            int mm = p.masked_m[g];
            mm = mm < 0 ? 0 : (mm > p.M ? p.M : mm);
            tl.g = g;
            tl.a_grp = g;
            tl.tok0 = tb * kTokRows;
            tl.a_row = tl.tok0;
            tl.tok_end = mm;
            tl.n0 = wb * kWRows;
            tl.ntok = min(kTokRows, mm - tl.tok0);
            return true;
        }
        const int nt = (p.M + kTokRows - 1) / kTokRows;
        if (kSwap) {
            tb = t / nw;
            wb = t - tb * nw;
        } else {
            const int per_band = kRasterM * nw;
            const int band = t / per_band;
            const int first = band * kRasterM;
            const int width = min(kRasterM, nt - first);
            const int local = t - band * per_band;
            tb = first + local % width;
            wb = local / width;
        }
        tl.tok0 = tb * kTokRows;
        tl.a_row = tl.tok0;
        tl.a_grp = 0;
        tl.tok_end = p.M;
        tl.n0 = wb * kWRows;
        tl.ntok = min(kTokRows, p.M - tl.tok0);
        tl.g = 0;
        if (kLayout == kContiguous) {
            const int g = __ldg(p.m_indices + tl.tok0);
            if (g < 0) return false;
            if (g >= p.G) return false;     // recorded by the producer
            tl.g = g;
        }
        return true;
    }
};

template <int kBN, bool kSwap, int kStages>
struct SmemLayout {
    static constexpr int kXBytes = kTileX * kBlockK;       // 16 KB
    static constexpr int kYBytes = kBN * kBlockK;
    static constexpr int kStageBytes = kXBytes + kYBytes;
    static constexpr int kStagesBytes = kStages * kStageBytes;
    // Per-stage scale slot: the tile's token-row scales sA[kb][tok0 ...] (one
    // float per token row), then the weight-block scale(s) sB[wblk][kb].
    static constexpr int kScaleRows = kSwap ? kBN : kTileX;
    static constexpr int kSlotFloats = kScaleRows + 4;
    static constexpr int kSlotBytes = kSlotFloats * 4;
    static constexpr int kSlotOffset = kStagesBytes;
    static constexpr int kBarOffset = kSlotOffset + kStages * kSlotBytes;
    static constexpr int kNumBars = 2 * kStages + 2 + 2 + 1;
    static constexpr int kMiscOffset = kBarOffset + kNumBars * 8;     // tmem addr, abort flag
    static constexpr int kPrefixOffset = (kMiscOffset + 16 + 15) / 16 * 16;
    static constexpr int kPrefixBytes = (kMaxGroups + 1) * 4;
    static constexpr int kUsed = kPrefixOffset + kPrefixBytes;
    static constexpr int kAlloc = (kUsed + 1024 > kMinSmem) ? kUsed + 1024 : kMinSmem;
    static constexpr int kTmemCols = 2 * kBN < 32 ? 32 : 2 * kBN;
    static_assert(kStageBytes % 1024 == 0, "stage must keep 1024-byte alignment");
    static_assert(kSlotBytes % 16 == 0, "bulk copies need 16-byte aligned slots");
    static_assert(kStagesBytes >= kTileX * kBN * 4, "split-K receive buffer reuses the stages");
    static_assert(kAlloc <= 227 * 1024, "shared memory budget");
    static_assert((kTmemCols & (kTmemCols - 1)) == 0, "TMEM allocation is a power of two");
};

template <int kBN, bool kSwap, int kStages, int kLayout>
__global__ void __launch_bounds__(kNumThreads, 1)
fp8_gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                const Params p) {
    using L = SmemLayout<kBN, kSwap, kStages>;
    using TM = TileMap<kBN, kSwap, kLayout>;
    static_assert(kBN == 64 || kBN == 128 || kBN == 256, "tile N");
    static_assert(kSwap || kLayout != kMasked, "masked layout runs in swap mode");
    constexpr int kHalf = kBN / 2;               // columns per promotion warpgroup
    constexpr int kChunk = kHalf > 64 ? 16 : 32; // TMEM columns per load (register budget)
    constexpr int kChunks = kHalf / kChunk;
    constexpr int kNumSB = (!kSwap && kBN == 256) ? 2 : 1;   // weight blocks per tile
    constexpr int kTokBox = 32;                               // swap mode: token rows per TMA box

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t s_base = ptx::smem_u32(smem);
    const uint32_t bar_base = s_base + L::kBarOffset;
    auto full_bar = [&](int s) { return bar_base + 8u * s; };
    auto empty_bar = [&](int s) { return bar_base + 8u * (kStages + s); };
    auto tfull_bar = [&](int b) { return bar_base + 8u * (2 * kStages + b); };
    auto tempty_bar = [&](int b) { return bar_base + 8u * (2 * kStages + 2 + b); };
    const uint32_t mma_done_bar = bar_base + 8u * (2 * kStages + 4);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kMiscOffset);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::kMiscOffset + 4);
    const uint32_t slot_base = s_base + L::kSlotOffset;
    const float *slots = reinterpret_cast<const float *>(smem + L::kSlotOffset);
    int *prefix = reinterpret_cast<int *>(smem + L::kPrefixOffset);

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    const BoundedWait wait{abort_flag, p.status, p.timeout_cycles};

    // ------------------------------------------------------------ set-up
    if (threadIdx.x == 0) {
        ptx::prefetch_tmap(&tm_a);
        ptx::prefetch_tmap(&tm_b);
        for (int s = 0; s < kStages; ++s) {
            ptx::mbar_init(full_bar(s), 1);
            ptx::mbar_init(empty_bar(s), 1 + 8);   // MMA commit + 8 promotion warps (scales read)
        }
        for (int b = 0; b < 2; ++b) {
            ptx::mbar_init(tfull_bar(b), 1);
            ptx::mbar_init(tempty_bar(b), 8);
        }
        ptx::mbar_init(mma_done_bar, 1);
        *abort_flag = 0;
        ptx::fence_mbar_init();
    }
    if (kLayout == kMasked && warp == 2) {
        // exclusive prefix of tiles per group: ceil(masked_m[g] / kTokRows) * weight blocks
        const int nw = (p.N + TM::kWRows - 1) / TM::kWRows;
        int carry = 0;
        for (int base = 0; base < p.G; base += 32) {
            const int g = base + lane;
            int tiles = 0;
            if (g < p.G) {
                int mm = __ldg(p.masked_m + g);
                if (mm < 0 || mm > p.M) {
                    record_status(p.status, kStatusInvalid, kSiteBadMask);
                    mm = mm < 0 ? 0 : p.M;
                }
                tiles = (mm + TM::kTokRows - 1) / TM::kTokRows * nw;
            }
            int incl = tiles;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int v = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += v;
            }
            if (g < p.G) prefix[g] = carry + incl - tiles;
            carry += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) prefix[p.G] = carry;
    }
    if (warp == 1) {
        ptx::tmem_alloc(ptx::smem_u32(tmem_slot), L::kTmemCols);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    // tile iteration: persistent (split == 1) or one tile per cluster (split > 1)
    const bool clustered = p.split > 1;
    const int num_tiles = clustered ? static_cast<int>(gridDim.y) : TM::count(p, prefix);
    const int t_first = clustered ? static_cast<int>(blockIdx.y) : static_cast<int>(blockIdx.x);
    const int t_step = clustered ? num_tiles : static_cast<int>(gridDim.x);
    int kb_begin = 0, kb_end = p.num_kb;
    if (clustered) {
        const int r = static_cast<int>(ptx::cluster_rank());
        kb_begin = (p.num_kb * r) / p.split;
        kb_end = (p.num_kb * (r + 1)) / p.split;
    }

    if (warp == 0) {
        // ======================================================== producer
        if (ptx::elect_one()) {
            int stage = 0;
            uint32_t phase = 0;
            long long issued = 0;
            bool ok = (p.debug_flags & kDebugProducerIdle) == 0;
            for (int t = t_first; ok && t < num_tiles; t += t_step) {
                Tile tl;
                if (!TM::decode(t, p, prefix, tl)) {
                    if (kLayout == kContiguous && __ldg(p.m_indices + tl.tok0) >= p.G)
                        record_status(p.status, kStatusInvalid, kSiteBadGroup);
                    continue;
                }
                const float *sfa_g = p.sfa + (kLayout == kMasked ? static_cast<size_t>(tl.g) * p.num_kb * p.ld_sfa : 0);
                const float *sfb_g = p.sfb + static_cast<size_t>(tl.g) * p.num_nb * p.num_kb;
                const int wblk0 = tl.n0 / 128;
                // token-row scales present in memory for this tile (ld_sfa - tok0 is a multiple of 4)
                // swap mode fetches only the tile's token rows, in boxes of kTokBox rows
                const int nload = kSwap ? (tl.ntok + kTokBox - 1) / kTokBox : 1;
                const uint32_t y_bytes = kSwap ? static_cast<uint32_t>(nload * kTokBox * kBlockK)
                                               : static_cast<uint32_t>(L::kYBytes);
                const int sa_rows = min(kSwap ? nload * kTokBox : L::kScaleRows, p.ld_sfa - tl.tok0);
                const uint32_t sa_bytes = static_cast<uint32_t>(sa_rows) * 4u;
                for (int kb = kb_begin; kb < kb_end; ++kb) {
                    if (!wait(empty_bar(stage), phase ^ 1u, kSiteProducerEmpty)) { ok = false; break; }
                    const uint32_t sx = s_base + stage * L::kStageBytes;
                    const uint32_t sy = sx + L::kXBytes;
                    const uint32_t slot = slot_base + stage * L::kSlotBytes;
#pragma unroll
                    for (int i = 0; i < kNumSB; ++i) {
                        const uint32_t dst = slot + (L::kScaleRows + i) * 4u;
                        if (wblk0 + i < p.num_nb)
                            ptx::cp_async_4(dst, sfb_g + static_cast<size_t>(wblk0 + i) * p.num_kb + kb);
                        else
                            ptx::st_shared_f32(dst, 0.f);
                    }
                    ptx::cp_async_arrive(full_bar(stage));
                    ptx::mbar_arrive_expect_tx(full_bar(stage), L::kXBytes + y_bytes + sa_bytes);
                    ptx::bulk_load(slot, sfa_g + static_cast<size_t>(kb) * p.ld_sfa + tl.tok0, sa_bytes,
                                   full_bar(stage));
                    if (kSwap) {
                        ptx::tma_load_3d(sx, &tm_b, full_bar(stage), kb * kBlockK, tl.n0, tl.g);
                        for (int i = 0; i < nload; ++i)
                            ptx::tma_load_3d(sy + i * kTokBox * kBlockK, &tm_a, full_bar(stage), kb * kBlockK,
                                             tl.a_row + i * kTokBox, tl.a_grp);
                    } else {
                        ptx::tma_load_3d(sx, &tm_a, full_bar(stage), kb * kBlockK, tl.a_row, tl.a_grp);
                        ptx::tma_load_3d(sy, &tm_b, full_bar(stage), kb * kBlockK, tl.n0, tl.g);
                    }
                    ++issued;
                    if (++stage == kStages) { stage = 0; phase ^= 1u; }
                }
            }
            // wind-down: never leave with TMA writes into this CTA's smem in flight
            // (the last kStages loads sit on distinct stages)
            const long long first = issued > kStages ? issued - kStages : 0;
            for (long long i = first; i < issued; ++i) {
                const int s = static_cast<int>(i % kStages);
                const uint32_t par = static_cast<uint32_t>((i / kStages) & 1);
                const long long start = clock64();
                while (!ptx::mbar_try_wait(full_bar(s), par)) {
                    if (clock64() - start > p.timeout_cycles) {
                        record_status(p.status, kStatusTimeout, kSiteTeardownLoads);
                        break;
                    }
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ======================================================== MMA issuer
        if (ptx::elect_one()) {
            int stage = 0, buf = 0;
            uint32_t phase = 0, tphase = 0;
            bool issued_any = false;
            bool ok = true;
            for (int t = t_first; ok && t < num_tiles; t += t_step) {
                Tile tl;
                if (!TM::decode(t, p, prefix, tl)) continue;
                const uint32_t idesc =
                    f8_idesc(kSwap ? (tl.ntok + kTokBox - 1) / kTokBox * kTokBox : kBN);
                for (int kb = kb_begin; kb < kb_end; ++kb) {
                    if (!wait(tempty_bar(buf), tphase ^ 1u, kSiteMmaTmemEmpty)) { ok = false; break; }
                    if (!wait(full_bar(stage), phase, kSiteMmaFull)) { ok = false; break; }
                    ptx::tc_fence_after();
                    const uint32_t sx = s_base + stage * L::kStageBytes;
                    const uint64_t dx = sw128_desc(sx);
                    const uint64_t dy = sw128_desc(sx + L::kXBytes);
                    const uint32_t dtm = tmem_base + static_cast<uint32_t>(buf * kBN);
#pragma unroll
                    for (int k = 0; k < kBlockK / 32; ++k)
                        ptx::mma_f8f6f4(dtm, dx + 2u * k, dy + 2u * k, idesc, k > 0 ? 1u : 0u);
                    ptx::mma_commit(empty_bar(stage));
                    ptx::mma_commit(tfull_bar(buf));
                    issued_any = true;
                    if (++stage == kStages) { stage = 0; phase ^= 1u; }
                    if (++buf == 2) { buf = 0; tphase ^= 1u; }
                }
            }
            if (issued_any) {
                // all MMAs of this thread complete before TMEM is released
                ptx::mma_commit(mma_done_bar);
                const long long start = clock64();
                while (!ptx::mbar_try_wait(mma_done_bar, 0)) {
                    if (clock64() - start > p.timeout_cycles) {
                        record_status(p.status, kStatusTimeout, kSiteTeardownMma);
                        break;
                    }
                }
            }
        }
        __syncwarp();
    }

    // ============================================================ promotion
    // (warps 2..9; warps 0 and 1 skip straight to the split-K barriers)
    //
    // Column ownership.  Normal mode: warpgroup h owns the contiguous columns
    // [h*kHalf, (h+1)*kHalf) (with kBN = 256 that is exactly one 128-row
    // weight block, so one sB per thread).  Swap mode: columns are tokens and
    // the tile may hold fewer than kBN of them, so the chunks of kChunk columns
    // are dealt alternately (chunk 2c+h to warpgroup h) to keep both
    // warpgroups busy; chunks past the tile's token count are skipped.
    float acc[kHalf];
    const bool promo = warp >= 2;
    const int quarter = warp & 3;                    // TMEM lane quarter this warp may access
    const int half = promo ? (warp - 2) >> 2 : 0;    // warpgroup
    const int lrow = quarter * 32 + lane;            // tile row = TMEM lane
    auto col_of = [&](int c) {                       // first tile column of local chunk c
        return kSwap ? (2 * c + half) * kChunk : half * kHalf + c * kChunk;
    };
    Tile last_tile{0, 0, 0, 0, 0, 0, 0};
    bool have_tile = false;
    int last_nvalid = 0;
    if (promo) {
        int stage = 0, buf = 0;
        uint32_t phase = 0, tphase = 0;
        bool ok = true;
        for (int t = t_first; ok && t < num_tiles; t += t_step) {
            Tile tl;
            if (!TM::decode(t, p, prefix, tl)) continue;
#pragma unroll
            for (int i = 0; i < kHalf; ++i) acc[i] = 0.f;
            const int my_tok = tl.tok0 + lrow;       // normal mode: this thread's token row
            const bool tok_ok = my_tok < tl.tok_end;
            // chunks of this warpgroup that hold columns of the tile
            const int ncols = kSwap ? (tl.ntok + kTokBox - 1) / kTokBox * kTokBox : kBN;
            const int nvalid = kSwap ? (ncols / kChunk - half + 1) / 2 : kChunks;
            for (int kb = kb_begin; kb < kb_end; ++kb) {
                // the stage's scales: visible once its full barrier completed
                if (!wait(full_bar(stage), phase, kSitePromoFull)) { ok = false; break; }
                const float *slot = slots + stage * L::kSlotFloats;
                float s = 0.f, sb = 0.f;
                if (!kSwap) {
                    s = slot[lrow] * slot[L::kScaleRows + (kNumSB == 2 ? half : 0)];
                    __syncwarp();
                    if (lane == 0) ptx::mbar_arrive(empty_bar(stage));
                } else {
                    sb = slot[L::kScaleRows];
                }
                if (!wait(tfull_bar(buf), tphase, kSitePromoFull)) { ok = false; break; }
                ptx::tc_fence_after();
                const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                                       static_cast<uint32_t>(buf * kBN);
                if (nvalid == 0) {
                    ptx::tc_fence_before();
                    __syncwarp();
                    if (lane == 0) ptx::mbar_arrive(tempty_bar(buf));
                }
#pragma unroll
                for (int c = 0; c < kChunks; ++c) {
                    if (c < nvalid) {
                        float v[kChunk];
                        if constexpr (kChunk == 32) ptx::tmem_ld32(taddr + col_of(c), v);
                        else ptx::tmem_ld16(taddr + col_of(c), v);
                        ptx::tmem_wait_ld();
                        if (c == nvalid - 1) {
                            ptx::tc_fence_before();
                            __syncwarp();
                            if (lane == 0) ptx::mbar_arrive(tempty_bar(buf));
                        }
                        float *a = acc + c * kChunk;
                        if (kSwap) {
                            // column (token) scales, broadcast from the slot
                            const float4 *sc = reinterpret_cast<const float4 *>(slot + col_of(c));
#pragma unroll
                            for (int i = 0; i < kChunk / 4; ++i) {
                                const float4 q4 = sc[i];
                                a[4 * i + 0] = fmaf(q4.x * sb, v[4 * i + 0], a[4 * i + 0]);
                                a[4 * i + 1] = fmaf(q4.y * sb, v[4 * i + 1], a[4 * i + 1]);
                                a[4 * i + 2] = fmaf(q4.z * sb, v[4 * i + 2], a[4 * i + 2]);
                                a[4 * i + 3] = fmaf(q4.w * sb, v[4 * i + 3], a[4 * i + 3]);
                            }
                        } else {
#pragma unroll
                            for (int i = 0; i < kChunk; ++i) a[i] = fmaf(s, v[i], a[i]);
                        }
                    }
                }
                if (kSwap) {
                    __syncwarp();
                    if (lane == 0) ptx::mbar_arrive(empty_bar(stage));
                }
                if (++stage == kStages) { stage = 0; phase ^= 1u; }
                if (++buf == 2) { buf = 0; tphase ^= 1u; }
            }
            if (!ok) break;
            last_tile = tl;
            last_nvalid = nvalid;
            have_tile = true;
            if (clustered) break;   // one tile; reduced below
            // ------------------------------------------------ epilogue (direct)
            const size_t row_base = kLayout == kMasked ? static_cast<size_t>(tl.g) * p.M : 0;
            if (!kSwap) {
                if (tok_ok) {
                    __nv_bfloat16 *drow = p.d + (row_base + my_tok) * static_cast<size_t>(p.N);
#pragma unroll
                    for (int j = 0; j < kHalf; j += 8) {
                        const int col = tl.n0 + half * kHalf + j;
                        if (col < p.N) {
                            uint4 pk;
                            __nv_bfloat162 h0 = __floats2bfloat162_rn(acc[j + 0], acc[j + 1]);
                            __nv_bfloat162 h1 = __floats2bfloat162_rn(acc[j + 2], acc[j + 3]);
                            __nv_bfloat162 h2 = __floats2bfloat162_rn(acc[j + 4], acc[j + 5]);
                            __nv_bfloat162 h3 = __floats2bfloat162_rn(acc[j + 6], acc[j + 7]);
                            pk.x = *reinterpret_cast<uint32_t *>(&h0);
                            pk.y = *reinterpret_cast<uint32_t *>(&h1);
                            pk.z = *reinterpret_cast<uint32_t *>(&h2);
                            pk.w = *reinterpret_cast<uint32_t *>(&h3);
                            *reinterpret_cast<uint4 *>(drow + col) = pk;
                        }
                    }
                }
            } else {
                const int n = tl.n0 + lrow;
                if (n < p.N) {
#pragma unroll
                    for (int c = 0; c < kChunks; ++c) {
                        if (c < nvalid) {
#pragma unroll
                            for (int i = 0; i < kChunk; ++i) {
                                const int m = tl.tok0 + col_of(c) + i;
                                if (m < tl.tok_end)
                                    p.d[(row_base + m) * static_cast<size_t>(p.N) + n] =
                                        __float2bfloat16_rn(acc[c * kChunk + i]);
                            }
                        }
                    }
                }
            }
        }
    }

    // ============================================================ split-K reduction
    if (clustered) {
        // (1) every CTA of the cluster is done with its main loop: stage memory is idle
        __syncwarp();
        ptx::cluster_sync_all();
        const int split = p.split;
        const int rows_per = kTileX / split;             // split divides 128 (1,2,4,8)
        const uint32_t my_rank = ptx::cluster_rank();
        if (promo && have_tile && !*abort_flag) {
            // (2) send this thread's row to its owner: slot [src rank][row % rows_per][column]
            const int owner = lrow / rows_per;
            const uint32_t local = s_base + static_cast<uint32_t>(
                ((my_rank * rows_per + (lrow % rows_per)) * kBN) * 4);
            const uint32_t remote = ptx::map_cluster(local, static_cast<uint32_t>(owner));
#pragma unroll
            for (int c = 0; c < kChunks; ++c) {
                if (c < last_nvalid) {
#pragma unroll
                    for (int i = 0; i < kChunk; i += 4)
                        ptx::st_cluster_v4(remote + (col_of(c) + i) * 4, acc[c * kChunk + i],
                                           acc[c * kChunk + i + 1], acc[c * kChunk + i + 2],
                                           acc[c * kChunk + i + 3]);
                }
            }
        }
        ptx::cluster_sync_all();
        // (3) each CTA sums its rows over the source ranks in rank order and stores
        if (promo && have_tile) {
            const float *recv = reinterpret_cast<const float *>(smem);
            const Tile &tl = last_tile;
            const size_t row_base = kLayout == kMasked ? static_cast<size_t>(tl.g) * p.M : 0;
            const int tid = (warp - 2) * 32 + lane;        // 0..255
            const int elems = rows_per * tl.ntok;
            for (int e = tid; e < elems; e += 256) {
                const int rr = e % rows_per;               // consecutive threads: consecutive n
                const int j = e / rows_per;
                float sum = 0.f;
                for (int src = 0; src < split; ++src) sum += recv[(src * rows_per + rr) * kBN + j];
                const int n = tl.n0 + static_cast<int>(my_rank) * rows_per + rr;
                const int m = tl.tok0 + j;
                if (n < p.N && m < tl.tok_end)
                    p.d[(row_base + m) * static_cast<size_t>(p.N) + n] = __float2bfloat16_rn(sum);
            }
        }
    }

    // ============================================================ teardown
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem_base, L::kTmemCols);
    }
}

}  // namespace dg
