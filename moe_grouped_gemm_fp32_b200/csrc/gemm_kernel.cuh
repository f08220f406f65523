// gemm_kernel.cuh -- the sm_100a kernel of the FP8 block-scaled NT GEMM.
//
// One warp-specialised kernel template covers the three layouts (DeepGEMM
// pages: page 2 "六大核心技术突破" items 1, 4 and 5 -- TMA loads, persistent
// warp specialisation overlapping data movement, tensor-core MMA and CUDA-core
// promotion, one block scheduler for dense and grouped GEMMs; page 5 "03" --
// swapAB on Blackwell for skinny token matrices; the 2-CTA pair below is the
// Blackwell counterpart of the pages' TMA multicast of a shared operand):
//
//   warp 0      producer: one thread issues, per 128-wide K-block and pipeline
//               stage, TMA tile loads of both operands (128B swizzle), a bulk
//               copy of the tile's activation scales and cp.async of the
//               weight-block scale(s) into the stage's scale slot.
//   warp 1      TMEM allocator + MMA issuer: one thread issues 4 x
//               tcgen05.mma.kind::f8f6f4 (K = 32 each) per K-block into a
//               fresh FP32 partial in TMEM (2-4 partial buffers in rotation).
//   warps 2..9  promotion + epilogue (two warpgroups): read the stage's
//               scales, tcgen05.ld the partial, acc += (sA*sB)*P in FP32
//               registers, release the partial; after the last K-block
//               convert to BF16 and store.
//
// Operand roles.  The MMA's "M" side is 128 TMEM lanes per CTA; its "N" side
// is kBN columns.  Normal mode puts 128 token rows of A on lanes and kBN
// weight rows of B on columns.  Swap-AB mode (small token counts) computes
// D^T = B * A^T: 128 weight rows on lanes, up to kBN token rows on columns, so
// a 64-token decode batch does not waste half of a 128-lane MMA; only the
// token rows present are fetched (32-row boxes) and multiplied (MMA N set per
// tile).  Both operands stay K-major.
//
// CTA pairs (kCtaGroup == 2, normal mode): a cluster of 2 CTAs computes one
// 256 x kBN tile with tcgen05.mma.cta_group::2.  Each CTA stages its own 128
// token rows and half of the tile's weight rows, so a stage costs each SM
// 16 KB + kBN/2 x 128 B instead of 16 KB + kBN x 128 B: twice the MMA work
// per byte held in shared memory and per byte pulled from L2.  The even CTA
// issues the MMAs; TMA bytes of both CTAs complete on its barrier, and the
// MMA completions are multicast to both CTAs' barriers.
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

enum Layout : int { kDense = 0, kContiguous = 1, kMasked = 2, kKGrouped = 3 };

constexpr int kBlockK = 128;         // K-block (one 128-byte swizzled row of FP8)
constexpr int kTileX = 128;          // MMA M per CTA (TMEM lanes)
constexpr int kMaxGroups = 1024;     // masked layout, group prefix table in smem
// Swap mode: 11 warps (producer, MMA, 8 promotion, scale preparation).
// Normal mode: 12 warps; warps 0-3 (producer, MMA, two idle) hand registers
// to the two promotion warpgroups (setmaxnreg), which keep up to 128
// accumulators per thread plus a TMEM batch.
__host__ __device__ constexpr int num_threads(bool swap) { return swap ? 352 : 384; }
constexpr int kPrepWarp = 10;        // swap mode: multiplies token scales by the weight scale
constexpr int kRegsLaunch = 168;     // normal mode: per-thread registers at launch (65536 / 384)
constexpr int kRegsIssue = 56;       // producer / MMA warpgroup after rebalancing
constexpr int kRegsPromo = 224;      // promotion warpgroups after rebalancing
static_assert(128 * (kRegsLaunch - kRegsIssue) == 256 * (kRegsPromo - kRegsLaunch),
              "register rebalancing must add up to the launch pool");
constexpr int kMinSmem = 120 * 1024; // > half an SM: one CTA per SM (TMEM is never contended)
constexpr int kTokBox = 32;          // swap mode: token rows per TMA box

// status word layout: low 8 bits = dg_status_t code, bits 8..15 = site, bits 16..31 = CTA
enum StatusCode : unsigned { kStatusInvalid = 1u, kStatusTimeout = 6u };
enum Site : unsigned {
    kSiteProducerEmpty = 1, kSiteMmaTmemEmpty = 2, kSiteMmaFull = 3, kSitePromoFull = 4,
    kSiteTeardownLoads = 5, kSiteTeardownMma = 6, kSiteBadGroup = 7, kSiteBadMask = 8, kSiteBadKs = 10,
    kSiteSplitKRecv = 11
};

struct Params {
    const float *sfa;
    const float *sfb;
    __nv_bfloat16 *d;
    const int32_t *m_indices;   // contiguous
    const int32_t *masked_m;    // masked
    const int32_t *ks;          // K-grouped: K columns per group (device)
    unsigned *status;           // device status word
    long long timeout_cycles;
    int ld_sfa;
    int M;      // dense: M; contiguous: M_total; masked: Mmax
    int N, K, G;
    int num_kb, num_nb;
    int split;  // CTAs per cluster along K (swap mode); 1 = persistent
    int debug_flags;
    // SwiGLU-quantise epilogue (fused expert FFN, first GEMM): E4M3 codes
    // [rows][N/2] and FP32 scales [N/256][ld_s_out] of silu(gate) * up
    uint8_t *q_out;
    float *s_out;
    int ld_s_out;
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

    // Returns true when the phase completed; false on timeout or abort.  Each
    // probe may sleep up to ~20 us waiting for the phase, so the deadline and the
    // abort flag are checked every few microseconds at most.
    __device__ __forceinline__ bool operator()(uint32_t bar, uint32_t parity, unsigned site) const {
        if (ptx::mbar_try_wait(bar, parity)) return true;
        const long long start = clock64();
        while (true) {
            if (ptx::mbar_try_wait_sleep(bar, parity, 20000u)) return true;
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

// Instruction descriptor: D = F32, A = B = E4M3, both K-major, M = m, N = n.
__host__ __device__ constexpr uint32_t f8_idesc(int m, int n) {
    return (1u << 4) | (static_cast<uint32_t>(n >> 3) << 17) | (static_cast<uint32_t>(m >> 4) << 24);
}

// Weight-block scales a tile of bn weight rows starting at a multiple of bn
// can touch (bn = 224 tiles start at multiples of 32 inside a block).
__host__ __device__ constexpr int weight_blocks_per_tile(int bn) {
    return (128 % bn == 0) ? 1 : (bn % 128 == 0 ? bn / 128 : bn / 128 + 2);
}

struct Tile {
    int g;       // group: B and sfb index
    int a_row;   // A tensor-map row coordinate of the tile's first token
    int a_grp;   // A tensor-map outer coordinate (masked: g, else 0)
    int tok0;    // first token row (within the group's rows)
    int tok_end; // exclusive bound of valid token rows
    int n0;      // first weight row
    int ntok;    // token rows of this tile that exist: min(rows per tile, tok_end - tok0)
    int store;   // CTA-pair tiles: bit r set = CTA r of the pair stores its rows
    int b_grp;   // B tensor-map outer coordinate and sfb group (K-grouped: 0)
    int kb0;     // the tile's K-blocks [kb0, kb1) (K-grouped: its group's)
    int kb1;
};

template <int kBN, bool kSwap, int kLayout, int kCtaGroup>
struct TileMap {
    static constexpr int kTokRows = kSwap ? kBN : kTileX * kCtaGroup;  // token rows per tile
    static constexpr int kWRows = kSwap ? kTileX : kBN;                // weight rows per tile
    static constexpr int kRasterM = 16 / kCtaGroup;                    // L2 raster band (token blocks)

    // Contiguous layout in CTA pairs: a pair tile covers two 128-row blocks.
    // When the two blocks belong to different groups, the tile runs twice: the
    // first pass (group of block 0) stores block 0's rows, a second pass (group
    // of block 1), listed after all first passes, stores block 1's rows.  The
    // pairs that need a second pass are listed in prefix[0..Q), Q in
    // prefix[kMaxGroups] (built at kernel set-up).
    static constexpr bool kPairedGroups = kLayout == kContiguous && kCtaGroup == 2;
    __device__ static int block_group(const Params &p, int blk) {
        if (blk >= p.M / kTileX) return -1;
        const int g = __ldg(p.m_indices + static_cast<size_t>(blk) * kTileX);
        return g < p.G ? g : -1;
    }

    // Number of tiles (masked: from the smem prefix table).
    __device__ static int count(const Params &p, const int *prefix) {
        const int nw = (p.N + kWRows - 1) / kWRows;
        if (kLayout == kMasked) return prefix[p.G];
        if (kLayout == kKGrouped) return p.G * ((p.M + kTokRows - 1) / kTokRows) * nw;
        if (kPairedGroups) {
            const int npairs = (p.M / kTileX + 1) / 2;
            return (npairs + prefix[kMaxGroups]) * nw;
        }
        const int nt = (p.M + kTokRows - 1) / kTokRows;
        return nt * nw;
    }

    // Decode tile t; false means the tile has no work (contiguous padding block).
    __device__ static bool decode(int t, const Params &p, const int *prefix, Tile &tl) {
        const int nw = (p.N + kWRows - 1) / kWRows;
        int tb, wb;
        tl.kb0 = 0;
        tl.kb1 = p.num_kb;
        if (kLayout == kKGrouped) {
            // group-major; inside a group the dense raster (bands of token blocks)
            const int nt = (p.M + kTokRows - 1) / kTokRows;
            const int g = t / (nt * nw);
            const int local_t = t - g * nt * nw;
            const int per_band = kRasterM * nw;
            const int band = local_t / per_band;
            const int first = band * kRasterM;
            const int width = min(kRasterM, nt - first);
            const int local = local_t - band * per_band;
            tb = first + local % width;
            wb = local / width;
            tl.g = g;
            tl.b_grp = 0;
            tl.a_grp = 0;
            tl.tok0 = tb * kTokRows;
            tl.a_row = tl.tok0;
            tl.tok_end = p.M;
            tl.n0 = wb * kWRows;
            tl.ntok = min(kTokRows, p.M - tl.tok0);
            tl.store = 3;
            tl.kb0 = prefix[g];
            tl.kb1 = prefix[g + 1];
            return true;
        }
        if (kLayout == kMasked) {
            int lo = 0, hi = p.G - 1;                // last g with prefix[g] <= t
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (prefix[mid] <= t) lo = mid; else hi = mid - 1;
            }
            const int g = lo, local = t - prefix[g];
            int mm = p.masked_m[g];
            mm = mm < 0 ? 0 : (mm > p.M ? p.M : mm);
            // within a group, the token blocks of one weight block are adjacent:
            // tiles that read the same B rows run at the same time (L2 reuse)
            const int ntb = (mm + kTokRows - 1) / kTokRows;
            wb = local / ntb;
            tb = local - wb * ntb;
            tl.g = g;
            tl.b_grp = g;
            tl.a_grp = g;
            tl.tok0 = tb * kTokRows;
            tl.a_row = tl.tok0;
            tl.tok_end = mm;
            tl.n0 = wb * kWRows;
            tl.ntok = min(kTokRows, mm - tl.tok0);
            tl.store = 3;
            return true;
        }
        if (kPairedGroups) {
            const int npairs = (p.M / kTileX + 1) / 2;
            const int first = npairs * nw;
            int pair, g, store;
            if (t < first) {
                const int per_band = kRasterM * nw;
                const int band = t / per_band;
                const int b0 = band * kRasterM;
                const int width = min(kRasterM, npairs - b0);
                const int local = t - band * per_band;
                pair = b0 + local % width;
                wb = local / width;
                const int g0 = block_group(p, 2 * pair), g1 = block_group(p, 2 * pair + 1);
                g = g0 >= 0 ? g0 : g1;
                if (g < 0) return false;
                store = (g0 == g ? 1 : 0) | (g1 == g ? 2 : 0);
            } else {
                const int q = (t - first) / nw;
                wb = t - first - q * nw;
                pair = prefix[q];
                g = block_group(p, 2 * pair + 1);
                store = 2;
            }
            tl.g = g;
            tl.b_grp = g;
            tl.tok0 = pair * kTokRows;
            tl.a_row = tl.tok0;
            tl.a_grp = 0;
            tl.tok_end = p.M;
            tl.n0 = wb * kWRows;
            tl.ntok = min(kTokRows, p.M - tl.tok0);
            tl.store = store;
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
        tl.b_grp = 0;
        tl.store = 3;
        if (kLayout == kContiguous) {
            const int g = __ldg(p.m_indices + tl.tok0);
            if (g < 0) return false;
            if (g >= p.G) return false;     // recorded by the producer
            tl.g = g;
            tl.b_grp = g;
        }
        return true;
    }
};

template <int kBN, bool kSwap, int kStages, int kCtaGroup, bool kSplitK = false>
struct SmemLayout {
    static constexpr int kYRows = kSwap ? kBN : kBN / kCtaGroup;   // rows of the Y operand per CTA
    static constexpr int kXBytes = kTileX * kBlockK;               // 16 KB
    static constexpr int kYBytes = kYRows * kBlockK;
    static constexpr int kStageBytes = kXBytes + kYBytes;
    static constexpr int kStagesBytes = kStages * kStageBytes;
    // Per-stage scale slot: this CTA's token-row scales sA[kb][rows ...] (one
    // float per token row), then the weight-block scale(s) sB[wblk][kb].
    static constexpr int kScaleRows = kSwap ? kBN : kTileX;
    static constexpr int kNumSB = kSwap ? 1 : weight_blocks_per_tile(kBN);
    static constexpr int kSlotFloats = kScaleRows + (kNumSB + 3) / 4 * 4;
    static constexpr int kSlotBytes = kSlotFloats * 4;
    // Swap mode keeps the scale slots in a ring of their own, deeper than the
    // operand stages, so an operand stage is free as soon as its MMAs ran.
    static constexpr int kSlots = kSwap ? 16 : kStages;
    static constexpr int kSlotOffset = kStagesBytes;
    static constexpr int kBarOffset = kSlotOffset + kSlots * kSlotBytes;
    // TMEM partial buffers: as many kBN-column buffers as fit in 512 columns (2..4).
    // Each K-block's partial lives from its MMA until the promotion warps have
    // read it; more buffers let the MMAs run further ahead of the promotion.
    static constexpr int kAccBufs = 512 / kBN >= 4 ? 4 : (512 / kBN >= 3 ? 3 : 2);
    // + 3: the split-K receive barrier and the SwiGLU epilogue's amax-exchange
    // barriers (one per tile parity)
    static constexpr int kNumBars = 2 * kStages + 2 * kAccBufs + 1 + (kSwap ? 3 * kSlots : 0) + 3;
    static constexpr int kMiscOffset = kBarOffset + kNumBars * 8;     // tmem addr, abort flag
    static constexpr int kPrefixOffset = (kMiscOffset + 16 + 15) / 16 * 16;
    static constexpr int kPrefixBytes = (kMaxGroups + 1) * 4;
    // split-K receive buffer: [source rank][owned row][column], rows padded by
    // 4 floats (bank spread); 136 rows cover any split of 128 rows into <= 8 owners
    static constexpr int kRecvStride = kBN + 4;
    static constexpr int kRecvRows = 136;
    static constexpr int kRecvOffset = (kPrefixOffset + kPrefixBytes + 127) / 128 * 128;
    static constexpr int kRecvBytes = kSplitK ? kRecvRows * kRecvStride * 4 : 0;
    // normal mode: per promotion warp a 32-row x 32-column BF16 staging box
    // (64-byte rows, 64B swizzle) for the TMA-store epilogue
    static constexpr int kOutBoxBytes = 32 * 64;
    static constexpr int kOutOffset = (kRecvOffset + kRecvBytes + 1023) / 1024 * 1024;
    // CTA pairs stage a whole finished tile instead (this CTA's 128 rows x kBN
    // columns of BF16, as kBN/32 boxes of 128 rows x 32 columns, 64B swizzle) and
    // one thread stores it, so the promotion warps never wait for the stores
    // (where it fits next to the pipeline stages; otherwise per-warp boxes)
    static constexpr int kStageBoxBytes = kTileX * 64;
    static constexpr bool kTileStaging =
        !kSwap && kCtaGroup == 2 && kOutOffset + (kBN / 32) * kStageBoxBytes + 1024 <= 227 * 1024;
    static constexpr int kOutBytes = kTileStaging ? (kBN / 32) * kStageBoxBytes : (kSwap ? 0 : 8 * kOutBoxBytes);
    static constexpr int kUsed = kOutOffset + kOutBytes;
    static constexpr int kAlloc = (kUsed + 1024 > kMinSmem) ? kUsed + 1024 : kMinSmem;
    static constexpr int kTmemCols = kAccBufs * kBN <= 32    ? 32
                                     : kAccBufs * kBN <= 64  ? 64
                                     : kAccBufs * kBN <= 128 ? 128
                                     : kAccBufs * kBN <= 256 ? 256 : 512;
    static_assert(kAccBufs * kBN <= 512, "TMEM holds 512 columns");
    static_assert(kStageBytes % 1024 == 0, "stage must keep 1024-byte alignment");
    static_assert(kSlotBytes % 16 == 0 && kSlotOffset % 16 == 0, "bulk copies need 16-byte aligned slots");
    static_assert(kBarOffset % 8 == 0, "mbarriers are 8-byte objects");
    static_assert(kPrefixOffset % 16 == 0, "prefix table alignment");
    static_assert(kRecvOffset % 16 == 0, "split-K pushes and reads are 16-byte vectors");
    static_assert(kOutOffset % 1024 == 0, "swizzled TMA-store boxes need aligned shared memory");
    static_assert(!kTileStaging || kBN % 32 == 0, "tile staging stores 32-column boxes");
    static_assert(kAlloc <= 227 * 1024, "shared memory budget");
};

template <int kBN, bool kSwap, int kStages, int kLayout, int kCtaGroup, bool kSwiGLU = false>
__global__ void __launch_bounds__(num_threads(kSwap), 1)
fp8_gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                const __grid_constant__ CUtensorMap tm_d, const Params p) {
    // SwiGLU epilogue: a 256-column tile is one 128-row gate block of the
    // weights followed by the matching 128-row up block; each promotion
    // warpgroup owns 64 gate columns and the 64 up columns they pair with
    static_assert(!kSwiGLU || (kBN == 256 && !kSwap && kCtaGroup == 1 && kLayout == kContiguous),
                  "SwiGLU epilogue: contiguous layout, 1-CTA 256-column tiles");
    // dense swap-mode kernels may run split-K (one tile per cluster)
    constexpr bool kSplitK = kSwap && kLayout == kDense && kBN <= 128;
    // the producer starts loading before the set-up barrier when nothing it
    // needs comes from other warps (not for CTA pairs or the masked layout)
    constexpr bool kEarly = kCtaGroup == 1 && kLayout != kMasked && kLayout != kKGrouped;
    using L = SmemLayout<kBN, kSwap, kStages, kCtaGroup, kSplitK>;
    using TM = TileMap<kBN, kSwap, kLayout, kCtaGroup>;
    static_assert(kBN == 64 || kBN == 128 || kBN == 160 || kBN == 224 || kBN == 256, "tile N");
    static_assert(kCtaGroup == 1 || (kCtaGroup == 2 && !kSwap && kLayout != kMasked),
                  "CTA pairs: dense or contiguous, normal mode");
    constexpr bool kPair = kCtaGroup == 2;
    constexpr int kHalf = kBN / 2;               // columns per promotion warpgroup
    constexpr int kChunk = kHalf > 64 ? 16 : 32; // TMEM columns per load (register budget)
    constexpr int kChunks = kHalf / kChunk;
    constexpr int kNumSB = L::kNumSB;
    constexpr int kPromoWarp0 = kSwap ? 2 : 4;    // first promotion warp
    static_assert(kHalf % kChunk == 0, "chunking");

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t s_base = ptx::smem_u32(smem);
    const uint32_t bar_base = s_base + L::kBarOffset;
    auto full_bar = [&](int s) { return bar_base + 8u * s; };
    auto empty_bar = [&](int s) { return bar_base + 8u * (kStages + s); };
    constexpr int kAccBufs = L::kAccBufs;
    auto tfull_bar = [&](int b) { return bar_base + 8u * (2 * kStages + b); };
    auto tempty_bar = [&](int b) { return bar_base + 8u * (2 * kStages + kAccBufs + b); };
    const uint32_t mma_done_bar = bar_base + 8u * (2 * kStages + 2 * kAccBufs);
    // swap mode scale ring: producer copies -> sfull, scale-prep warp -> sready,
    // promotion warps done -> sempty
    constexpr int kSlots = L::kSlots;
    auto sfull_bar = [&](int i) { return bar_base + 8u * (2 * kStages + 2 * kAccBufs + 1 + i); };
    auto sready_bar = [&](int i) { return bar_base + 8u * (2 * kStages + 2 * kAccBufs + 1 + kSlots + i); };
    auto sempty_bar = [&](int i) { return bar_base + 8u * (2 * kStages + 2 * kAccBufs + 1 + 2 * kSlots + i); };
    auto xchg_bar = [&](int i) { return bar_base + 8u * (L::kNumBars - 2 + i); };
    const uint32_t recv_bar = bar_base + 8u * (L::kNumBars - 3);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kMiscOffset);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::kMiscOffset + 4);
    const uint32_t slot_base = s_base + L::kSlotOffset;
    float *slots = reinterpret_cast<float *>(smem + L::kSlotOffset);
    int *prefix = reinterpret_cast<int *>(smem + L::kPrefixOffset);

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    const BoundedWait wait{abort_flag, p.status, p.timeout_cycles};
    // CTA pair: rank 0 issues the MMAs; its barriers count both CTAs' operand bytes
    const uint32_t pair_rank = kPair ? (ptx::cluster_rank() & 1u) : 0u;
    const bool mma_cta = pair_rank == 0;
    auto leader_addr = [&](uint32_t local) { return kPair ? ptx::map_cluster(local, 0) : local; };

    // ------------------------------------------------------------ set-up
    // warp 0 initialises the barriers, one lane per barrier (dozens of them in
    // swap mode: initialised one after another they delay the first load)
    if (warp == 0) {
        if (lane == 0) {
            ptx::prefetch_tmap(&tm_a);
            ptx::prefetch_tmap(&tm_b);
            *abort_flag = 0;
        }
        for (int s = lane; s < kStages; s += 32) {
            ptx::mbar_init(full_bar(s), 1);
            // MMA commit (+ 8 promotion warps that read the stage's scales, normal mode)
            ptx::mbar_init(empty_bar(s), kSwap ? 1 : 1 + 8);
        }
        if constexpr (kSwap) {
            for (int i = lane; i < kSlots; i += 32) {
                ptx::mbar_init(sfull_bar(i), 1);
                ptx::mbar_init(sready_bar(i), 32);
                ptx::mbar_init(sempty_bar(i), 8);
            }
        }
        if (lane < kAccBufs) {
            ptx::mbar_init(tfull_bar(lane), 1);
            ptx::mbar_init(tempty_bar(lane), 8 * kCtaGroup);   // every promotion warp of the pair
        }
        if (lane == 31) ptx::mbar_init(mma_done_bar, 1);
        if (lane == 30) ptx::mbar_init(xchg_bar(0), 256);     // both promotion warpgroups
        if (lane == 29) ptx::mbar_init(xchg_bar(1), 256);
        if (lane == 28) ptx::mbar_init(recv_bar, 1);     // split-K: the owner's expect-tx arrival
        ptx::fence_mbar_init();
        __syncwarp();
    }
    if (kLayout == kMasked && warp == kPromoWarp0) {
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
    if (kLayout == kKGrouped && warp == kPromoWarp0) {
        // exclusive prefix of K-blocks per group (group g owns [prefix[g], prefix[g+1])).
        // A size that is negative or not a multiple of 128, or a running total past
        // K, is recorded and clipped: such a group gets only the K-blocks that exist.
        int carry = 0;
        for (int base = 0; base < p.G; base += 32) {
            const int g = base + lane;
            int kbs = 0;
            if (g < p.G) {
                const int kg = __ldg(p.ks + g);
                if (kg < 0 || kg % kBlockK != 0) record_status(p.status, kStatusInvalid, kSiteBadKs);
                kbs = kg > 0 ? kg / kBlockK : 0;
            }
            int incl = kbs;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int v = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += v;
            }
            if (g < p.G) {
                const int lo = carry + incl - kbs, hi = carry + incl;
                if (hi > p.num_kb) record_status(p.status, kStatusInvalid, kSiteBadKs);
                prefix[g] = min(lo, p.num_kb);
            }
            carry += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) {
            if (carry != p.num_kb) record_status(p.status, kStatusInvalid, kSiteBadKs);   // sizes must add up to K
            prefix[p.G] = min(carry, p.num_kb);
        }
    }
    if (TM::kPairedGroups && warp == kPromoWarp0) {
        // pairs of 128-row blocks whose groups differ: they get a second pass
        const int nblk = p.M / kTileX, npairs = (nblk + 1) / 2;
        int count = 0;
        for (int base = 0; base < npairs; base += 32) {
            const int pr = base + lane;
            bool second = false;
            if (pr < npairs) {
                for (int b = 2 * pr; b <= 2 * pr + 1 && b < nblk; ++b)
                    if (__ldg(p.m_indices + static_cast<size_t>(b) * kTileX) >= p.G)
                        record_status(p.status, kStatusInvalid, kSiteBadGroup);
                const int g0 = TM::block_group(p, 2 * pr), g1 = TM::block_group(p, 2 * pr + 1);
                second = g0 >= 0 && g1 >= 0 && g0 != g1;
            }
            const unsigned ballot = __ballot_sync(0xffffffffu, second);
            const int slot = count + __popc(ballot & ((1u << lane) - 1u));
            if (second && slot < kMaxGroups) prefix[slot] = pr;
            count += __popc(ballot);
        }
        if (count > kMaxGroups) {
            if (lane == 0) record_status(p.status, kStatusInvalid, kSiteBadGroup);
            count = kMaxGroups;
        }
        if (lane == 0) prefix[kMaxGroups] = count;
    }
    if (warp == 1) {
        if constexpr (kPair) {
            ptx::tmem_alloc_pair(ptx::smem_u32(tmem_slot), L::kTmemCols);
            ptx::tmem_relinquish_pair();
        } else {
            ptx::tmem_alloc(ptx::smem_u32(tmem_slot), L::kTmemCols);
            ptx::tmem_relinquish();
        }
    }
    ptx::tc_fence_before();
    if constexpr (kEarly) {
        // warp 0 (the producer; it initialised the barriers) arrives and
        // goes on; the other warps wait until the barriers and TMEM are ready
        if (warp == 0) ptx::named_bar_arrive(1, num_threads(kSwap));
        else ptx::named_bar_sync(1, num_threads(kSwap));
    } else {
        __syncthreads();
    }
    if constexpr (kPair) ptx::cluster_sync_all();   // the peer's barriers exist before any remote use
    ptx::tc_fence_after();
    const uint32_t tmem_base = warp == 0 && kEarly ? 0u : *tmem_slot;

    // tile iteration: persistent (split == 1) or one tile per cluster (split > 1)
    const bool clustered = kSplitK && p.split > 1;   // split-K: dense swap-mode path
    const int num_tiles = clustered ? static_cast<int>(gridDim.y) : TM::count(p, prefix);
    const int t_first = clustered ? static_cast<int>(blockIdx.y) : static_cast<int>(blockIdx.x) / kCtaGroup;
    const int t_step = clustered ? num_tiles : static_cast<int>(gridDim.x) / kCtaGroup;
    int kb_begin = 0, kb_end = p.num_kb;
    // split-K: every CTA's barriers exist before any other CTA of the cluster
    // signals them (their initialisation was fenced with release at cluster
    // scope, so a relaxed arrival suffices); the wait comes just before the
    // exchange, long after, so nobody stalls here
    if (clustered) ptx::cluster_arrive_relaxed();
    if (clustered) {
        const int r = static_cast<int>(ptx::cluster_rank());
        kb_begin = (p.num_kb * r) / p.split;
        kb_end = (p.num_kb * (r + 1)) / p.split;
    }
    // this CTA's token rows inside a (pair) tile
    const int my_row0 = kPair ? static_cast<int>(pair_rank) * kTileX : 0;

    // The two role groups below never share code after this point: the
    // register rebalancing (setmaxnreg) gives each its own budget, which the
    // compiler can only honour on disjoint paths.  Each group runs its own copy
    // of the teardown barriers.
    if (warp < kPromoWarp0) {
    if constexpr (!kSwap) ptx::regs_dec<kRegsIssue>();
    if (warp == 0) {
        // ======================================================== producer
        // (one elected thread; the warp-wide sync orders it after the warp's
        // barrier initialisation when the producer starts before the set-up barrier)
        __syncwarp();
        if (ptx::elect_one()) {
            int stage = 0, sslot = 0;
            uint32_t phase = 0, sphase = 0;
            long long issued = 0, issued_s = 0;   // operand stages / swap-mode scale slots loaded
            bool ok = (p.debug_flags & kDebugProducerIdle) == 0;
            for (int t = t_first; ok && t < num_tiles; t += t_step) {
                Tile tl;
                if (!TM::decode(t, p, prefix, tl)) {
                    // a block whose group index is out of range (single-CTA tiles;
                    // on CTA pairs, where a tile without work leaves tl unset, the
                    // set-up pass over every block records it)
                    if (kLayout == kContiguous && !TM::kPairedGroups && __ldg(p.m_indices + tl.tok0) >= p.G)
                        record_status(p.status, kStatusInvalid, kSiteBadGroup);
                    continue;
                }
                const float *sfa_g = p.sfa + (kLayout == kMasked ? static_cast<size_t>(tl.g) * p.num_kb * p.ld_sfa : 0);
                const float *sfb_g = p.sfb + static_cast<size_t>(tl.b_grp) * p.num_nb * p.num_kb;
                const int wblk0 = tl.n0 / 128;
                // swap mode fetches only the tile's token rows, in boxes of kTokBox rows
                const int nload = kSwap ? (tl.ntok + kTokBox - 1) / kTokBox : 1;
                const uint32_t y_bytes = kSwap ? static_cast<uint32_t>(nload * kTokBox * kBlockK)
                                               : static_cast<uint32_t>(L::kYBytes);
                // this CTA's token-row scales present in memory (ld_sfa - row0 is a multiple of 4)
                const int sa_row0 = tl.tok0 + my_row0;
                const int sa_rows = max(0, min(kSwap ? nload * kTokBox : L::kScaleRows, p.ld_sfa - sa_row0));
                const uint32_t sa_bytes = static_cast<uint32_t>(sa_rows) * 4u;
                // operand bytes on this CTA's full barrier (a pair's MMA CTA counts both CTAs')
                const uint32_t op_bytes = kPair ? (mma_cta ? 2u * (L::kXBytes + y_bytes) : 0u)
                                                : L::kXBytes + y_bytes;
                const int kb_lo = max(kb_begin, tl.kb0), kb_hi = min(kb_end, tl.kb1);
                for (int kb = kb_lo; kb < kb_hi; ++kb) {
                    if (!wait(empty_bar(stage), phase ^ 1u, kSiteProducerEmpty)) { ok = false; break; }
                    const uint32_t sx = s_base + stage * L::kStageBytes;
                    const uint32_t sy = sx + L::kXBytes;
                    if constexpr (kSwap) {
                        // swap mode keeps the scales on their own barrier ring: the operand
                        // loads go first (the first bytes of a decode-shaped GEMM are on its
                        // critical path), then the scales once their slot is free
                        ptx::mbar_arrive_expect_tx(full_bar(stage), op_bytes);
                        ptx::tma_load_3d(sx, &tm_b, full_bar(stage), kb * kBlockK, tl.n0, tl.b_grp);
                        for (int i = 0; i < nload; ++i)
                            ptx::tma_load_3d(sy + i * kTokBox * kBlockK, &tm_a, full_bar(stage), kb * kBlockK,
                                             tl.a_row + i * kTokBox, tl.a_grp);
                        ++issued;
                        if (++stage == kStages) { stage = 0; phase ^= 1u; }
                        if (!wait(sempty_bar(sslot), sphase ^ 1u, kSiteProducerEmpty)) { ok = false; break; }
                    }
                    const uint32_t slot = slot_base + (kSwap ? sslot : stage) * L::kSlotBytes;
                    const uint32_t scale_bar = kSwap ? sfull_bar(sslot) : full_bar(stage);
#pragma unroll
                    for (int i = 0; i < kNumSB; ++i) {
                        const uint32_t dst = slot + (L::kScaleRows + i) * 4u;
                        if (wblk0 + i < p.num_nb)
                            ptx::cp_async_4(dst, sfb_g + static_cast<size_t>(wblk0 + i) * p.num_kb + kb);
                        else
                            ptx::st_shared_f32(dst, 0.f);
                    }
                    ptx::cp_async_arrive(scale_bar);
                    if (kSwap) ptx::mbar_arrive_expect_tx(scale_bar, sa_bytes);
                    else ptx::mbar_arrive_expect_tx(full_bar(stage), op_bytes + sa_bytes);
                    if (sa_bytes)
                        ptx::bulk_load(slot, sfa_g + static_cast<size_t>(kb) * p.ld_sfa + sa_row0, sa_bytes,
                                       scale_bar);
                    if (kSwap) {
                        ++issued_s;
                        if (++sslot == kSlots) { sslot = 0; sphase ^= 1u; }
                        continue;
                    } else if (kPair) {
                        // both CTAs' operand bytes complete on the MMA CTA's barrier
                        const uint32_t fb = leader_addr(full_bar(stage));
                        ptx::tma_load_3d_pair(sx, &tm_a, fb, kb * kBlockK, tl.a_row + my_row0, tl.a_grp);
                        ptx::tma_load_3d_pair(sy, &tm_b, fb, kb * kBlockK,
                                              tl.n0 + static_cast<int>(pair_rank) * L::kYRows, tl.b_grp);
                    } else {
                        ptx::tma_load_3d(sx, &tm_a, full_bar(stage), kb * kBlockK, tl.a_row, tl.a_grp);
                        ptx::tma_load_3d(sy, &tm_b, full_bar(stage), kb * kBlockK, tl.n0, tl.b_grp);
                    }
                    ++issued;
                    if (++stage == kStages) { stage = 0; phase ^= 1u; }
                }
            }
            // wind-down: never leave with TMA writes into this CTA's smem in flight
            // (the last kStages loads sit on distinct stages).  A pair's second CTA
            // cannot see its operand bytes land on its own barrier; for it the final
            // cluster barrier, reached only after the MMA CTA consumed every stage or
            // ran out of time waiting for it, covers them.
            auto drain = [&](long long depth, long long count, auto bar_of) {
                const long long first = count > depth ? count - depth : 0;
                for (long long i = first; i < count; ++i) {
                    const uint32_t bar = bar_of(static_cast<int>(i % depth));
                    const uint32_t par = static_cast<uint32_t>((i / depth) & 1);
                    const long long start = clock64();
                    while (!ptx::mbar_try_wait(bar, par)) {
                        if (clock64() - start > p.timeout_cycles) {
                            record_status(p.status, kStatusTimeout, kSiteTeardownLoads);
                            break;
                        }
                    }
                }
            };
            drain(kStages, issued, full_bar);
            if constexpr (kSwap) drain(kSlots, issued_s, sfull_bar);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ======================================================== MMA issuer
        if (mma_cta && ptx::elect_one()) {
            int stage = 0, buf = 0;
            uint32_t phase = 0, tphase = 0;
            bool issued_any = false;
            bool ok = true;
            for (int t = t_first; ok && t < num_tiles; t += t_step) {
                Tile tl;
                if (!TM::decode(t, p, prefix, tl)) continue;
                const uint32_t idesc = f8_idesc(kTileX * kCtaGroup,
                                                kSwap ? (tl.ntok + kTokBox - 1) / kTokBox * kTokBox : kBN);
                const int kb_lo = max(kb_begin, tl.kb0), kb_hi = min(kb_end, tl.kb1);
                for (int kb = kb_lo; kb < kb_hi; ++kb) {
                    if (!wait(tempty_bar(buf), tphase ^ 1u, kSiteMmaTmemEmpty)) { ok = false; break; }
                    if (!wait(full_bar(stage), phase, kSiteMmaFull)) { ok = false; break; }
                    ptx::tc_fence_after();
                    const uint32_t sx = s_base + stage * L::kStageBytes;
                    const uint64_t dx = sw128_desc(sx);
                    const uint64_t dy = sw128_desc(sx + L::kXBytes);
                    const uint32_t dtm = tmem_base + static_cast<uint32_t>(buf * kBN);
                    if constexpr (kPair) {
#pragma unroll
                        for (int k = 0; k < kBlockK / 32; ++k)
                            ptx::mma_f8f6f4_pair(dtm, dx + 2u * k, dy + 2u * k, idesc, k > 0 ? 1u : 0u);
                        ptx::mma_commit_pair(empty_bar(stage), 0x3);
                        ptx::mma_commit_pair(tfull_bar(buf), 0x3);
                    } else {
#pragma unroll
                        for (int k = 0; k < kBlockK / 32; ++k)
                            ptx::mma_f8f6f4(dtm, dx + 2u * k, dy + 2u * k, idesc, k > 0 ? 1u : 0u);
                        ptx::mma_commit(empty_bar(stage));
                        ptx::mma_commit(tfull_bar(buf));
                    }
                    issued_any = true;
                    if (++stage == kStages) { stage = 0; phase ^= 1u; }
                    if (++buf == kAccBufs) { buf = 0; tphase ^= 1u; }
                }
            }
            // every MMA completes before TMEM is released (a pair tells both CTAs);
            // the commit is issued even when nothing ran, so the wait below is uniform
            (void)issued_any;
            if constexpr (kPair) ptx::mma_commit_pair(mma_done_bar, 0x3);
            else ptx::mma_commit(mma_done_bar);
        }
        __syncwarp();
    }

    if (clustered) {   // completes the set-up arrival (matches the promotion warps)
        __syncwarp();
        ptx::cluster_wait_acquire();
    }
    // ------------------------------------------------------------ teardown (issue warps)
    if (warp == 1 && ptx::elect_one()) {
        // Every MMA that wrote this CTA's TMEM (or read its smem) has completed.
        // The MMA CTA committed mma_done after its last MMA (a pair multicasts
        // it); the wait is bounded.
        const long long start = clock64();
        while (!ptx::mbar_try_wait(mma_done_bar, 0)) {
            if (clock64() - start > p.timeout_cycles) {
                record_status(p.status, kStatusTimeout, kSiteTeardownMma);
                break;
            }
        }
    }
    __syncwarp();
    if (clustered) ptx::cluster_sync_all();   // split-K: the exchange's final barrier
    ptx::tc_fence_before();
    __syncthreads();
    if constexpr (kPair) ptx::cluster_sync_all();   // no CTA leaves while its peer may touch its smem
    if (warp == 1) {
        ptx::tc_fence_after();
        if constexpr (kPair) ptx::tmem_dealloc_pair(tmem_base, L::kTmemCols);
        else ptx::tmem_dealloc(tmem_base, L::kTmemCols);
    }
    } else if (kSwap && warp == kPrepWarp) {
    // ============================================================ scale preparation (swap mode)
    // For each K-block, turn the slot's per-token scales sA[tok] into
    // sA[tok] * sB, so the promotion does one FMA per element.
    {
        int sslot = 0;
        uint32_t sphase = 0;
        bool ok = true;
        for (int t = t_first; ok && t < num_tiles; t += t_step) {
            Tile tl;
            if (!TM::decode(t, p, prefix, tl)) continue;
            const int ncols = (tl.ntok + kTokBox - 1) / kTokBox * kTokBox;
            const int kb_lo = max(kb_begin, tl.kb0), kb_hi = min(kb_end, tl.kb1);
            for (int kb = kb_lo; kb < kb_hi; ++kb) {
                if (!wait(sfull_bar(sslot), sphase, kSitePromoFull)) { ok = false; break; }
                float *sl = slots + sslot * L::kSlotFloats;
                const float sb = sl[L::kScaleRows];
                for (int j = lane; j < ncols; j += 32) sl[j] *= sb;
                ptx::mbar_arrive(sready_bar(sslot));     // each lane: its own stores are released
                if (++sslot == kSlots) { sslot = 0; sphase ^= 1u; }
            }
        }
    }
    if (clustered) {   // completes the set-up arrival, then the exchange's final barrier
        __syncwarp();
        ptx::cluster_wait_acquire();
        ptx::cluster_sync_all();
    }
    ptx::tc_fence_before();
    __syncthreads();
    } else {
    if constexpr (!kSwap) ptx::regs_inc<kRegsPromo>();
    // ============================================================ promotion
    // (warps kPromoWarp0 and up)
    //
    // Column ownership.  Normal mode: warpgroup h owns the contiguous columns
    // [h*kHalf, (h+1)*kHalf) (224-wide tiles: alternate 32-column rounds, see
    // round_col); every 16-column group lies inside one 128-row weight block,
    // whose scale it uses.  Swap mode: columns
    // are tokens and the tile may hold fewer than kBN of them, so the chunks
    // are dealt alternately (chunk 2c+h to warpgroup h) to keep both
    // warpgroups busy; chunks past the tile's token count are skipped.
    float acc[kHalf];
    const bool promo = warp >= kPromoWarp0;
    const int quarter = warp & 3;                    // TMEM lane quarter this warp may access
    const int half = promo ? (warp - kPromoWarp0) >> 2 : 0;    // warpgroup
    const int lrow = quarter * 32 + lane;            // tile row = TMEM lane
    auto col_of = [&](int c) {                       // first tile column of local chunk c
        return kSwap ? (2 * c + half) * kChunk : half * kHalf + c * kChunk;
    };
    // Normal mode, tiles wider than 192: the tile column of this warpgroup's
    // 32-column round r (the last round may hold 16).  Tiles start on a multiple
    // of 32 (224-wide) or of 256, so every 128-row weight-block boundary inside a
    // tile lies on a multiple of 32 relative to it.  256-wide tiles give each
    // warpgroup one contiguous half, whose rounds start on multiples of 32; the
    // SwiGLU epilogue's warpgroup takes two gate rounds, then the two matching up
    // rounds.  224-wide tiles interleave the six full rounds between the
    // warpgroups (round r of warpgroup h is tile columns 32 (2r + h) ..) and split
    // the last 32 columns 16/16 (no boundary at 208).  Either way no round
    // straddles a weight block.
    constexpr bool kInterleave = !kSwap && kHalf > 96 && kHalf % 32 != 0;
    auto round_col = [&](int r) -> int {
        if constexpr (kSwiGLU) return r < 2 ? 64 * half + 32 * r : 128 + 64 * half + 32 * (r - 2);
        if constexpr (kInterleave) return r < kHalf / 32 ? 32 * (2 * r + half) : 2 * (kHalf / 32) * 32 + 16 * half;
        return half * kHalf + r * 32;
    };
    // tile column of this thread's accumulator j (normal mode)
    auto out_col = [&](int j) -> int {
        if constexpr (kInterleave) return round_col(j / 32) + j % 32;
        return half * kHalf + j;
    };
    static_assert(!kInterleave || kBN == 224, "interleaved rounds are laid out for 224-wide tiles");
    // the partial buffers are released on the MMA CTA's barrier (remote for a pair's second CTA)
    const bool remote_release = kPair && !mma_cta;
    const uint32_t tempty_target0 = remote_release ? leader_addr(tempty_bar(0)) : tempty_bar(0);
    auto release_tmem = [&](uint32_t target) {
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) {
            if (remote_release) ptx::mbar_arrive_remote(target);
            else ptx::mbar_arrive(target);
        }
    };
    Tile last_tile{0, 0, 0, 0, 0, 0, 0, 3};
    bool have_tile = false;
    int epi_parity = 0;   // SwiGLU epilogue: exchange-buffer parity
    int last_nvalid = 0;
    if (promo) {
        int stage = 0, buf = 0, sslot = 0;
        uint32_t phase = 0, tphase = 0, sphase = 0;
        bool ok = true;
        // contiguous layout: the next tile is decoded before this tile's epilogue,
        // so its group-index loads from global memory overlap the stores
        constexpr bool kDecodeAhead = kLayout == kContiguous;
        Tile tl_ahead;
        bool ahead_valid = false;
        int t_ahead = -1;
        for (int t = t_first; ok && t < num_tiles; t += t_step) {
            Tile tl;
            if (kDecodeAhead && t == t_ahead) {
                if (!ahead_valid) continue;
                tl = tl_ahead;
            } else if (!TM::decode(t, p, prefix, tl)) {
                continue;
            }
#pragma unroll
            for (int i = 0; i < kHalf; ++i) acc[i] = 0.f;
            const int my_tok = tl.tok0 + my_row0 + lrow;   // normal mode: this thread's token row
            const bool tok_ok = my_tok < tl.tok_end && ((tl.store >> pair_rank) & 1);
            // chunks of this warpgroup that hold columns of the tile
            const int ncols = kSwap ? (tl.ntok + kTokBox - 1) / kTokBox * kTokBox : kBN;
            const int nvalid = kSwap ? (ncols / kChunk - half + 1) / 2 : kChunks;
            const int wblk0 = tl.n0 / 128;
            const int kb_lo = max(kb_begin, tl.kb0), kb_hi = min(kb_end, tl.kb1);
            for (int kb = kb_lo; kb < kb_hi; ++kb) {
                // the K-block's scales: normal mode, visible once the stage's full
                // barrier completed; swap mode, once the scale-prep warp is done
                if (!wait(kSwap ? sready_bar(sslot) : full_bar(stage), kSwap ? sphase : phase,
                          kSitePromoFull)) { ok = false; break; }
                const float *slot = slots + (kSwap ? sslot : stage) * L::kSlotFloats;
                float sa_row = 0.f;
                float sbv[kNumSB];
                if (!kSwap) {
                    sa_row = slot[lrow];
#pragma unroll
                    for (int i = 0; i < kNumSB; ++i) sbv[i] = slot[L::kScaleRows + i];
                    __syncwarp();
                    if (lane == 0) ptx::mbar_arrive(empty_bar(stage));
                }
                if (!wait(tfull_bar(buf), tphase, kSitePromoFull)) { ok = false; break; }
                ptx::tc_fence_after();
                const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                                       static_cast<uint32_t>(buf * kBN);
                const uint32_t tempty_target = tempty_target0 + 8u * buf;
                if constexpr (!kSwap && kHalf <= 96) {
                    // Normal mode, narrow tiles: all kHalf columns of the warpgroup are
                    // loaded before one wait and the partial buffer is released at once,
                    // before the FMAs, so the MMA can reuse it as early as possible.
                    float v[kHalf];
                    const uint32_t ta = taddr + static_cast<uint32_t>(half * kHalf);
#pragma unroll
                    for (int o = 0; o + 32 <= kHalf; o += 32) ptx::tmem_ld32p(ta + o, v + o);
                    if constexpr (kHalf % 32 >= 16) ptx::tmem_ld16p(ta + kHalf / 32 * 32, v + kHalf / 32 * 32);
                    if constexpr (kHalf % 16 == 8) ptx::tmem_ld8p(ta + kHalf - 8, v + kHalf - 8);
                    ptx::tmem_wait_ld();
                    release_tmem(tempty_target);
                    float sblk[kNumSB];
#pragma unroll
                    for (int i = 0; i < kNumSB; ++i) sblk[i] = sa_row * sbv[i];
                    // one scale per 16 columns: tiles start on multiples of 32 and the
                    // warpgroup halves on multiples of 16, so no 16-column group
                    // straddles a 128-row weight block
#pragma unroll
                    for (int q = 0; q < kHalf / 16; ++q) {
                        const int col = half * kHalf + q * 16;
                        const int blk = (tl.n0 + col) / 128 - wblk0;
                        float sc = sblk[0];
#pragma unroll
                        for (int i = 1; i < kNumSB; ++i) sc = blk == i ? sblk[i] : sc;
#pragma unroll
                        for (int i = 0; i < 16; i += 2)
                            ptx::ffma2(acc[q * 16 + i], acc[q * 16 + i + 1], sc, v[q * 16 + i], v[q * 16 + i + 1]);
                    }
                    static_assert(kHalf % 16 == 0, "16-column scale groups");
                    if (++stage == kStages) { stage = 0; phase ^= 1u; }
                    if (++buf == kAccBufs) { buf = 0; tphase ^= 1u; }
                    continue;
                } else if constexpr (!kSwap) {
                    // Normal mode: this warpgroup's kHalf columns in rounds of up to 32
                    // (round_col() gives their place in the tile); each round loads its
                    // columns before one wait.  No round straddles a 128-row weight
                    // block, so each round takes one scale, chosen once per round.
                    constexpr int kRounds = (kHalf + 31) / 32;
                    float sblk[kNumSB];
#pragma unroll
                    for (int i = 0; i < kNumSB; ++i) sblk[i] = sa_row * sbv[i];
#pragma unroll
                    for (int r = 0; r < kRounds; ++r) {
                        constexpr int kFull = 32;
                        const int ncol = (r + 1) * 32 <= kHalf ? kFull : kHalf - r * 32;   // 32 or 16
                        float v[32];
                        const int rcol = round_col(r);
                        const uint32_t ta = taddr + static_cast<uint32_t>(rcol);
                        if (ncol == 32) ptx::tmem_ld32p(ta, v);
                        else ptx::tmem_ld16p(ta, v);
                        ptx::tmem_wait_ld();
                        if (r == kRounds - 1) release_tmem(tempty_target);
                        const int blk = (tl.n0 + rcol) / 128 - wblk0;
                        float sc = sblk[0];
#pragma unroll
                        for (int i = 1; i < kNumSB; ++i) sc = blk == i ? sblk[i] : sc;
                        float *a = acc + r * 32;
#pragma unroll
                        for (int i = 0; i < 32; i += 2)
                            if (i < ncol) ptx::ffma2(a[i], a[i + 1], sc, v[i], v[i + 1]);
                    }
                    if (++stage == kStages) { stage = 0; phase ^= 1u; }
                    if (++buf == kAccBufs) { buf = 0; tphase ^= 1u; }
                    continue;
                }
                // Swap mode.  Batched: every chunk of the thread is loaded before one
                // wait, so the TMEM read latency is paid once per K-block.
                constexpr bool kBatch = kHalf <= 64 && kChunk == 32;
                float vb[kBatch ? kHalf : 1];
                if constexpr (kBatch) {
#pragma unroll
                    for (int c = 0; c < kChunks; ++c)
                        if (c < nvalid) ptx::tmem_ld32p(taddr + col_of(c), vb + c * kChunk);
                    ptx::tmem_wait_ld();
                    if (nvalid > 0) release_tmem(tempty_target);
                }
                if (nvalid == 0) release_tmem(tempty_target);
#pragma unroll
                for (int c = 0; c < kChunks; ++c) {
                    if (c < nvalid) {
                        float vs[kBatch ? 1 : kChunk];
                        float *v = kBatch ? vb + c * kChunk : vs;
                        if constexpr (!kBatch) {
                            if constexpr (kChunk == 32) ptx::tmem_ld32p(taddr + col_of(c), v);
                            else ptx::tmem_ld16(taddr + col_of(c), vs);
                            ptx::tmem_wait_ld();
                            if (c == nvalid - 1) release_tmem(tempty_target);
                        }
                        float *a = acc + c * kChunk;
                        // column (token) scales sA * sB, broadcast from the slot
                        const float4 *sc = reinterpret_cast<const float4 *>(slot + col_of(c));
#pragma unroll
                        for (int i = 0; i < kChunk / 4; ++i) {
                            const float4 q4 = sc[i];
                            a[4 * i + 0] = fmaf(q4.x, v[4 * i + 0], a[4 * i + 0]);
                            a[4 * i + 1] = fmaf(q4.y, v[4 * i + 1], a[4 * i + 1]);
                            a[4 * i + 2] = fmaf(q4.z, v[4 * i + 2], a[4 * i + 2]);
                            a[4 * i + 3] = fmaf(q4.w, v[4 * i + 3], a[4 * i + 3]);
                        }
                    }
                }
                if (kSwap) {
                    __syncwarp();
                    if (lane == 0) ptx::mbar_arrive(sempty_bar(sslot));
                    if (++sslot == kSlots) { sslot = 0; sphase ^= 1u; }
                }
                if (++stage == kStages) { stage = 0; phase ^= 1u; }
                if (++buf == kAccBufs) { buf = 0; tphase ^= 1u; }
            }
            if (!ok) break;
            last_tile = tl;
            last_nvalid = nvalid;
            have_tile = true;
            if (clustered) break;   // one tile; reduced below
            if (kDecodeAhead && t + t_step < num_tiles) {
                t_ahead = t + t_step;
                ahead_valid = TM::decode(t_ahead, p, prefix, tl_ahead);
            }
            // ------------------------------------------------ epilogue (direct)
            const size_t row_base = (kLayout == kMasked || kLayout == kKGrouped) ? static_cast<size_t>(tl.g) * p.M : 0;
            // the TMA store may write every row of this CTA's 128-row block:
            // dense (rows past M are outside the D map), contiguous (padding rows
            // are don't-care), masked and K-grouped only when the block is full
            const bool tma_epilogue = !kSwap && ((tl.store >> pair_rank) & 1) != 0 &&
                                      (kLayout == kDense || kLayout == kContiguous ||
                                       tl.tok0 + my_row0 + kTileX <= tl.tok_end);
            if constexpr (kSwiGLU) {
                // act = silu(gate) * up for this thread's 64 columns of the tile's
                // 128-column activation block; the block's amax is combined with
                // the other warpgroup's through shared memory (one float per row,
                // double-buffered by tile parity), then the 64 values are quantised
                // like the per-token 1x128 quantiser: s = amax / 448, codes =
                // E4M3_RNE(act / s) with the IEEE quotient.
                float pmax = 0.f;
#pragma unroll
                for (int c = 0; c < 64; ++c) {
                    const float g = acc[c];
                    const float a = g / (1.0f + expf(-g)) * acc[64 + c];
                    acc[c] = a;
                    pmax = fmaxf(pmax, fabsf(a));
                }
                const int par = epi_parity & 1;
                float *xbuf = reinterpret_cast<float *>(prefix) + par * 256;
                xbuf[half * 128 + lrow] = pmax;
                ptx::mbar_arrive(xchg_bar(par));          // release: the store above is visible
                if (!wait(xchg_bar(par), static_cast<uint32_t>((epi_parity >> 1) & 1), kSitePromoFull)) break;
                const float amax = fmaxf(pmax, xbuf[(half ^ 1) * 128 + lrow]);
                ++epi_parity;
                const float sc = amax == 0.0f ? 1.0f : __fdiv_rn(amax, 448.0f);
                if (tok_ok) {
                    const int ablk = tl.n0 / 256;                 // 128-column activation block
                    const int ncols = p.N / 2;
                    uint8_t *qrow = p.q_out + (row_base + my_tok) * static_cast<size_t>(ncols) + ablk * 128 + 64 * half;
#pragma unroll
                    for (int c = 0; c < 64; c += 16) {
                        uint32_t w[4];
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            uint16_t lo, hi;
                            const float t0 = __fdiv_rn(acc[c + 4 * j + 0], sc), t1 = __fdiv_rn(acc[c + 4 * j + 1], sc);
                            const float t2 = __fdiv_rn(acc[c + 4 * j + 2], sc), t3 = __fdiv_rn(acc[c + 4 * j + 3], sc);
                            asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(lo) : "f"(t1), "f"(t0));
                            asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(hi) : "f"(t3), "f"(t2));
                            w[j] = static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
                        }
                        *reinterpret_cast<uint4 *>(qrow + c) = make_uint4(w[0], w[1], w[2], w[3]);
                    }
                    if (half == 0) p.s_out[static_cast<size_t>(ablk) * p.ld_s_out + row_base + my_tok] = sc;
                }
            } else if (L::kTileStaging && tma_epilogue) {
                // CTA pairs: the whole tile is staged as BF16 (box c = tile columns
                // [32c, 32c + 32), 128 rows of 64 bytes, 64B swizzle) and one thread
                // issues the boxes' TMA stores; the warps go on to the next tile at
                // once.  The staging of the previous tile must have been read first.
                const bool issuer = warp == kPromoWarp0 && lane == 0;
                if (issuer) ptx::bulk_wait_read0();
                ptx::named_bar_sync(3, 256);
                uint8_t *stg = smem + L::kOutOffset;
                const int sw = (lrow >> 1) & 3;                    // 64B swizzle of this row
#pragma unroll
                for (int j = 0; j < kHalf; j += 8) {
                    const int col = out_col(j);                    // tile column (a multiple of 8)
                    __nv_bfloat162 h0 = __floats2bfloat162_rn(acc[j + 0], acc[j + 1]);
                    __nv_bfloat162 h1 = __floats2bfloat162_rn(acc[j + 2], acc[j + 3]);
                    __nv_bfloat162 h2 = __floats2bfloat162_rn(acc[j + 4], acc[j + 5]);
                    __nv_bfloat162 h3 = __floats2bfloat162_rn(acc[j + 6], acc[j + 7]);
                    const int q = (col & 31) >> 3;                 // 16-byte chunk within the box row
                    *reinterpret_cast<uint4 *>(stg + (col >> 5) * L::kStageBoxBytes + lrow * 64 + ((q ^ sw) << 4)) =
                        make_uint4(*reinterpret_cast<uint32_t *>(&h0), *reinterpret_cast<uint32_t *>(&h1),
                                   *reinterpret_cast<uint32_t *>(&h2), *reinterpret_cast<uint32_t *>(&h3));
                }
                ptx::fence_proxy_async_smem();
                ptx::named_bar_sync(3, 256);
                if (issuer) {
                    const int drow0 = static_cast<int>(row_base) + tl.tok0 + my_row0;
#pragma unroll 1
                    for (int c = 0; c < kBN / 32; ++c) {
                        const int col0 = tl.n0 + 32 * c;
                        if (col0 < p.N)
                            ptx::tma_store_2d(&tm_d, ptx::smem_u32(stg + c * L::kStageBoxBytes), col0, drow0);
                    }
                    ptx::bulk_commit();
                }
            } else if (!kSwap && tma_epilogue) {
                // TMA-store epilogue: each warp converts its 32 rows x 32 columns
                // to BF16 in a 64B-swizzled staging box and one lane stores the box
                // with cp.async.bulk.tensor (rows past M and columns past N fall
                // outside the D map and are not written)
                uint8_t *box = smem + L::kOutOffset + (warp - kPromoWarp0) * L::kOutBoxBytes;
                const uint32_t box_s = ptx::smem_u32(box);
                const int wrow = tl.tok0 + my_row0 + quarter * 32;     // this warp's first tile row
                const bool rows_in = kLayout == kMasked || kLayout == kKGrouped || wrow < p.M;
                const int drow0 = static_cast<int>(row_base) + wrow;    // its row in the D map
                const int sw = (lane >> 1) & 3;                         // 64B swizzle of this lane's row
                constexpr int kFull = kHalf / 32;
#pragma unroll
                for (int c = 0; c < kFull; ++c) {
                    uint32_t w[16];
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        __nv_bfloat162 h2 = __floats2bfloat162_rn(acc[c * 32 + 2 * j], acc[c * 32 + 2 * j + 1]);
                        w[j] = *reinterpret_cast<uint32_t *>(&h2);
                    }
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        *reinterpret_cast<uint4 *>(box + lane * 64 + ((q ^ sw) * 16)) =
                            make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
                    ptx::fence_proxy_async_smem();
                    __syncwarp();
                    const int col0 = tl.n0 + out_col(c * 32);
                    if (lane == 0 && rows_in && col0 < p.N) {
                        ptx::tma_store_2d(&tm_d, box_s, col0, drow0);
                        ptx::bulk_commit();
                        ptx::bulk_wait_read0();          // the box may be rewritten
                    }
                    __syncwarp();
                }
                if constexpr (kHalf % 32 != 0) {
                    // the 16-column remainder of a 224-wide pair tile: direct stores
                    if (tok_ok) {
                        __nv_bfloat16 *drow = p.d + (row_base + my_tok) * static_cast<size_t>(p.N);
#pragma unroll
                        for (int j = kFull * 32; j < kHalf; j += 8) {
                            const int col = tl.n0 + out_col(j);
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
                }
            } else if (!kSwap) {
                if (tok_ok) {
                    __nv_bfloat16 *drow = p.d + (row_base + my_tok) * static_cast<size_t>(p.N);
#pragma unroll
                    for (int j = 0; j < kHalf; j += 8) {
                        const int col = tl.n0 + out_col(j);
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
        // every TMA store of this warp has completed before the CTA can exit
        if (!kSwap && lane == 0) ptx::bulk_wait0();
    }

    // ============================================================ split-K reduction
    if (clustered) {
        // Rows are owned in blocks of rows_per by the cluster's ranks.  (1) each
        // CTA stages its FP32 partial tile row-major ([weight row][token], rows
        // padded to kRecvStride floats) in the idle operand stages; (2) one thread
        // ships each owner's rows with one bulk copy into the owner's receive
        // buffer, slot [source rank][owned row][token], completing on the owner's
        // receive barrier; (3) the owner waits for the other ranks' bytes
        // (bounded) and sums in rank order.  No per-thread remote stores, and no
        // cluster-wide barrier before the reduction.
        const int split = p.split;
        const int rows_per = (kTileX + split - 1) / split;     // the last owner may get fewer
        const uint32_t my_rank = ptx::cluster_rank();
        const uint32_t recv_base = s_base + L::kRecvOffset;
        const uint32_t row_bytes = L::kRecvStride * 4;
        float *stg = reinterpret_cast<float *>(smem);          // operand stages: all loads consumed
        const bool sending = have_tile && !*abort_flag;
        if (sending) {
            float *row = stg + lrow * L::kRecvStride;
#pragma unroll
            for (int c = 0; c < kChunks; ++c) {
                if (c < last_nvalid) {
#pragma unroll
                    for (int i = 0; i < kChunk; i += 4)
                        *reinterpret_cast<float4 *>(row + col_of(c) + i) =
                            make_float4(acc[c * kChunk + i], acc[c * kChunk + i + 1], acc[c * kChunk + i + 2],
                                        acc[c * kChunk + i + 3]);
                }
            }
        }
        ptx::fence_proxy_async_smem();            // the bulk copies read the staging
        ptx::named_bar_sync(2, 256);              // every promotion thread has staged
        __syncwarp();
        ptx::cluster_wait_acquire();              // every CTA's receive barrier exists
        const int my_rows = max(0, min(rows_per, kTileX - static_cast<int>(my_rank) * rows_per));
        if (warp == kPromoWarp0 && lane == 0) {
            if (have_tile && my_rows > 0)
                ptx::mbar_arrive_expect_tx(recv_bar, static_cast<uint32_t>((split - 1) * my_rows) * row_bytes);
            if (sending) {
                for (int o = 0; o < split; ++o) {
                    const int rows_o = min(rows_per, kTileX - o * rows_per);
                    if (o == static_cast<int>(my_rank) || rows_o <= 0) continue;
                    const uint32_t src = s_base + static_cast<uint32_t>(o * rows_per) * row_bytes;
                    const uint32_t dst = ptx::map_cluster(
                        recv_base + static_cast<uint32_t>(my_rank * rows_per) * row_bytes, static_cast<uint32_t>(o));
                    ptx::bulk_copy_to_cluster(dst, src, static_cast<uint32_t>(rows_o) * row_bytes,
                                              ptx::map_cluster(recv_bar, static_cast<uint32_t>(o)));
                }
            }
        }
        bool got = true;
        if (have_tile && my_rows > 0) got = wait(recv_bar, 0u, kSiteSplitKRecv);
        // (3) each CTA sums its rows over the source ranks in rank order and stores.
        // Thread -> (row rr, 4 columns j4): consecutive threads take consecutive rows,
        // so a quarter-warp's 16-byte reads hit distinct banks (padded row stride)
        // and a warp's BF16 stores of one column are contiguous in D.
        if (have_tile && got) {
            const float4 *recv = reinterpret_cast<const float4 *>(smem + L::kRecvOffset);
            const float4 *own = reinterpret_cast<const float4 *>(stg);
            const Tile &tl = last_tile;
            const size_t row_base = (kLayout == kMasked || kLayout == kKGrouped) ? static_cast<size_t>(tl.g) * p.M : 0;
            const int tid = (warp - kPromoWarp0) * 32 + lane;        // 0..255
            const int groups = (tl.ntok + 3) / 4;
            const int elems = my_rows * groups;
            const int row0 = static_cast<int>(my_rank) * rows_per;
            const int n = tl.n0 + row0;
            for (int e = tid; e < elems; e += 256) {
                const int rr = e % my_rows;
                const int j4 = e / my_rows;
                float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
                for (int src = 0; src < split; ++src) {
                    const float4 v = src == static_cast<int>(my_rank)
                                         ? own[((row0 + rr) * L::kRecvStride) / 4 + j4]
                                         : recv[((src * rows_per + rr) * L::kRecvStride) / 4 + j4];
                    sum.x += v.x; sum.y += v.y; sum.z += v.z; sum.w += v.w;
                }
                const float vals[4] = {sum.x, sum.y, sum.z, sum.w};
                if (n + rr < p.N) {
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const int m = tl.tok0 + 4 * j4 + q;
                        if (m < tl.tok_end)
                            p.d[(row_base + m) * static_cast<size_t>(p.N) + n + rr] = __float2bfloat16_rn(vals[q]);
                    }
                }
            }
        }
        // no CTA leaves while a peer's bulk copy may still read its staging or
        // write its receive buffer
        __syncwarp();
        ptx::cluster_sync_all();
    }

    // ------------------------------------------------------------ teardown (promotion warps)
    ptx::tc_fence_before();
    __syncthreads();
    if constexpr (kPair) ptx::cluster_sync_all();
    }
}

}  // namespace dg
