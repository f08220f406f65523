// bf16_kernel.cuh -- the sm_100a kernel of the BF16 NT GEMM (DeepGEMM pages:
// page 3 "核心功能" -- FP8, FP4 and BF16 GEMMs in the same dense and
// m-grouped layouts).
//
//   D[m,n] = sum_k A[m,k] * B[n,k]     (A [M,K], B [N,K] BF16, K-major; D BF16)
//
// No block scales, so nothing is promoted on CUDA cores: the tensor cores
// accumulate the whole K range in one FP32 TMEM accumulator per tile.  The
// kernel is persistent and warp-specialised over the same tile scheduler as
// the FP8 kernel (TileMap: dense raster, contiguous group lookup, masked tile
// list built on the device):
//
//   warp 0      producer: one thread issues TMA loads of the A tile (128 rows)
//               and the B tile (kBN rows) per 64-element K-block (128 bytes,
//               128B swizzle -- the same shared-memory tiling as the FP8 path).
//   warp 1      TMEM allocator + MMA issuer: 4 x tcgen05.mma.kind::f16 (K=16)
//               per K-block into the tile's accumulator; two accumulators in
//               rotation so the next tile's MMAs overlap this tile's epilogue.
//   warps 4..7  epilogue: tcgen05.ld of the accumulator in 32-column chunks,
//               BF16 round-to-nearest-even, 16-byte stores of each row.
//
// CTA pairs (kCtaGroup == 2; dense and contiguous layouts with many tiles): a
// cluster of 2 CTAs computes one 256 x kBN tile with tcgen05.mma.cta_group::2.
// Each CTA stages its own 128 token rows and half of the tile's weight rows, so
// a K-block costs each SM 16 KB + kBN/2 x 128 B of shared memory and of L2 reads
// instead of 16 KB + kBN x 128 B: the weight operand, which bounds single-CTA
// tiles' shared-memory reads, is halved.  The even CTA issues the MMAs; both
// CTAs' TMA bytes complete on its barrier, the MMA completions are multicast to
// both CTAs, and each CTA's epilogue drains its own 128 accumulator rows and
// releases the accumulator on the even CTA's barrier.
//
// Every wait is bounded (BoundedWait): on timeout the kernel records
// DG_ERR_TIMEOUT in the device status word and winds down instead of hanging.
#pragma once

#include "gemm_kernel.cuh"

namespace dg {

constexpr int kBf16Threads = 256;
constexpr int kBf16BlockK = 64;          // BF16 elements per 128-byte K-block

// Instruction descriptor, kind::f16: D = F32, A = B = BF16, both K-major.
__host__ __device__ constexpr uint32_t bf16_idesc(int m, int n) {
    return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(n >> 3) << 17) |
           (static_cast<uint32_t>(m >> 4) << 24);
}

template <int kBN, int kStages, bool kSplitK = false, int kCtaGroup = 1>
struct Bf16Smem {
    static constexpr int kXBytes = kTileX * 128;        // 128 rows x 64 BF16
    static constexpr int kYBytes = kBN / kCtaGroup * 128;   // this CTA's weight rows
    static constexpr int kStageBytes = kXBytes + kYBytes;
    static constexpr int kAccBufs = 2;
    static constexpr int kBarOffset = kStages * kStageBytes;
    static constexpr int kNumBars = 2 * kStages + 2 * kAccBufs + 2;   // + split-K receive barrier
    static constexpr int kMiscOffset = kBarOffset + kNumBars * 8;   // tmem addr, abort flag
    static constexpr int kPrefixOffset = (kMiscOffset + 16 + 15) / 16 * 16;
    static constexpr int kPrefixBytes = (kMaxGroups + 1) * 4;
    // split-K: receive buffer [source rank][owned row][column], rows padded by 4
    // floats; 136 rows cover any split of 128 rows into <= 8 owners
    static constexpr int kRecvStride = kBN + 4;
    static constexpr int kRecvOffset = (kPrefixOffset + kPrefixBytes + 127) / 128 * 128;
    static constexpr int kRecvBytes = kSplitK ? 136 * kRecvStride * 4 : 0;
    static constexpr int kUsed = kRecvOffset + kRecvBytes;
    static constexpr int kAlloc = (kUsed + 1024 > kMinSmem) ? kUsed + 1024 : kMinSmem;
    static constexpr int kTmemCols = kAccBufs * kBN <= 256 ? 256 : 512;
    static_assert(kAccBufs * kBN <= 512, "TMEM holds 512 columns");
    static_assert(kStageBytes % 1024 == 0, "stage must keep 1024-byte alignment");
    static_assert(kAlloc <= 227 * 1024, "shared memory budget");
    static_assert(!kSplitK || kTileX * kRecvStride * 4 <= kStages * kStageBytes,
                  "split-K staging lives in the operand stages");
};

template <int kBN, int kStages, int kLayout, bool kSplitK = false, int kCtaGroup = 1>
__global__ void __launch_bounds__(kBf16Threads, 1)
bf16_gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                 const Params p) {
    using L = Bf16Smem<kBN, kStages, kSplitK, kCtaGroup>;
    static_assert(!kSplitK || kLayout == kDense, "split-K: dense layout");
    constexpr bool kPair = kCtaGroup == 2;
    static_assert(!kPair || ((kLayout == kDense || kLayout == kContiguous) && !kSplitK),
                  "CTA pairs: dense or contiguous, no split-K");
    using TM = TileMap<kBN, false, kLayout, kCtaGroup>;
    static_assert(kBN == 128 || kBN == 224 || kBN == 256, "tile N");
    static_assert(kLayout != kKGrouped, "BF16: dense, contiguous and masked layouts");
    constexpr int kAccBufs = L::kAccBufs;
    constexpr int kEpiWarp0 = 4;

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t s_base = ptx::smem_u32(smem);
    const uint32_t bar_base = s_base + L::kBarOffset;
    auto full_bar = [&](int s) { return bar_base + 8u * s; };
    auto empty_bar = [&](int s) { return bar_base + 8u * (kStages + s); };
    auto tfull_bar = [&](int b) { return bar_base + 8u * (2 * kStages + b); };
    auto tempty_bar = [&](int b) { return bar_base + 8u * (2 * kStages + kAccBufs + b); };
    const uint32_t mma_done_bar = bar_base + 8u * (2 * kStages + 2 * kAccBufs);
    const uint32_t recv_bar = bar_base + 8u * (2 * kStages + 2 * kAccBufs + 1);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kMiscOffset);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::kMiscOffset + 4);
    int *prefix = reinterpret_cast<int *>(smem + L::kPrefixOffset);

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    const BoundedWait wait{abort_flag, p.status, p.timeout_cycles};
    // CTA pair: rank 0 issues the MMAs; its barriers count both CTAs' operand bytes
    const uint32_t pair_rank = kPair ? (ptx::cluster_rank() & 1u) : 0u;
    const bool mma_cta = pair_rank == 0;
    auto leader_addr = [&](uint32_t local) { return kPair ? ptx::map_cluster(local, 0) : local; };

    if (threadIdx.x == 0) {
        ptx::prefetch_tmap(&tm_a);
        ptx::prefetch_tmap(&tm_b);
        for (int i = 0; i < kStages; ++i) {
            ptx::mbar_init(full_bar(i), 1);
            ptx::mbar_init(empty_bar(i), 1);
        }
        for (int b = 0; b < kAccBufs; ++b) {
            ptx::mbar_init(tfull_bar(b), 1);
            ptx::mbar_init(tempty_bar(b), 4 * kCtaGroup);   // one arrival per epilogue warp of the pair
        }
        ptx::mbar_init(mma_done_bar, 1);
        ptx::mbar_init(recv_bar, 1);               // split-K: the owner's expect-tx arrival
        *abort_flag = 0;
        ptx::fence_mbar_init();
    }
    if (kLayout == kMasked && warp == kEpiWarp0) {
        // exclusive prefix of tiles per group: ceil(masked_m[g] / 128) * weight blocks
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
    if (TM::kPairedGroups && warp == kEpiWarp0) {
        // contiguous layout on CTA pairs: the pairs of 128-row blocks whose groups
        // differ get a second pass (the tile scheduler lists them after the first
        // passes); the table of such pairs, as in the FP8 kernel
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
    __syncthreads();
    if constexpr (kPair) ptx::cluster_sync_all();   // the peer's barriers exist before any remote use
    ptx::tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    // this CTA's token rows inside a pair tile
    const int my_row0 = kPair ? static_cast<int>(pair_rank) * kTileX : 0;

    // split-K (dense, few tiles): a cluster of p.split CTAs shares one tile, each
    // CTA takes a contiguous range of K-blocks; the FP32 partials are summed in
    // rank order through distributed shared memory (see the epilogue)
    const bool clustered = kSplitK && p.split > 1;
    const int num_tiles = clustered ? static_cast<int>(gridDim.y) : TM::count(p, prefix);
    const int t_first = clustered ? static_cast<int>(blockIdx.y) : static_cast<int>(blockIdx.x) / kCtaGroup;
    const int t_step = clustered ? num_tiles : static_cast<int>(gridDim.x) / kCtaGroup;
    int kb_begin = 0, kb_end = p.num_kb;
    if (clustered) {
        // every CTA's receive barrier exists before another CTA signals it (its
        // initialisation was fenced at cluster scope); the wait comes much later
        ptx::cluster_arrive_relaxed();
        const int r = static_cast<int>(ptx::cluster_rank());
        kb_begin = (p.num_kb * r) / p.split;
        kb_end = (p.num_kb * (r + 1)) / p.split;
    }

    if (warp == 0) {
        // ============================================================ producer
        __syncwarp();
        if (ptx::elect_one()) {
            int stage = 0;
            uint32_t phase = 0;
            long long issued = 0;
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
                for (int kb = kb_begin; kb < kb_end; ++kb) {
                    if (!wait(empty_bar(stage), phase ^ 1u, kSiteProducerEmpty)) { ok = false; break; }
                    const uint32_t sx = s_base + stage * L::kStageBytes;
                    if constexpr (kPair) {
                        // both CTAs' bytes complete on the MMA CTA's barrier
                        if (mma_cta) ptx::mbar_arrive_expect_tx(full_bar(stage), 2u * L::kStageBytes);
                        const uint32_t fb = leader_addr(full_bar(stage));
                        ptx::tma_load_3d_pair(sx, &tm_a, fb, kb * kBf16BlockK, tl.a_row + my_row0, tl.a_grp);
                        ptx::tma_load_3d_pair(sx + L::kXBytes, &tm_b, fb, kb * kBf16BlockK,
                                              tl.n0 + static_cast<int>(pair_rank) * (kBN / 2), tl.b_grp);
                    } else {
                        ptx::mbar_arrive_expect_tx(full_bar(stage), L::kStageBytes);
                        ptx::tma_load_3d(sx, &tm_a, full_bar(stage), kb * kBf16BlockK, tl.a_row, tl.a_grp);
                        ptx::tma_load_3d(sx + L::kXBytes, &tm_b, full_bar(stage), kb * kBf16BlockK, tl.n0,
                                         tl.b_grp);
                    }
                    ++issued;
                    if (++stage == kStages) { stage = 0; phase ^= 1u; }
                }
            }
            // never leave with TMA writes into shared memory in flight.  A pair's
            // second CTA cannot see its bytes land on its own barrier; for it the
            // final cluster barrier, reached only after the MMA CTA consumed every
            // stage (or ran out of time waiting for it), covers them.
            const long long first = !mma_cta ? issued : (issued > kStages ? issued - kStages : 0);
            for (long long i = first; i < issued; ++i) {
                const uint32_t bar = full_bar(static_cast<int>(i % kStages));
                const uint32_t par = static_cast<uint32_t>((i / kStages) & 1);
                const long long start = clock64();
                while (!ptx::mbar_try_wait(bar, par)) {
                    if (clock64() - start > p.timeout_cycles) {
                        record_status(p.status, kStatusTimeout, kSiteTeardownLoads);
                        break;
                    }
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ============================================================ MMA issuer
        if (mma_cta && ptx::elect_one()) {
            int stage = 0, buf = 0;
            uint32_t phase = 0, tphase = 0;
            bool ok = true;
            const uint32_t idesc = bf16_idesc(kTileX * kCtaGroup, kBN);
            for (int t = t_first; ok && t < num_tiles; t += t_step) {
                Tile tl;
                if (!TM::decode(t, p, prefix, tl)) continue;
                if (!wait(tempty_bar(buf), tphase ^ 1u, kSiteMmaTmemEmpty)) { ok = false; break; }
                const uint32_t dtm = tmem_base + static_cast<uint32_t>(buf * kBN);
                for (int kb = kb_begin; kb < kb_end; ++kb) {
                    if (!wait(full_bar(stage), phase, kSiteMmaFull)) { ok = false; break; }
                    ptx::tc_fence_after();
                    const uint32_t sx = s_base + stage * L::kStageBytes;
                    const uint64_t dx = sw128_desc(sx);
                    const uint64_t dy = sw128_desc(sx + L::kXBytes);
                    if constexpr (kPair) {
#pragma unroll
                        for (int k = 0; k < kBf16BlockK / 16; ++k)
                            ptx::mma_f16_pair(dtm, dx + 2u * k, dy + 2u * k, idesc, (kb > kb_begin || k > 0) ? 1u : 0u);
                        ptx::mma_commit_pair(empty_bar(stage), 0x3);
                    } else {
#pragma unroll
                        for (int k = 0; k < kBf16BlockK / 16; ++k)
                            ptx::mma_f16(dtm, dx + 2u * k, dy + 2u * k, idesc, (kb > kb_begin || k > 0) ? 1u : 0u);
                        ptx::mma_commit(empty_bar(stage));
                    }
                    if (++stage == kStages) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                if constexpr (kPair) ptx::mma_commit_pair(tfull_bar(buf), 0x3);
                else ptx::mma_commit(tfull_bar(buf));
                if (++buf == kAccBufs) { buf = 0; tphase ^= 1u; }
            }
            // the commit is issued even when nothing ran, so every wait on it is uniform
            if constexpr (kPair) ptx::mma_commit_pair(mma_done_bar, 0x3);
            else ptx::mma_commit(mma_done_bar);
        }
        __syncwarp();
    } else if (warp >= kEpiWarp0) {
        // ============================================================ epilogue
        const int quarter = warp & 3;
        const int lrow = quarter * 32 + lane;
        int buf = 0;
        uint32_t tphase = 0;
        Tile split_tile{};
        bool have_split_tile = false;
        for (int t = t_first; t < num_tiles; t += t_step) {
            Tile tl;
            if (!TM::decode(t, p, prefix, tl)) continue;
            if (!wait(tfull_bar(buf), tphase, kSitePromoFull)) break;
            ptx::tc_fence_after();
            const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                                   static_cast<uint32_t>(buf * kBN);
            if (clustered) {
                // stage the FP32 partial tile row-major (rows padded to kRecvStride
                // floats) in the idle operand stages, then exchange (below)
                float *row = reinterpret_cast<float *>(smem) + lrow * L::kRecvStride;
#pragma unroll 1
                for (int c = 0; c < kBN / 32; ++c) {
                    float v[32];
                    ptx::tmem_ld32p(taddr + c * 32, v);
                    ptx::tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 32; j += 4)
                        *reinterpret_cast<float4 *>(row + c * 32 + j) = make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
                }
                split_tile = tl;
                have_split_tile = true;
                break;   // one tile per cluster
            }
            const int my_tok = tl.tok0 + my_row0 + lrow;
            const bool row_ok = my_tok < tl.tok_end && ((tl.store >> pair_rank) & 1);
            const size_t row_base = kLayout == kMasked ? static_cast<size_t>(tl.g) * p.M : 0;
            __nv_bfloat16 *drow = p.d + (row_base + my_tok) * static_cast<size_t>(p.N);
#pragma unroll 1
            for (int c = 0; c < kBN / 32; ++c) {
                float v[32];
                ptx::tmem_ld32p(taddr + c * 32, v);
                ptx::tmem_wait_ld();
                if (row_ok) {
#pragma unroll
                    for (int j = 0; j < 32; j += 8) {
                        const int col = tl.n0 + c * 32 + j;
                        if (col < p.N) {
                            uint4 pk;
                            __nv_bfloat162 h0 = __floats2bfloat162_rn(v[j + 0], v[j + 1]);
                            __nv_bfloat162 h1 = __floats2bfloat162_rn(v[j + 2], v[j + 3]);
                            __nv_bfloat162 h2 = __floats2bfloat162_rn(v[j + 4], v[j + 5]);
                            __nv_bfloat162 h3 = __floats2bfloat162_rn(v[j + 6], v[j + 7]);
                            pk.x = *reinterpret_cast<uint32_t *>(&h0);
                            pk.y = *reinterpret_cast<uint32_t *>(&h1);
                            pk.z = *reinterpret_cast<uint32_t *>(&h2);
                            pk.w = *reinterpret_cast<uint32_t *>(&h3);
                            *reinterpret_cast<uint4 *>(drow + col) = pk;
                        }
                    }
                }
            }
            // the accumulator is free for the MMA warp's next tile (released on the
            // MMA CTA's barrier: remote for a pair's second CTA)
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                if (kPair && !mma_cta) ptx::mbar_arrive_remote(leader_addr(tempty_bar(buf)));
                else ptx::mbar_arrive(tempty_bar(buf));
            }
            if (++buf == kAccBufs) { buf = 0; tphase ^= 1u; }
        }
        if (clustered) {
            // Token rows are owned in blocks of rows_per by the cluster's ranks: one
            // thread ships each owner's rows of this CTA's staged partial with one
            // bulk copy into the owner's receive buffer, slot [source rank][owned
            // row][column], completing on the owner's receive barrier; the owner
            // waits for the other ranks' bytes (bounded), sums in rank order and
            // stores BF16 rows.
            const int split = p.split;
            const Tile &tl = split_tile;
            const int ntok = have_split_tile ? tl.ntok : 0;
            const int rows_per = (ntok + split - 1) / split;
            const uint32_t my_rank = ptx::cluster_rank();
            const uint32_t row_bytes = L::kRecvStride * 4;
            const uint32_t recv_base = s_base + L::kRecvOffset;
            const int my_rows = max(0, min(rows_per, ntok - static_cast<int>(my_rank) * rows_per));
            const bool sending = have_split_tile && !*abort_flag;
            ptx::fence_proxy_async_smem();            // the bulk copies read the staging
            ptx::named_bar_sync(2, 128);              // the four epilogue warps have staged
            __syncwarp();
            ptx::cluster_wait_acquire();              // every CTA's receive barrier exists
            if (warp == kEpiWarp0 && lane == 0) {
                if (my_rows > 0)
                    ptx::mbar_arrive_expect_tx(recv_bar, static_cast<uint32_t>((split - 1) * my_rows) * row_bytes);
                if (sending) {
                    for (int o = 0; o < split; ++o) {
                        const int rows_o = min(rows_per, ntok - o * rows_per);
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
            if (my_rows > 0) got = wait(recv_bar, 0u, kSitePromoFull);
            if (have_split_tile && got && my_rows > 0) {
                const float *own = reinterpret_cast<const float *>(smem);
                const float *recv = reinterpret_cast<const float *>(smem + L::kRecvOffset);
                const int row0 = static_cast<int>(my_rank) * rows_per;
                constexpr int kGroups = kBN / 8;                       // 8 columns = one 16-byte store
                const int tid = (warp - kEpiWarp0) * 32 + lane;        // 0..127
                for (int e = tid; e < my_rows * kGroups; e += 128) {
                    const int rr = e / kGroups, c8 = e - rr * kGroups;
                    float acc8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                    for (int src = 0; src < split; ++src) {
                        const float *rowp = src == static_cast<int>(my_rank)
                                                ? own + (row0 + rr) * L::kRecvStride
                                                : recv + (src * rows_per + rr) * L::kRecvStride;
                        const float4 a = *reinterpret_cast<const float4 *>(rowp + 8 * c8);
                        const float4 b = *reinterpret_cast<const float4 *>(rowp + 8 * c8 + 4);
                        acc8[0] += a.x; acc8[1] += a.y; acc8[2] += a.z; acc8[3] += a.w;
                        acc8[4] += b.x; acc8[5] += b.y; acc8[6] += b.z; acc8[7] += b.w;
                    }
                    const int col = tl.n0 + 8 * c8;
                    const int tok = tl.tok0 + row0 + rr;
                    if (col < p.N && tok < tl.tok_end) {
                        uint4 pk;
                        __nv_bfloat162 h0 = __floats2bfloat162_rn(acc8[0], acc8[1]);
                        __nv_bfloat162 h1 = __floats2bfloat162_rn(acc8[2], acc8[3]);
                        __nv_bfloat162 h2 = __floats2bfloat162_rn(acc8[4], acc8[5]);
                        __nv_bfloat162 h3 = __floats2bfloat162_rn(acc8[6], acc8[7]);
                        pk.x = *reinterpret_cast<uint32_t *>(&h0);
                        pk.y = *reinterpret_cast<uint32_t *>(&h1);
                        pk.z = *reinterpret_cast<uint32_t *>(&h2);
                        pk.w = *reinterpret_cast<uint32_t *>(&h3);
                        *reinterpret_cast<uint4 *>(p.d + static_cast<size_t>(tok) * p.N + col) = pk;
                    }
                }
            }
        }
    }
    if (clustered) {
        // warps outside the epilogue complete the set-up arrival here; then no
        // CTA leaves while a peer's bulk copy may still read its staging or
        // write its receive buffer
        if (warp < kEpiWarp0) ptx::cluster_wait_acquire();
        __syncwarp();
        ptx::cluster_sync_all();
    }

    // ---------------------------------------------------------------- teardown
    if (warp == 1 && ptx::elect_one()) {
        const long long start = clock64();
        while (!ptx::mbar_try_wait(mma_done_bar, 0)) {
            if (clock64() - start > p.timeout_cycles) {
                record_status(p.status, kStatusTimeout, kSiteTeardownMma);
                break;
            }
        }
    }
    __syncwarp();
    ptx::tc_fence_before();
    __syncthreads();
    if constexpr (kPair) ptx::cluster_sync_all();   // no CTA leaves while its peer may touch its smem
    if (warp == 1) {
        ptx::tc_fence_after();
        if constexpr (kPair) ptx::tmem_dealloc_pair(tmem_base, L::kTmemCols);
        else ptx::tmem_dealloc(tmem_base, L::kTmemCols);
    }
}

}  // namespace dg
