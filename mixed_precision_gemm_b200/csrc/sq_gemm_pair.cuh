// Dual-path GEMM on CTA pairs (tcgen05 cta_group::2): the same computation as
// sq_gemm_common.cuh (OSC, arXiv:2604.12782, abstract: a 4-bit GEMM path plus a
// 16-bit branch GEMM on the compact outlier tensor, fused), with 256 x 256
// output tiles shared by the two CTAs of a cluster.
//
// In a pair MMA each CTA supplies half of A (its 128 token rows) and half of
// B (128 of the 256 output channels) from its own shared memory, and receives
// its 128 rows x 256 columns of D in its own tensor memory.  Per SM that is
// the 128 x 256 tile of the single-CTA kernel with a third fewer operand bytes
// to fetch and expand, which is what the INT4 -> int8 expansion is bound by.
//
// Roles (18 warps per CTA, one cluster of 2 CTAs per SM pair, tiles handed
// out round-robin to clusters):
//   warp 0 (each CTA)        TMA producer of the packed INT4 tiles (this CTA's
//                            X rows and W rows) into a staging ring.
//   warp 1 of the first CTA  issues every pair MMA; its commits arrive on the
//                            barriers of both CTAs (multicast commit).
//   warps 2..9 (each CTA)    epilogue of the CTA's 128 rows (two warps per TMEM
//                            lane quarter); they report to the first CTA's
//                            acc_empty barrier when TMEM is read.  Y goes out
//                            per lane (16-byte stores), or with C::YB > 0
//                            through 32 x 16 staging boxes and bulk tensor
//                            stores.
//   warps 10..17 (each CTA)  operand producers for the CTA's halves, in ring
//                            order: bf16 blocks by TMA (.cta_group::2 form, no
//                            multicast, completion bytes counted on the first
//                            CTA's barrier); INT4 blocks expanded from the
//                            staging ring into int8 operand tiles (see
//                            sq_gemm_common.cuh).  Every producer warp of both CTAs
//                            arrives on the first CTA's op_full.
// The packed tiles travel by TMA into a staging ring (asynchronous, C::STG
// K-blocks deep) and are expanded from shared memory, so no producer thread
// has long global loads outstanding when it publishes a tile.
// TMEM per CTA: acc_f in columns [0, 256), acc_i in [256, 512).
//
// MX low path (kLowMx): the packed E2M1 tiles travel by TMA straight into
// the operand ring, together with their E8M0 scales (tiles of 128 rows x 4
// blocks, see sq_mxquant.cuh).  The scales land on a barrier of their own CTA
// (sf_full); the four warps of the producer group that owns the ring slot,
// one per TMEM lane quarter, write them into the slot's scale columns
// (MX_SFA_COL / MX_SFB_COL + MX_SF_SLOT * slot, tcgen05.st) and only then
// arrive on op_full, so the MMA thread issues nothing but the K-block's four
// kind::mxf4 MMAs and the scale writes of later slots run beside them.  (A
// tcgen05.cp per scale tile from the MMA thread, six per K-block, shared the
// in-order MMA pipe and cost about a quarter of the MMA time.)  The
// block-scaled products and the 16-bit
// branch accumulate into the one fp32 accumulator in columns [0, 256), and
// the epilogue only rounds it to bf16.
#pragma once

#include "sq_gemm_common.cuh"

namespace sqg {

constexpr int PAIR_BM = 256;     // tile rows of the pair (128 per CTA)
constexpr int PAIR_BN = 256;     // tile columns (128 W rows per CTA)
constexpr int PAIR_EPI_WARP0 = 2;
constexpr int PAIR_EPI_WARPS = 8;  // two per TMEM lane quarter, each half of the columns
constexpr int PAIR_EXP_WARP0 = PAIR_EPI_WARP0 + PAIR_EPI_WARPS;
constexpr int PAIR_THREADS = 32 * (PAIR_EXP_WARP0 + NUM_EXP_WARPS);

template <int OPS_, int STG_, int NG_, int SF_ = 0, int YB_ = 0>
struct CfgPair {
    static constexpr int OPS = OPS_;                  // operand ring stages (expanded int8 or bf16 tiles)
    static constexpr int STG = STG_;                  // staging ring stages (packed INT4 tiles)
    static constexpr int NG = NG_;                    // producer groups; group g owns ring uses u = g mod NG
    static constexpr int GW = NUM_EXP_WARPS / NG;     // warps per producer group
    static constexpr int GT = 32 * GW;                // threads per producer group
    static constexpr int A_BYTES = 128 * ROWB;        // this CTA's X rows
    static constexpr int B_BYTES = 128 * ROWB;        // this CTA's W rows
    static constexpr int OP_BYTES = A_BYTES + B_BYTES;
    static constexpr int PA_BYTES = 128 * PROWB;      // packed X rows of one K-block
    static constexpr int STG_BYTES = 256 * PROWB;     // packed X + W rows of one K-block
    static constexpr int SF_BYTES = SF_;              // block scales per operand stage (MX only)
    static constexpr int YB = YB_;                    // Y staging boxes per epilogue warp (1 KB each); 0: per-lane stores
    static constexpr int OFF_OP = 0;
    static constexpr int OFF_SF = OPS * OP_BYTES;
    static constexpr int OFF_STG = OFF_SF + OPS * SF_BYTES;
    static constexpr int OFF_BAR = OFF_STG + STG * STG_BYTES;
    // barriers: op_full[OPS] op_empty[OPS] stg_full[STG] stg_empty[STG] acc_full acc_empty drain
    // low_full conv_done sf_full[OPS] (MX scales)
    static constexpr int NBAR = 2 * OPS + 2 * STG + 5 + (SF_ > 0 ? OPS : 0);
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr int OFF_SW = (OFF_MISC + 16 + 15) / 16 * 16;   // per epilogue warp: its 128 s_w values
    // Per epilogue warp: YB boxes of 32 x 16 bf16, the source of bulk tensor
    // stores, whose shared-memory address must be 128-byte aligned.
    static constexpr int OFF_YST = (OFF_SW + PAIR_EPI_WARPS * 128 * 4 + 127) / 128 * 128;
    static constexpr int SMEM_BYTES = OFF_YST + PAIR_EPI_WARPS * YB * 1024 + 1024;
    static constexpr int TMEM_COLS = 512;
    static constexpr int EXP_CHUNKS = 256 * (PROWB / 16) / GT;  // packed 16-byte chunks per thread per K-block
    static_assert(SMEM_BYTES <= 232448, "shared memory");
    static_assert(YB >= 0 && YB <= 2, "Y staging boxes");
    static_assert(OFF_YST % 128 == 0 && OFF_OP % 1024 == 0 && OFF_STG % 1024 == 0 && OFF_SF % 128 == 0,
                  "bulk tensor copies need 128-byte aligned shared memory (1024 for the 128-byte swizzle)");
    // Each slot of both rings must be used by a single producer group: a group
    // waiting on a slot only knows that its own earlier blocks have landed, and
    // bulk copies may complete out of order, so a slot shared by two groups
    // could still hold (or be receiving) the other group's block when the
    // phase-parity wait passes.
    static_assert(NUM_EXP_WARPS % NG == 0 && OPS % NG == 0 && STG % NG == 0,
                  "every ring slot must belong to one producer group");
};

// LOW selects the low path.  kLowFp8: E4M3 x E4M3 (kind::f8f6f4, OSC's FP8
// fallback for the inputs of W2) and kLowMx: block-scaled E2M1 (kind::mxf4):
// their tiles are plain bytes that TMA writes straight into the operand ring,
// so the staging ring and the expansion are compiled out and the low-path
// accumulator is fp32.  tm_sx / tm_sw (block scales) are used by kLowMx only.
template <class C, bool DBG, int LOW>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(PAIR_THREADS, 1)
dual_gemm_pair_kernel(const __grid_constant__ CUtensorMap tm_xo, const __grid_constant__ CUtensorMap tm_wo,
                      const __grid_constant__ CUtensorMap tm_xn, const __grid_constant__ CUtensorMap tm_wn,
                      const __grid_constant__ CUtensorMap tm_sx, const __grid_constant__ CUtensorMap tm_sw,
                      const __grid_constant__ CUtensorMap tm_y, const GemmArgs args)
{
    constexpr bool FP8 = LOW == kLowFp8;
    constexpr bool MX = LOW == kLowMx;
    constexpr bool SQF = LOW == kLowSqf;
    constexpr bool EXPAND = LOW == kLowInt4 || SQF;
    constexpr int OPS = C::OPS, EC = C::EXP_CHUNKS;
    static_assert(!MX || (C::GW == 4 && MX_SFA_COL + MX_SF_SLOT * OPS <= C::TMEM_COLS),
                  "MX: one producer warp per TMEM lane quarter, every slot's scale columns inside TMEM");
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = sqd::smem_u32(smem);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = sqd::cluster_ctarank();
    const bool leader = (rank == 0);
    sqd::pdl_launch_dependents();

    const uint32_t bar0 = sbase + C::OFF_BAR;
    auto op_full = [&](int e) { return bar0 + 8u * e; };
    auto op_empty = [&](int e) { return bar0 + 8u * (OPS + e); };
    constexpr int STG = C::STG;
    auto stg_full = [&](int i) { return bar0 + 8u * (2 * OPS + i); };
    auto stg_empty = [&](int i) { return bar0 + 8u * (2 * OPS + STG + i); };
    const uint32_t acc_full = bar0 + 8u * (2 * OPS + 2 * STG);
    const uint32_t acc_empty = acc_full + 8u;
    const uint32_t drain = acc_full + 16u;
    const uint32_t low_full = acc_full + 24u;   // (not MX) a tile's low-path sums are complete
    const uint32_t conv_done = acc_full + 32u;  // (not MX) both CTAs' epilogue warps have folded them
    auto sf_full = [&](int e) { return acc_full + 40u + 8u * e; };   // (MX) this CTA's scales of slot e landed
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::OFF_MISC);
    volatile uint32_t *abort_flag = reinterpret_cast<volatile uint32_t *>(smem + C::OFF_MISC + 4);
    auto op_a = [&](int e) { return sbase + C::OFF_OP + e * C::OP_BYTES; };
    auto stg_a = [&](int i) { return sbase + C::OFF_STG + i * C::STG_BYTES; };

    if (threadIdx.x == 0) {
        for (int e = 0; e < OPS; ++e) {
            // the owning group's warps in both CTAs (first CTA's copy); MX: plus the
            // byte-count arrival of each CTA's TMA thread
            sqd::mbar_init(op_full(e), 2 * (C::GW + (MX ? 1 : 0)));
            sqd::mbar_init(op_empty(e), 1);                 // multicast commit
            if constexpr (MX) sqd::mbar_init(sf_full(e), 1);   // this CTA's TMA thread (expect-tx)
        }
        for (int i = 0; i < STG; ++i) {
            sqd::mbar_init(stg_full(i), 1);                 // this CTA's staging TMA (expect-tx)
            sqd::mbar_init(stg_empty(i), C::GW);            // the consuming group's warps
        }
        sqd::mbar_init(acc_full, 1);                        // multicast commit
        sqd::mbar_init(acc_empty, 2 * PAIR_EPI_WARPS);      // epilogue warps of both CTAs (first CTA's copy)
        sqd::mbar_init(drain, 1);
        sqd::mbar_init(low_full, 1);                        // multicast commit
        sqd::mbar_init(conv_done, 2 * PAIR_EPI_WARPS);      // epilogue warps of both CTAs (first CTA's copy)
        *abort_flag = 0u;
        sqd::fence_barrier_init();
        sqd::fence_proxy_async_smem();
    }
    if (warp == 0 && lane == 0) {
        if (args.nkb_o > 0) {
            sqd::prefetch_tensormap(&tm_xo);
            sqd::prefetch_tensormap(&tm_wo);
        }
        if (args.nkb_i > 0) {
            sqd::prefetch_tensormap(&tm_xn);
            sqd::prefetch_tensormap(&tm_wn);
            if constexpr (MX) {
                sqd::prefetch_tensormap(&tm_sx);
                sqd::prefetch_tensormap(&tm_sw);
            }
        }
        if (args.y_tma) sqd::prefetch_tensormap(&tm_y);
    }
    if (warp == 1) {
        sqd::tmem_alloc_pair(sqd::smem_u32(tmem_slot), C::TMEM_COLS);
        sqd::tmem_relinquish_pair();
    }
    sqd::tc_fence_before();
    sqd::cluster_sync();  // barriers of both CTAs initialised, TMEM allocated in both
    sqd::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    sqd::pdl_wait();  // operands and Y may belong to the previous kernel

    const int nkb_i = args.nkb_i, nkb_o = args.nkb_o;
    const int per_tile = nkb_o + nkb_i;
    const int num_tiles = args.tiles_m * args.tiles_n;
    const int pair = static_cast<int>(blockIdx.x >> 1);
    const int num_pairs = static_cast<int>(gridDim.x >> 1);
    const int my_tiles = (num_tiles - pair + num_pairs - 1) / num_pairs;

    if (warp == 0) {
        // ------------------------------------------------------------ staging producer (each CTA)
        // Packed INT4 tiles of this CTA's X rows and W rows, one K-block per
        // stage, in the order the expansion warps consume them.
        if constexpr (EXPAND) if (lane == 0 && nkb_i > 0) {
            const int F = my_tiles * nkb_i;
            const int r0 = static_cast<int>(rank) * 128;
            int last_armed = -1;
            bool ok = true;
            for (int f = 0; f < F; ++f) {
                const int lt = f / nkb_i;
                const int kb = f - lt * nkb_i;
                int tmi, tni;
                tile_coords(args, pair + lt * num_pairs, tmi, tni);
                const int si = f % STG;
                if (!sqd::mbar_wait(stg_empty(si), ((f / STG) & 1) ^ 1u, abort_flag, SITE_EXP_OP)) { ok = false; break; }
                sqd::mbar_arrive_expect_tx(stg_full(si), C::STG_BYTES);
                sqd::tma_load_2d(stg_a(si), &tm_xn, stg_full(si), kb * PROWB, tmi * PAIR_BM + r0);
                sqd::tma_load_2d(stg_a(si) + C::PA_BYTES, &tm_wn, stg_full(si), kb * PROWB, tni * PAIR_BN + r0);
                last_armed = f;
            }
            if (!ok && last_armed >= 0) sqd::mbar_drain(stg_full(last_armed % STG), (last_armed / STG) & 1);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer (first CTA)
        if (leader && lane == 0) {
            constexpr uint32_t idesc_bf = sqd::make_idesc(false, PAIR_BM, PAIR_BN);
            constexpr uint32_t idesc_i8 = sqd::make_idesc(true, PAIR_BM, PAIR_BN);
            constexpr uint32_t idesc_f8 = sqd::make_idesc_e4m3(PAIR_BM, PAIR_BN);
            constexpr uint32_t idesc_mx = sqd::make_idesc_mxf4(PAIR_BM, PAIR_BN);
            bool ok = true;
            if (!MX && nkb_o == 0) {
                // No 16-bit branch: two acc_i buffers, columns [0, 256) for even tiles and
                // [256, 512) for odd ones, so tile t+1's MMAs run under tile t's epilogue.
                // Buffer r: full = acc_full / low_full, free = acc_empty / conv_done.
                for (int lt = 0; lt < my_tiles && ok; ++lt) {
                    const int r = lt & 1;
                    if (lt >= 2) {
                        if (!sqd::mbar_wait(r ? conv_done : acc_empty, static_cast<uint32_t>(((lt >> 1) - 1) & 1),
                                            abort_flag, SITE_MMA_ACC)) { ok = false; break; }
                        sqd::tc_fence_after();
                    }
                    const uint32_t d = tmem + static_cast<uint32_t>(r * PAIR_BN);
                    for (int i = 0; i < nkb_i; ++i) {
                        const int u = lt * per_tile + i;
                        const int e = u % OPS;
                        if (!sqd::mbar_wait(op_full(e), (u / OPS) & 1, abort_flag, SITE_MMA_FULL)) { ok = false; break; }
                        sqd::tc_fence_after();
                        const uint64_t adesc = sqd::make_sw128_desc(op_a(e));
                        const uint64_t bdesc = sqd::make_sw128_desc(op_a(e) + C::A_BYTES);
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            const uint32_t acc = (i == 0 && k == 0) ? 0u : 1u;
                            if constexpr (FP8) sqd::mma_f8_pair(d, adesc + 2 * k, bdesc + 2 * k, idesc_f8, acc);
                            else if constexpr (!MX) sqd::mma_s8_pair(d, adesc + 2 * k, bdesc + 2 * k, idesc_i8, acc);
                        }
                        sqd::mma_commit_pair_multicast(op_empty(e), 0x3);
                    }
                    if (ok) sqd::mma_commit_pair_multicast(r ? low_full : acc_full, 0x3);
                }
            } else if constexpr (!MX) {
                // Per tile: the low-path blocks into acc_i (columns [0, 256)); the epilogue
                // warps fold acc_i * s_x * s_w into columns [256, 512) (conv_done), which
                // frees acc_i for the next tile at once; the bf16 blocks then accumulate
                // on top of the folded values, and the epilogue only rounds and stores
                // them while the next tile's low blocks run.
                for (int lt = 0; lt < my_tiles && ok; ++lt) {
                    for (int i = 0; i < nkb_i; ++i) {
                        const int u = lt * per_tile + i;
                        const int e = u % OPS;
                        if (!sqd::mbar_wait(op_full(e), (u / OPS) & 1, abort_flag, SITE_MMA_FULL)) { ok = false; break; }
                        sqd::tc_fence_after();
                        const uint64_t adesc = sqd::make_sw128_desc(op_a(e));
                        const uint64_t bdesc = sqd::make_sw128_desc(op_a(e) + C::A_BYTES);
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            const uint32_t acc = (i == 0 && k == 0) ? 0u : 1u;
                            if constexpr (FP8) sqd::mma_f8_pair(tmem, adesc + 2 * k, bdesc + 2 * k, idesc_f8, acc);
                            else sqd::mma_s8_pair(tmem, adesc + 2 * k, bdesc + 2 * k, idesc_i8, acc);
                        }
                        sqd::mma_commit_pair_multicast(op_empty(e), 0x3);
                    }
                    if (!ok) break;
                    if (nkb_i > 0) sqd::mma_commit_pair_multicast(low_full, 0x3);
                    // The folded values are in place (and the previous tile's stores have read
                    // columns [256, 512)) once every epilogue warp of both CTAs has arrived.
                    if (!sqd::mbar_wait(conv_done, lt & 1, abort_flag, SITE_MMA_ACC)) { ok = false; break; }
                    sqd::tc_fence_after();
                    for (int i = nkb_i; i < per_tile; ++i) {
                        const int u = lt * per_tile + i;
                        const int e = u % OPS;
                        if (!sqd::mbar_wait(op_full(e), (u / OPS) & 1, abort_flag, SITE_MMA_FULL)) { ok = false; break; }
                        sqd::tc_fence_after();
                        const uint64_t adesc = sqd::make_sw128_desc(op_a(e));
                        const uint64_t bdesc = sqd::make_sw128_desc(op_a(e) + C::A_BYTES);
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            // without a low part nothing was folded in: the first MMA clears
                            const uint32_t acc = (nkb_i == 0 && i == 0 && k == 0) ? 0u : 1u;
                            sqd::mma_bf16_pair(tmem + static_cast<uint32_t>(PAIR_BN), adesc + 2 * k, bdesc + 2 * k,
                                               idesc_bf, acc);
                        }
                        sqd::mma_commit_pair_multicast(op_empty(e), 0x3);
                    }
                    if (ok) sqd::mma_commit_pair_multicast(acc_full, 0x3);
                }
            } else {
                // MX: the block-scaled products and the 16-bit branch share one fp32
                // accumulator (columns [0, 256)); the bf16 blocks come first.
                for (int lt = 0; lt < my_tiles && ok; ++lt) {
                    if (!sqd::mbar_wait(acc_empty, (lt & 1) ^ 1u, abort_flag, SITE_MMA_ACC)) { ok = false; break; }
                    sqd::tc_fence_after();
                    for (int i = 0; i < per_tile; ++i) {
                        const int u = lt * per_tile + i;
                        const int e = u % OPS;
                        if (!sqd::mbar_wait(op_full(e), (u / OPS) & 1, abort_flag, SITE_MMA_FULL)) { ok = false; break; }
                        sqd::tc_fence_after();
                        const bool is_bf = i < nkb_o;
                        const uint64_t adesc = sqd::make_sw128_desc(op_a(e));
                        const uint64_t bdesc = sqd::make_sw128_desc(op_a(e) + C::A_BYTES);
                        // the producer group wrote this slot's scales before arriving on op_full
                        const uint32_t sb = tmem + MX_SF_SLOT * static_cast<uint32_t>(e);
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            const uint32_t acc = (i == 0 && k == 0) ? 0u : 1u;
                            if (is_bf) {
                                sqd::mma_bf16_pair(tmem, adesc + 2 * k, bdesc + 2 * k, idesc_bf, acc);
                            } else {
                                // MMA k covers scale blocks 2k, 2k+1: K-tile k / 2, bytes 2 (k % 2) and up.
                                const uint32_t id = 2u * static_cast<uint32_t>(k & 1);
                                const uint32_t sfa = (sb + MX_SFA_COL + 4 * (k >> 1)) | (id << 30);
                                const uint32_t sfb = (sb + MX_SFB_COL + 8 * (k >> 1)) | (id << 30);
                                sqd::mma_mxf4_pair(tmem, adesc + 2 * k, bdesc + 2 * k, idesc_mx | (id << 29) | (id << 4),
                                                   acc, sfa, sfb);
                            }
                        }
                        sqd::mma_commit_pair_multicast(op_empty(e), 0x3);
                    }
                    if (ok) sqd::mma_commit_pair_multicast(acc_full, 0x3);
                }
            }
            if (!ok) {
                sqd::mma_commit_pair(drain);
                sqd::mbar_drain(drain, 0);
            }
        }
    } else if (warp >= PAIR_EXP_WARP0) {
        // ------------------------------------------------------------ operand producers
        const int gi = (warp - PAIR_EXP_WARP0) / C::GW;              // producer group
        const int et = threadIdx.x - (PAIR_EXP_WARP0 + gi * C::GW) * 32;  // thread index inside the group
        const uint32_t r0 = rank * 128u;  // this CTA's row offset inside the pair tile

        // INT4 block f: packed rows from staging stage f % STG -> int8 rows in
        // operand stage e (the tile's X rows, then its W rows).
        auto store = [&](int f) -> bool {
          if constexpr (!EXPAND) {
            return false;  // E4M3 and E2M1 tiles are never expanded
          } else {
            const int lt = f / nkb_i;
            const int kb = f - lt * nkb_i;
            const int u = lt * per_tile + kb;   // low blocks open the tile (not MX)
            const int e = u % OPS;
            const int si = f % STG;
            if (!sqd::mbar_wait(stg_full(si), (f / STG) & 1, abort_flag, SITE_EXP_OP)) return false;
            if (!sqd::mbar_wait(op_empty(e), ((u / OPS) & 1) ^ 1u, abort_flag, SITE_EXP_OP)) return false;
            const uint32_t src = stg_a(si);
            const uint32_t dst = op_a(e);
            uint4 w[EC];
#pragma unroll
            for (int c = 0; c < EC; ++c) {
                const int q = et + c * C::GT;
                w[c] = sqd::lds128(src + (q >> 2) * PROWB + (q & 3) * 16);
            }
#pragma unroll
            for (int c = 0; c < EC; ++c) {
                const int q = et + c * C::GT;
                const int r = q >> 2;
                const uint32_t j = static_cast<uint32_t>(q & 3);
                const uint32_t sw = static_cast<uint32_t>(r & 7);
                const uint32_t row = dst + r * ROWB;
                auto ex = [&](uint32_t v) { return SQF ? clear_mask_code(v) : v; };
                sqd::sts128(row + (((2u * j) ^ sw) << 4),
                            ex((w[c].x << 4) & 0xF0F0F0F0u), ex(w[c].x & 0xF0F0F0F0u),
                            ex((w[c].y << 4) & 0xF0F0F0F0u), ex(w[c].y & 0xF0F0F0F0u));
                sqd::sts128(row + (((2u * j + 1u) ^ sw) << 4),
                            ex((w[c].z << 4) & 0xF0F0F0F0u), ex(w[c].z & 0xF0F0F0F0u),
                            ex((w[c].w << 4) & 0xF0F0F0F0u), ex(w[c].w & 0xF0F0F0F0u));
            }
            sqd::fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                sqd::mbar_arrive(stg_empty(si));
                sqd::mbar_arrive_cluster(sqd::map_to_cta(op_full(e), 0));
            }
            return true;
          }
        };

        const bool tma_thread = (et == 0);
        int last_armed = -1;
        // Ring use u (tile lt) filled by TMA: the X and W tiles of map mx / mw
        // at K offset x (elements).  The group's first thread issues the two
        // loads with their byte count; every other warp of the group arrives.
        auto produce_tma = [&](int lt, int u, const CUtensorMap *mx, const CUtensorMap *mw, int x) -> bool {
            int tmi, tni;
            tile_coords(args, pair + lt * num_pairs, tmi, tni);
            const int e = u % OPS;
            if (!sqd::mbar_wait(op_empty(e), ((u / OPS) & 1) ^ 1u, abort_flag, SITE_EXP_OP)) return false;
            const uint32_t full_leader = sqd::map_to_cta(op_full(e), 0);
            if (tma_thread) {
                sqd::mbar_arrive_expect_tx_cluster(full_leader, C::OP_BYTES);
                sqd::tma_load_2d_pair(op_a(e), mx, full_leader, x, tmi * PAIR_BM + static_cast<int>(r0));
                sqd::tma_load_2d_pair(op_a(e) + C::A_BYTES, mw, full_leader, x, tni * PAIR_BN + static_cast<int>(r0));
                last_armed = u;
                if constexpr (MX) {
                    // no scales in this block: the first warp's own arrival, and the slot's
                    // sf_full phase passes too, so its parity keeps counting the slot's uses
                    sqd::mbar_arrive_cluster(full_leader);
                    sqd::mbar_arrive(sf_full(e));
                }
            } else if (lane == 0) {
                sqd::mbar_arrive_cluster(full_leader);
            }
            return true;
        };

        // MX ring use u (tile lt, low K-block kb): the packed E2M1 tiles plus
        // the block scales of this CTA's 128 X rows (one box: K-tiles 2kb,
        // 2kb+1) and of all 256 W rows of the tile (two boxes, one per
        // 128-row band).  Both CTAs of the pair need every W-row scale.  The
        // scales land on this CTA's sf_full; then each warp of the group writes
        // them into its lane quarter of the slot's TMEM scale columns: a tile's
        // byte 16 r + 4 c + j goes to byte j of column c of lane r in every
        // quarter (the layout the block-scaled MMA reads).
        int last_sf = -1;
        auto produce_mx = [&](int lt, int u, int kb) -> bool {
            if constexpr (MX) {
                int tmi, tni;
                tile_coords(args, pair + lt * num_pairs, tmi, tni);
                const int e = u % OPS;
                if (!sqd::mbar_wait(op_empty(e), ((u / OPS) & 1) ^ 1u, abort_flag, SITE_EXP_OP)) return false;
                sqd::tc_fence_after();   // the MMAs that read slot e's scale columns are done
                const uint32_t full_leader = sqd::map_to_cta(op_full(e), 0);
                const uint32_t sf = sbase + C::OFF_SF + e * C::SF_BYTES;
                if (tma_thread) {
                    const int na = 2 * nkb_i;  // scale tiles per 128-row band
                    sqd::mbar_arrive_expect_tx_cluster(full_leader, C::OP_BYTES);
                    sqd::tma_load_2d_pair(op_a(e), &tm_xn, full_leader, kb * (KB_MX / 2),
                                          tmi * PAIR_BM + static_cast<int>(r0));
                    sqd::tma_load_2d_pair(op_a(e) + C::A_BYTES, &tm_wn, full_leader, kb * (KB_MX / 2),
                                          tni * PAIR_BN + static_cast<int>(r0));
                    sqd::mbar_arrive_expect_tx(sf_full(e), C::SF_BYTES);
                    sqd::tma_load_2d(sf, &tm_sx, sf_full(e), 0, ((2 * tmi + static_cast<int>(rank)) * na + 2 * kb) * 4);
                    sqd::tma_load_2d(sf + 1024, &tm_sw, sf_full(e), 0, ((2 * tni) * na + 2 * kb) * 4);
                    sqd::tma_load_2d(sf + 2048, &tm_sw, sf_full(e), 0, ((2 * tni + 1) * na + 2 * kb) * 4);
                    last_armed = u;
                    last_sf = u;
                }
                if (!sqd::mbar_wait(sf_full(e), (u / OPS) & 1, abort_flag, SITE_EXP_OP)) return false;
                // columns +0..7: X rows, K-tiles 0 and 1; +8..23: W rows 0-127 and 128-255 of
                // K-tile 0, then of K-tile 1
                const uint4 x0 = sqd::lds128(sf + 16 * lane), x1 = sqd::lds128(sf + 512 + 16 * lane);
                const uint4 w00 = sqd::lds128(sf + 1024 + 16 * lane), w10 = sqd::lds128(sf + 2048 + 16 * lane);
                const uint4 w01 = sqd::lds128(sf + 1536 + 16 * lane), w11 = sqd::lds128(sf + 2560 + 16 * lane);
                const uint32_t va[16] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w,
                                         w00.x, w00.y, w00.z, w00.w, w10.x, w10.y, w10.z, w10.w};
                const uint32_t vb[8] = {w01.x, w01.y, w01.z, w01.w, w11.x, w11.y, w11.z, w11.w};
                const uint32_t tq = tmem + (static_cast<uint32_t>(32 * (warp & 3)) << 16) +
                                    static_cast<uint32_t>(MX_SFA_COL + MX_SF_SLOT * e);
                sqd::tmem_st_32x32b_x16(tq, va);
                sqd::tmem_st_32x32b_x8(tq + 16, vb);
                sqd::tmem_wait_st();
                sqd::tc_fence_before();
                __syncwarp();
                if (lane == 0) sqd::mbar_arrive_cluster(full_leader);
                return true;
            } else {
                return false;
            }
        };

        // Ring uses of this group, in order: u = gi, gi + NG, ...  Per tile the
        // low-path blocks (E4M3 by TMA, or INT4 expanded), then the bf16 blocks;
        // MX: the bf16 blocks, then the E2M1 blocks.
        bool ok = true;
        const int total = my_tiles * per_tile;
        for (int u = gi; u < total && ok; u += C::NG) {
            const int lt = u / per_tile;
            const int i = u - lt * per_tile;
            if constexpr (MX) {
                if (i < nkb_o) ok = produce_tma(lt, u, &tm_xo, &tm_wo, i * KB_BF);
                else ok = produce_mx(lt, u, i - nkb_o);
            } else if (i >= nkb_i) {
                ok = produce_tma(lt, u, &tm_xo, &tm_wo, (i - nkb_i) * KB_BF);
            } else if constexpr (FP8) {
                ok = produce_tma(lt, u, &tm_xn, &tm_wn, i * KB_I8);
            } else {
                ok = store(lt * nkb_i + i);
            }
        }
        if (!ok && tma_thread && last_armed >= 0 && leader) {
            // Let the last copies that were issued land before the CTA exits.
            sqd::mbar_drain(op_full(last_armed % OPS), (last_armed / OPS) & 1);
        }
        if (MX && !ok && tma_thread && last_sf >= 0) sqd::mbar_drain(sf_full(last_sf % OPS), (last_sf / OPS) & 1);
    } else if (warp >= PAIR_EPI_WARP0 && warp < PAIR_EPI_WARP0 + PAIR_EPI_WARPS) {
        // ------------------------------------------------------------ epilogue (each CTA: its 128 rows)
        // Warp w serves TMEM lane quarter w % 4 and half (w - 2) / 4 of the 256
        // columns, 16 columns at a time, the load of the next 16 columns in
        // flight while the current ones are processed.
        //
        // Not MX, per tile: (1) fold -- once the low-path sums are complete, each
        // value y0 = ((float)acc_i * s_x) * s_w (+ the SQ-format high part) is
        // written into the columns of the 16-bit branch, [256, 512), which frees
        // acc_i for the next tile's MMAs (conv_done); the bf16 MMAs then
        // accumulate the branch on top of y0 in the same fp32 accumulator.
        // (2) store -- once the tile is complete, the columns are rounded to
        // bf16 and written to Y while the next tile's low blocks run.
        // With debug outputs the fold writes zeros instead, so the branch sum
        // stays separate, and the store adds y0 (from the exact sums just
        // written to dbg_i) the same way.
        // MX: the single accumulator is rounded into registers after the tile and handed
        // back before the stores (debug builds: one pass that also writes the fp32 sums).
        const int sub = warp & 3;
        const int half = (warp - PAIR_EPI_WARP0) >> 2;
        const uint32_t tl = tmem + (static_cast<uint32_t>(sub * 32) << 16);
        const bool has_i = nkb_i > 0, has_o = nkb_o > 0;
        const uint32_t empty_leader = sqd::map_to_cta(acc_empty, 0);
        const uint32_t conv_leader = sqd::map_to_cta(conv_done, 0);
        constexpr int CW = 16;                   // columns per TMEM load
        constexpr int NCH = (PAIR_BN / 2) / CW;  // 8 loads per accumulator per warp
        static_assert(CW == 16, "one staging box is 16 columns");
        const bool y_tma = C::YB > 0 && args.y_tma != 0;
        const bool split = DBG && args.dbg_i != nullptr;   // keep the branch sum apart (debug outputs)
        const uint32_t yst = sbase + C::OFF_YST + (warp - PAIR_EPI_WARP0) * C::YB * 1024;
        const uint32_t sw_smem = sbase + C::OFF_SW + (warp - PAIR_EPI_WARP0) * 512;
        const uint32_t acc_col = MX ? 0u : static_cast<uint32_t>(PAIR_BN);   // what the store pass reads
        // Y is written once: its lines go first when L2 needs room, so the X band
        // and the W tiles that later tiles reuse stay resident.
        const uint64_t y_policy = sqd::l2_evict_first();
        // Not MX and no 16-bit branch: two acc_i buffers, no fold; the store pass
        // applies the scales itself.
        const bool dbuf = !MX && !has_o;
        int last_box = -1;  // staging box of this warp's latest bulk store
        for (int lt = 0; lt < my_tiles; ++lt) {
            int tmi, tni;
            tile_coords(args, pair + lt * num_pairs, tmi, tni);
            const int m = tmi * PAIR_BM + static_cast<int>(rank) * 128 + sub * 32 + lane;
            const bool row_ok = m < args.M;
            const int c_base = half * (PAIR_BN / 2);
            // Scales of this warp's 128 columns and of this lane's row, fetched
            // while the tile's MMAs still run.
            const int ncol = tni * PAIR_BN + c_base + 4 * lane;
            const float4 swp = (!MX && ncol < args.N) ? __ldg(reinterpret_cast<const float4 *>(args.s_w + ncol))
                                                      : make_float4(0.f, 0.f, 0.f, 0.f);
            const float sx = (!MX && row_ok) ? args.s_x[m] : 0.0f;
            uint16_t *yrow = args.Y + static_cast<long long>(row_ok ? m : 0) * args.ldy;
            const int m0 = tmi * PAIR_BM + static_cast<int>(rank) * 128 + sub * 32;  // this warp's first row

            if (!MX && !dbuf) {
                // ---------------------------------------------------- (1) fold
                if (has_i) {
                    if (!sqd::mbar_wait(low_full, lt & 1, abort_flag, SITE_EPI)) break;
                    sqd::tc_fence_after();
                    sqd::sts128(sw_smem + 16 * lane, __float_as_uint(swp.x), __float_as_uint(swp.y),
                                __float_as_uint(swp.z), __float_as_uint(swp.w));
                    __syncwarp();
                    uint32_t va[2][CW];
                    sqd::tmem_ld_32x32b_x16(tl + c_base, va[0]);
                    sqd::tmem_wait_ld_dep1(va[0]);
#pragma unroll
                    for (int ch = 0; ch < NCH; ++ch) {
                        const int b = ch & 1;
                        if (ch + 1 < NCH) sqd::tmem_ld_32x32b_x16(tl + c_base + (ch + 1) * CW, va[b ^ 1]);
                        const int n0 = tni * PAIR_BN + c_base + ch * CW;
                        uint32_t y0[CW];
#pragma unroll
                        for (int g = 0; g < CW / 8; ++g) {
                            const int n = n0 + 8 * g;
                            const bool ok8 = row_ok && n < args.N;  // N is a multiple of 8
                            const uint4 sw0 = sqd::lds128(sw_smem + 4 * (ch * CW + 8 * g));
                            const uint4 sw1 = sqd::lds128(sw_smem + 4 * (ch * CW + 8 * g + 4));
                            const float swv[8] = {__uint_as_float(sw0.x), __uint_as_float(sw0.y), __uint_as_float(sw0.z),
                                                  __uint_as_float(sw0.w), __uint_as_float(sw1.x), __uint_as_float(sw1.y),
                                                  __uint_as_float(sw1.z), __uint_as_float(sw1.w)};
                            float adv[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                            if constexpr (SQF) {
                                // the precomputed high part of these 8 outputs
                                if (ok8 && !split) {
                                    const float4 *ap = reinterpret_cast<const float4 *>(args.addend + static_cast<long long>(m) * args.N + n);
                                    const float4 a0 = ap[0], a1 = ap[1];
                                    adv[0] = a0.x; adv[1] = a0.y; adv[2] = a0.z; adv[3] = a0.w;
                                    adv[4] = a1.x; adv[5] = a1.y; adv[6] = a1.z; adv[7] = a1.w;
                                }
                            }
#pragma unroll
                            for (int q = 0; q < 8; ++q) {
                                const int t = 8 * g + q;
                                // exact int32 sum (x256) for INT4, fp32 sum for E4M3
                                float al;
                                int32_t dbg_lo;
                                if constexpr (FP8) {
                                    al = __uint_as_float(va[b][t]);
                                    dbg_lo = __float_as_int(al);
                                } else {
                                    const int ai = static_cast<int>(va[b][t]) >> 8;
                                    al = static_cast<float>(ai);
                                    dbg_lo = ai;
                                }
                                const float v = __fadd_rn(__fmul_rn(__fmul_rn(al, sx), swv[q]), adv[q]);
                                y0[t] = split ? 0u : __float_as_uint(v);
                                if constexpr (DBG) {
                                    if (ok8 && args.dbg_i) args.dbg_i[static_cast<long long>(m) * args.N + n + q] = dbg_lo;
                                }
                            }
                        }
                        sqd::tmem_st_32x32b_x16(tl + PAIR_BN + c_base + ch * CW, y0);
                        if (ch + 1 < NCH) sqd::tmem_wait_ld_dep1(va[b ^ 1]);
                    }
                    sqd::tmem_wait_st();
                }
                // acc_i has been read and [256, 512) holds y0 (and this warp's stores of
                // the previous tile have read those columns): the MMAs may go on.
                sqd::tc_fence_before();
                __syncwarp();
                if (lane == 0) sqd::mbar_arrive_cluster(conv_leader);
            }

            if constexpr (MX && !DBG) {
                // MX: the warp's 128 columns are rounded to bf16 into registers as they are
                // read, the accumulator goes back to the next tile's MMAs, and only then are
                // the rows stored (the stores overlap the next tile's MMAs).
                if (!sqd::mbar_wait(acc_full, lt & 1, abort_flag, SITE_EPI)) break;
                sqd::tc_fence_after();
                uint32_t pk[NCH][CW / 2];
#pragma unroll
                for (int ch = 0; ch < NCH; ++ch) {
                    uint32_t v[CW];
                    sqd::tmem_ld_32x32b_x16(tl + c_base + ch * CW, v);
                    sqd::tmem_wait_ld_dep1(v);
#pragma unroll
                    for (int h = 0; h < CW / 2; ++h) {
                        const __nv_bfloat162 b2 = __floats2bfloat162_rn(__uint_as_float(v[2 * h]), __uint_as_float(v[2 * h + 1]));
                        pk[ch][h] = *reinterpret_cast<const uint32_t *>(&b2);
                    }
                }
                sqd::tc_fence_before();
                __syncwarp();
                if (lane == 0) sqd::mbar_arrive_cluster(empty_leader);
#pragma unroll
                for (int ch = 0; ch < NCH; ++ch) {
                    const int n0 = tni * PAIR_BN + c_base + ch * CW;
                    if (!(y_tma ? (m0 < args.M && n0 < args.N) : (row_ok && n0 < args.N))) continue;
                    if (y_tma) {
                        // the one staging box of this warp: its previous bulk store has read it
                        if (lane == 0) sqd::bulk_wait_read<0>();
                        __syncwarp();
                        const uint32_t box = yst;
                        sqd::sts128(box + 32 * lane, pk[ch][0], pk[ch][1], pk[ch][2], pk[ch][3]);
                        sqd::sts128(box + 32 * lane + 16, pk[ch][4], pk[ch][5], pk[ch][6], pk[ch][7]);
                        sqd::fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0) {
                            sqd::tma_store_2d_hint(&tm_y, box, n0, m0, y_policy);
                            sqd::bulk_commit();
                        }
                    } else {
#pragma unroll
                        for (int g = 0; g < CW / 8; ++g) {
                            const int n = n0 + 8 * g;
                            if (n < args.N)
                                sqd::stg128_hint(yrow + n, make_uint4(pk[ch][4 * g], pk[ch][4 * g + 1], pk[ch][4 * g + 2],
                                                                      pk[ch][4 * g + 3]), y_policy);
                        }
                    }
                }
                continue;
            }

            // -------------------------------------------------------- (2) store
            const int rb = dbuf ? (lt & 1) : 0;   // accumulator buffer of this tile (double-buffer mode)
            if (!sqd::mbar_wait(rb ? low_full : acc_full, static_cast<uint32_t>(dbuf ? ((lt >> 1) & 1) : (lt & 1)),
                                abort_flag, SITE_EPI))
                break;
            sqd::tc_fence_after();
            if (dbuf) {
                sqd::sts128(sw_smem + 16 * lane, __float_as_uint(swp.x), __float_as_uint(swp.y), __float_as_uint(swp.z),
                            __float_as_uint(swp.w));
                __syncwarp();
            }
            const uint32_t col = dbuf ? static_cast<uint32_t>(rb * PAIR_BN) : acc_col;
            const bool has_acc = MX || has_i || has_o;
            uint32_t vf[2][CW] = {};
            if (has_acc) {
                sqd::tmem_ld_32x32b_x16(tl + col + c_base, vf[0]);
                sqd::tmem_wait_ld_dep1(vf[0]);
            }
#pragma unroll
            for (int ch = 0; ch < NCH; ++ch) {
                const int b = ch & 1;
                if (has_acc && ch + 1 < NCH) sqd::tmem_ld_32x32b_x16(tl + col + c_base + (ch + 1) * CW, vf[b ^ 1]);
                const int n0 = tni * PAIR_BN + c_base + ch * CW;
                // Bulk-store form: all 32 lanes fill the 32 x 16 box (the store
                // drops rows past M and columns past N); otherwise each lane
                // stores its own row.
                if (y_tma ? (m0 < args.M && n0 < args.N) : (row_ok && n0 < args.N)) {
                    // Staging box (two alternate when YB == 2): wait until the bulk
                    // store that last read it is done.
                    const int bb = C::YB == 2 ? b : 0;
                    const uint32_t box = yst + 1024u * static_cast<uint32_t>(bb);
                    if (y_tma) {
                        if (lane == 0) {
                            if (C::YB == 2 && last_box == (bb ^ 1)) sqd::bulk_wait_read<1>();
                            else sqd::bulk_wait_read<0>();
                        }
                        __syncwarp();
                    }
#pragma unroll
                    for (int g = 0; g < CW / 8; ++g) {
                        const int n = n0 + 8 * g;
                        const bool ok8 = row_ok && n < args.N;  // N is a multiple of 8
                        float swv[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                        float adv[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                        if (dbuf) {
                            const uint4 sw0 = sqd::lds128(sw_smem + 4 * (ch * CW + 8 * g));
                            const uint4 sw1 = sqd::lds128(sw_smem + 4 * (ch * CW + 8 * g + 4));
                            swv[0] = __uint_as_float(sw0.x); swv[1] = __uint_as_float(sw0.y);
                            swv[2] = __uint_as_float(sw0.z); swv[3] = __uint_as_float(sw0.w);
                            swv[4] = __uint_as_float(sw1.x); swv[5] = __uint_as_float(sw1.y);
                            swv[6] = __uint_as_float(sw1.z); swv[7] = __uint_as_float(sw1.w);
                            if constexpr (SQF) {
                                // the precomputed high part of these 8 outputs
                                if (ok8) {
                                    const float4 *ap = reinterpret_cast<const float4 *>(args.addend + static_cast<long long>(m) * args.N + n);
                                    const float4 a0 = ap[0], a1 = ap[1];
                                    adv[0] = a0.x; adv[1] = a0.y; adv[2] = a0.z; adv[3] = a0.w;
                                    adv[4] = a1.x; adv[5] = a1.y; adv[6] = a1.z; adv[7] = a1.w;
                                }
                            }
                        }
                        uint32_t out[4];
#pragma unroll
                        for (int h = 0; h < 4; ++h) {
                            float y2[2];
#pragma unroll
                            for (int u = 0; u < 2; ++u) {
                                const int t = 8 * g + 2 * h + u;
                                const float acc = __uint_as_float(vf[b][t]);
                                y2[u] = acc;
                                if (dbuf) {
                                    // exact int32 sum (x256) for INT4, fp32 sum for E4M3, scaled here
                                    float al;
                                    int32_t dbg_lo;
                                    if constexpr (FP8) {
                                        al = has_i ? acc : 0.0f;
                                        dbg_lo = __float_as_int(al);
                                    } else {
                                        const int ai = has_i ? (static_cast<int>(vf[b][t]) >> 8) : 0;
                                        al = static_cast<float>(ai);
                                        dbg_lo = ai;
                                    }
                                    y2[u] = __fadd_rn(__fmul_rn(__fmul_rn(al, sx), swv[2 * h + u]), adv[2 * h + u]);
                                    if constexpr (DBG) {
                                        const long long o = static_cast<long long>(m) * args.N + n + 2 * h + u;
                                        if (ok8 && args.dbg_i) args.dbg_i[o] = dbg_lo;
                                        if (ok8 && args.dbg_f) args.dbg_f[o] = adv[2 * h + u];
                                    }
                                    continue;
                                }
                                if constexpr (DBG) {
                                    const long long o = static_cast<long long>(m) * args.N + n + 2 * h + u;
                                    if (MX && ok8 && args.dbg_f) args.dbg_f[o] = acc;
                                    if (!MX && !has_i && ok8 && args.dbg_i) args.dbg_i[o] = 0;  // no low part
                                    if (!MX && split && ok8) {
                                        // y0 from the exact low-path sum written by the fold pass
                                        float al = 0.0f, swq = 0.0f;
                                        if (has_i) {
                                            al = FP8 ? __int_as_float(args.dbg_i[o]) : static_cast<float>(args.dbg_i[o]);
                                            swq = __uint_as_float(sqd::lds32(sw_smem + 4 * (ch * CW + 8 * g + 2 * h + u)));
                                        }
                                        const float af = SQF ? args.addend[o] : acc;
                                        y2[u] = __fadd_rn(__fmul_rn(__fmul_rn(al, sx), swq), af);
                                        if (args.dbg_f) args.dbg_f[o] = af;
                                    }
                                }
                            }
                            const __nv_bfloat162 b2 = __floats2bfloat162_rn(y2[0], y2[1]);
                            out[h] = *reinterpret_cast<const uint32_t *>(&b2);
                        }
                        if (y_tma) sqd::sts128(box + 32 * lane + 16 * g, out[0], out[1], out[2], out[3]);
                        else if (n < args.N) sqd::stg128_hint(yrow + n, make_uint4(out[0], out[1], out[2], out[3]), y_policy);
                    }
                    if (y_tma) {
                        sqd::fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0) {
                            sqd::tma_store_2d_hint(&tm_y, box, n0, m0, y_policy);
                            sqd::bulk_commit();
                        }
                        last_box = bb;
                    }
                }
                if (has_acc && ch + 1 < NCH) {
                    sqd::tmem_wait_ld_dep1(vf[b ^ 1]);
                    if ((MX || dbuf) && ch + 2 == NCH) {
                        // Last load of this warp landed: the accumulator (buffer) may be reused.
                        sqd::tc_fence_before();
                        __syncwarp();
                        if (lane == 0) sqd::mbar_arrive_cluster(rb ? conv_leader : empty_leader);
                    }
                }
            }
        }
        if (y_tma && lane == 0) sqd::bulk_wait_all();  // the staging boxes stay valid until stored
    }

    sqd::tc_fence_before();
    sqd::cluster_sync();  // every pair MMA and every TMEM read of both CTAs is done
    if (warp == 1) {
        sqd::tc_fence_after();
        sqd::tmem_dealloc_pair(tmem, C::TMEM_COLS);
    }
}

}  // namespace sqg
