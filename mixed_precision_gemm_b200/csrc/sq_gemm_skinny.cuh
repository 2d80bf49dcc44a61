// Dual-path GEMM for few tokens (M <= 128): swapped operands, K split over a
// cluster.  Same computation as sq_gemm_pair.cuh (OSC, arXiv:2604.12782,
// abstract: a 4-bit GEMM path plus a 16-bit branch GEMM on the compact
// outlier tensor, fused).
//
// With few tokens the layer is a stream over the weights: every packed W byte
// is read once and the arithmetic per byte is small.  Three choices follow.
//
// Swapped operands.  The MMA computes D^T = W . X^T: the 128 W rows of a tile
// are the MMA's M side (the TMEM lanes) and the MP tokens (MP = M rounded up
// to 16, 32, 64 or 128) are its N side, so no MMA work is spent on token rows
// that do not exist.  D holds 128 output channels x MP tokens.
//
// Split K.  The K-blocks of one 128-row W tile (INT4 blocks of 128 channels
// first, then bf16 blocks of 64 outlier channels, weighted 1 and 2 by their
// bytes) are divided into S contiguous ranges of equal byte count, one per
// CTA of a cluster of S (S <= 8), so that tiles_n * S CTAs stream W at once.
// The S partial accumulators are summed through distributed shared memory:
// CTA r of the cluster owns rows [r*RP, (r+1)*RP) of the tile (RP =
// ceil(128/S)); every CTA sends the owner its int32 and fp32 partials of
// those rows; the owner adds them (int32 exactly, fp32 in rank order) and
// writes Y.  The reduction buffer reuses the rings, which are idle once every
// MMA of the cluster has completed (first cluster barrier).
//
// Wide loads, deep ring.  Weight rows are fetched 128 bytes at a time (two
// packed INT4 K-blocks, or one bf16 K-block) with the 128-byte swizzle, into
// a staging ring of 96-180 KB, which keeps enough bytes in flight per SM to
// stream HBM.  bf16 stages are read by the MMA where they land; INT4 stages
// are expanded into a small ring of int8 operand slots (with C::TA: the W
// rows into tensor memory, the token rows into shared memory).
//
// Roles (6 warps, one tile-split per CTA):
//   warp 0      TMA producer of the staging ring: for each stage, 128 W rows
//               and MP token rows of 128 bytes.
//   warp 1      allocates TMEM; one lane issues every MMA and commits.
//   warps 2..5  expand INT4 stages (both K-blocks at once) into the operand
//               ring, in order: with C::TA one thread per W row (its TMEM
//               lane), writing the row's int8 codes with tcgen05.st, and the
//               token rows spread over all threads; otherwise eight threads
//               per 128-byte row.  Afterwards they run the epilogue.
// Stage order is every INT4 stage, then every bf16 stage.  The INT4 stages
// are consumed by the expansion warps and the bf16 stages by the MMA issuer;
// because all INT4 stages come first, each consumer's earlier uses of a slot
// were its own or were consumed before it reached the slot, so the
// phase-parity waits cannot alias.
// TMEM: acc_i (int32) in columns [0, MP), acc_f (fp32) in [MP, 2 MP); with
// C::TA the W-operand slots follow from column C::TA_COL, 32 columns each.
//
// MX low path (kLowMx): a stage is one K-block of 256 E2M1 codes (128 bytes
// per row) read by the MMA in place, plus two 1 KB scale boxes: the W rows'
// (two K-tiles of the tile's 128-row band) and the tokens' (band 0).  The MMA
// thread copies them into TMEM (columns MP .. MP+7 for W, MP+8 .. MP+15 for
// the tokens) before the K-block's four kind::mxf4 MMAs; the 16-bit branch
// adds into the same fp32 accumulator in [0, MP), and only that accumulator
// is reduced over the cluster.
#pragma once

#include "sq_gemm_common.cuh"

namespace sqg {

constexpr int SK_PROD_WARP0 = 2;
constexpr int SK_PROD_WARPS = 4;
constexpr int SK_THREADS = 32 * (SK_PROD_WARP0 + SK_PROD_WARPS);
constexpr int SK_PT = 32 * SK_PROD_WARPS;  // expansion threads (= TMEM lanes)
constexpr int SK_MAX_SPLITS = 8;

enum : unsigned { SITE_SK_STG = 0x501, SITE_SK_OP = 0x502, SITE_SK_MMA = 0x503, SITE_SK_EPI = 0x504 };

template <int MP_, int NST_, int OPS_, int SF_ = 0, bool TA_ = false>
struct CfgSkinny {
    static constexpr int MP = MP_;                    // token columns of D (MMA N)
    static constexpr int NST = NST_;                  // staging ring stages
    static constexpr int OPS = OPS_;                  // expanded int8 operand ring stages
    static constexpr int SF_BYTES = SF_;              // block scales per staging stage (MX only)
    // INT4 with the W operand in tensor memory: each expansion thread writes
    // its W row's int8 codes straight into TMEM (the MMA's A operand), and only
    // the token rows go through a shared-memory operand tile.
    static constexpr bool TA = TA_;
    static constexpr int ROWS = 128 + MP;             // W rows, then token rows, in every tile
    static constexpr int A_BYTES = 128 * ROWB;
    static constexpr int TILE_BYTES = ROWS * ROWB;    // one stage = one operand tile (128-byte rows)
    static constexpr int OP_BYTES = TA ? MP * ROWB : TILE_BYTES;  // one operand ring slot
    static constexpr int OFF_STG = 0;
    static constexpr int OFF_OP = NST * TILE_BYTES;
    static constexpr int OFF_SF = OFF_OP + OPS * OP_BYTES;
    static constexpr int OFF_BAR = OFF_SF + NST * SF_BYTES;
    // barriers: stg_full[NST] stg_empty[NST] op_full[OPS] op_empty[OPS] acc_full drain
    static constexpr int NBAR = 2 * NST + 2 * OPS + 2;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr int OFF_CNT = OFF_MISC + 16;           // per staging slot: expansion warps done
    // Row scales for the epilogue, fetched at the start: s_w of the tile's 128
    // W rows, then s_x of the MP token columns (0 past N or M).
    static constexpr int OFF_SCL = (OFF_CNT + NST * 4 + 15) / 16 * 16;
    static constexpr int SMEM_BYTES = OFF_SCL + (128 + MP) * 4 + 1024;
    // MX: the accumulator [0, MP) and 16 scale columns; otherwise two
    // accumulators, and with TA the OPS W-operand slots (32 columns = 128 int8
    // K-elements per lane each) from column TA_COL.
    static constexpr int COL_F = SF_ > 0 ? 0 : MP;   // fp32 accumulator of the 16-bit branch
    static constexpr int TA_COL = 2 * MP < 32 ? 32 : 2 * MP;
    static constexpr int TMEM_NEED = SF_ > 0 ? MP + 16 : TA ? TA_COL + 32 * OPS : 2 * MP;
    static constexpr int TMEM_COLS = TMEM_NEED <= 32 ? 32 : TMEM_NEED <= 64 ? 64 : TMEM_NEED <= 128 ? 128
                                   : TMEM_NEED <= 256 ? 256 : 512;
    static constexpr int EXP_CHUNKS = ROWS * 8 / SK_PT;   // 16-byte packed chunks per thread per stage
    // Reduction buffer (aliases the rings): int32 and fp32 regions of
    // S * RP <= 128 + S - 1 partial rows, RSTRIDE words apart.
    static constexpr int RSTRIDE = MP + 4;
    static constexpr int RED_ROWS = 128 + SK_MAX_SPLITS - 1;
    static constexpr int OFF_RED_I = 0;
    static constexpr int OFF_RED_F = RED_ROWS * RSTRIDE * 4;
    static_assert(MP == 16 || MP == 32 || MP == 64 || MP == 128, "MP");
    static_assert(TILE_BYTES % 1024 == 0 && OP_BYTES % 1024 == 0, "tiles must stay 1024-byte aligned");
    static_assert(TMEM_NEED <= 512, "tensor memory");
    static_assert(!TA || SF_ == 0, "TA is an INT4 layout");
    static_assert(ROWS * 8 % SK_PT == 0, "expansion work split");
    static_assert(OPS >= 2 || SF_ > 0, "an INT4 stage fills two operand tiles");
    static_assert(2 * RED_ROWS * RSTRIDE * 4 <= OFF_BAR, "reduction buffer must fit in the rings");
    static_assert(SMEM_BYTES <= 232448, "shared memory");
};

struct SkinnyArgs {
    const float *addend;   // SQF: fp32 [M, N] added in place of the 16-bit branch
    const float *s_x;
    const float *s_w;
    uint16_t *Y;
    int32_t *dbg_i;
    float *dbg_f;
    int M, N;
    long long ldy;
    int nkb_i;   // INT4 K-blocks (kn_pad / 128)
    int nkb_o;   // bf16 K-blocks (no_pad / 64)
    int splits;  // CTAs per cluster = K ranges per W tile
};

// First K-block of split r of S: blocks 0..nkb_i-1 are low-path blocks of
// lw 64-byte units per W row (INT4: 1; MX: 2), then nkb_o bf16 blocks (2
// units); the split points are the block boundaries at or after r/S of the
// total bytes.
__device__ __forceinline__ int skinny_first_block(int r, int S, int nkb_i, int nkb_o, int lw)
{
    const int cost = lw * nkb_i + 2 * nkb_o;
    const int c = static_cast<int>(static_cast<long long>(cost) * r / S);
    return c <= lw * nkb_i ? (c + lw - 1) / lw : nkb_i + (c - lw * nkb_i + 1) / 2;
}

// LOW selects the low path.  kLowFp8 (E4M3 x E4M3, kind::f8f6f4, OSC's FP8
// fallback for the inputs of W2) and kLowMx (block-scaled E2M1, kind::mxf4):
// a stage carries one K-block of bytes that the MMA reads in place, as for
// bf16 stages; the expansion warps only run the epilogue, and the low-path
// partials are fp32.  tm_sx / tm_sw (block scales) are used by kLowMx only.
template <class C, bool DBG, int LOW>
__global__ void __launch_bounds__(SK_THREADS, 1)
dual_gemm_skinny_kernel(const __grid_constant__ CUtensorMap tm_xo, const __grid_constant__ CUtensorMap tm_wo,
                        const __grid_constant__ CUtensorMap tm_xn, const __grid_constant__ CUtensorMap tm_wn,
                        const __grid_constant__ CUtensorMap tm_sx, const __grid_constant__ CUtensorMap tm_sw,
                        const SkinnyArgs args)
{
    constexpr bool FP8 = LOW == kLowFp8;
    constexpr bool MX = LOW == kLowMx;
    constexpr bool DIRECT = FP8 || MX;   // low-path stages read by the MMA in place
    constexpr bool SQF = LOW == kLowSqf;  // INT4 stages with the mask code -8 cleared, fp32 addend
    constexpr int MP = C::MP, NST = C::NST, OPS = C::OPS, EC = C::EXP_CHUNKS;
    // Modulus of the INT4 operand ring.  The direct-read configurations have no
    // ring (OPS = 0) and never run the code that uses it.
    constexpr int OPR = OPS > 0 ? OPS : 1;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = sqd::smem_u32(smem);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int S = args.splits;
    const int rank = static_cast<int>(sqd::cluster_ctarank());
    const int n0 = static_cast<int>(blockIdx.x) / S * 128;
    sqd::pdl_launch_dependents();

    const uint32_t bar0 = sbase + C::OFF_BAR;
    auto stg_full = [&](int s) { return bar0 + 8u * s; };
    auto stg_empty = [&](int s) { return bar0 + 8u * (NST + s); };
    auto op_full = [&](int e) { return bar0 + 8u * (2 * NST + e); };
    auto op_empty = [&](int e) { return bar0 + 8u * (2 * NST + OPS + e); };
    const uint32_t acc_full = bar0 + 8u * (2 * NST + 2 * OPS);
    const uint32_t drain = acc_full + 8u;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::OFF_MISC);
    volatile uint32_t *abort_flag = reinterpret_cast<volatile uint32_t *>(smem + C::OFF_MISC + 4);
    uint32_t *stg_done = reinterpret_cast<uint32_t *>(smem + C::OFF_CNT);
    auto stg_a = [&](int s) { return sbase + C::OFF_STG + s * C::TILE_BYTES; };
    auto op_a = [&](int e) { return sbase + C::OFF_OP + e * C::OP_BYTES; };
    // token rows of operand slot e (with TA the slot holds nothing else)
    auto op_b = [&](int e) { return op_a(e) + (C::TA ? 0 : C::A_BYTES); };

    // This CTA's K range: INT4 blocks [i_lo, i_lo + n_i) in ns_i stages of
    // two, then bf16 blocks [o_lo, o_lo + n_o), one stage each.
    const int nkb_i = args.nkb_i, nkb_o = args.nkb_o;
    const int lw = MX ? 2 : 1;
    const int b_lo = skinny_first_block(rank, S, nkb_i, nkb_o, lw);
    const int b_hi = skinny_first_block(rank + 1, S, nkb_i, nkb_o, lw);
    const int i_lo = min(b_lo, nkb_i);
    const int n_i = min(b_hi, nkb_i) - i_lo;
    const int o_lo = max(b_lo, nkb_i) - nkb_i;
    const int n_o = max(b_hi, nkb_i) - nkb_i - o_lo;
    const int ns_i = DIRECT ? n_i : (n_i + 1) / 2;
    const int ns = ns_i + n_o;

    if (threadIdx.x == 0) {
        for (int s = 0; s < NST; ++s) {
            sqd::mbar_init(stg_full(s), 1);   // TMA producer (expect-tx)
            sqd::mbar_init(stg_empty(s), 1);  // the last expansion warp, or the MMA commit
            stg_done[s] = 0u;
        }
        for (int e = 0; e < OPS; ++e) {
            sqd::mbar_init(op_full(e), SK_PROD_WARPS);
            sqd::mbar_init(op_empty(e), 1);
        }
        sqd::mbar_init(acc_full, 1);
        sqd::mbar_init(drain, 1);
        *abort_flag = 0u;
        sqd::fence_barrier_init();
        sqd::fence_proxy_async_smem();
    }
    if (warp == 0 && lane == 0) {
        if (n_o > 0) {
            sqd::prefetch_tensormap(&tm_xo);
            sqd::prefetch_tensormap(&tm_wo);
        }
        if (n_i > 0) {
            sqd::prefetch_tensormap(&tm_xn);
            sqd::prefetch_tensormap(&tm_wn);
            if constexpr (MX) {
                sqd::prefetch_tensormap(&tm_sx);
                sqd::prefetch_tensormap(&tm_sw);
            }
        }
    }
    if (warp == 1) {
        sqd::tmem_alloc(sqd::smem_u32(tmem_slot), C::TMEM_COLS);
        sqd::tmem_relinquish();
    }
    sqd::tc_fence_before();
    __syncthreads();
    sqd::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    sqd::pdl_wait();  // operands and Y may belong to the previous kernel

    // The epilogue's row scales, loaded now so that their latency is hidden
    // behind the main loop (read after the cluster barriers below).
    float *scl_w = reinterpret_cast<float *>(smem + C::OFF_SCL);
    float *scl_x = scl_w + 128;
    if (!MX && warp >= SK_PROD_WARP0) {
        const int et = threadIdx.x - SK_PROD_WARP0 * 32;
        scl_w[et] = n0 + et < args.N ? __ldg(args.s_w + n0 + et) : 0.0f;
        if (et < MP) scl_x[et] = et < args.M ? __ldg(args.s_x + et) : 0.0f;
    }

    if (warp == 0) {
        // ------------------------------------------------------------ staging producer
        if (lane == 0) {
            int last_armed = -1;
            bool ok = true;
            for (int t = 0; t < ns; ++t) {
                const int s = t % NST;
                if (!sqd::mbar_wait(stg_empty(s), ((t / NST) & 1) ^ 1u, abort_flag, SITE_SK_STG)) { ok = false; break; }
                if constexpr (MX) {
                    if (t < ns_i) {
                        // codes of K-block kb (128 bytes per row), and the scale tiles 2kb, 2kb+1 of
                        // the W rows' band and of the tokens' band 0
                        const int kb = i_lo + t;
                        const uint32_t sf = sbase + C::OFF_SF + s * C::SF_BYTES;
                        sqd::mbar_arrive_expect_tx(stg_full(s), C::TILE_BYTES + C::SF_BYTES);
                        sqd::tma_load_2d(stg_a(s), &tm_wn, stg_full(s), kb * (KB_MX / 2), n0);
                        sqd::tma_load_2d(stg_a(s) + C::A_BYTES, &tm_xn, stg_full(s), kb * (KB_MX / 2), 0);
                        sqd::tma_load_2d(sf, &tm_sw, stg_full(s), 0, ((n0 / 128) * 2 * nkb_i + 2 * kb) * 4);
                        sqd::tma_load_2d(sf + 1024, &tm_sx, stg_full(s), 0, (2 * kb) * 4);
                        last_armed = t;
                        continue;
                    }
                }
                sqd::mbar_arrive_expect_tx(stg_full(s), C::TILE_BYTES);
                if (t < ns_i) {
                    // byte offset of the stage's first K-block (two INT4 blocks, or one E4M3 block)
                    const int x = FP8 ? (i_lo + t) * KB_I8 : (i_lo + 2 * t) * PROWB;
                    sqd::tma_load_2d(stg_a(s), &tm_wn, stg_full(s), x, n0);
                    sqd::tma_load_2d(stg_a(s) + C::A_BYTES, &tm_xn, stg_full(s), x, 0);
                } else {
                    const int x = (o_lo + t - ns_i) * KB_BF;
                    sqd::tma_load_2d(stg_a(s), &tm_wo, stg_full(s), x, n0);
                    sqd::tma_load_2d(stg_a(s) + C::A_BYTES, &tm_xo, stg_full(s), x, 0);
                }
                last_armed = t;
            }
            if (!ok && last_armed >= 0) sqd::mbar_drain(stg_full(last_armed % NST), (last_armed / NST) & 1);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_bf = sqd::make_idesc(false, 128, MP);
            constexpr uint32_t idesc_i8 = sqd::make_idesc(true, 128, MP);
            constexpr uint32_t idesc_f8 = sqd::make_idesc_e4m3(128, MP);
            constexpr uint32_t idesc_mx = sqd::make_idesc_mxf4(128, MP);
            bool ok = true;
            if constexpr (MX) {
                for (int t = 0; t < ns_i && ok; ++t) {  // E2M1 blocks and their scales from the staging ring
                    const int s = t % NST;
                    if (!sqd::mbar_wait(stg_full(s), (t / NST) & 1, abort_flag, SITE_SK_MMA)) { ok = false; break; }
                    sqd::tc_fence_after();
                    const uint32_t sf = sbase + C::OFF_SF + s * C::SF_BYTES;
                    sqd::sf_copy(tmem + MP, sqd::make_sf_desc(sf));                // W rows, K-tile 0
                    sqd::sf_copy(tmem + MP + 4, sqd::make_sf_desc(sf + 512));      // W rows, K-tile 1
                    sqd::sf_copy(tmem + MP + 8, sqd::make_sf_desc(sf + 1024));     // tokens, K-tile 0
                    sqd::sf_copy(tmem + MP + 12, sqd::make_sf_desc(sf + 1536));    // tokens, K-tile 1
                    const uint64_t adesc = sqd::make_sw128_desc(stg_a(s));
                    const uint64_t bdesc = sqd::make_sw128_desc(stg_a(s) + C::A_BYTES);
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const uint32_t id = 2u * static_cast<uint32_t>(k & 1);
                        const uint32_t sfa = (tmem + MP + 4 * (k >> 1)) | (id << 30);
                        const uint32_t sfb = (tmem + MP + 8 + 4 * (k >> 1)) | (id << 30);
                        sqd::mma_mxf4(tmem, adesc + 2 * k, bdesc + 2 * k, idesc_mx | (id << 29) | (id << 4),
                                      (t == 0 && k == 0) ? 0u : 1u, sfa, sfb);
                    }
                    sqd::mma_commit(stg_empty(s));
                }
            }
            if constexpr (FP8) {
                for (int t = 0; t < ns_i && ok; ++t) {  // E4M3 blocks straight from the staging ring
                    const int s = t % NST;
                    if (!sqd::mbar_wait(stg_full(s), (t / NST) & 1, abort_flag, SITE_SK_MMA)) { ok = false; break; }
                    sqd::tc_fence_after();
                    const uint64_t adesc = sqd::make_sw128_desc(stg_a(s));
                    const uint64_t bdesc = sqd::make_sw128_desc(stg_a(s) + C::A_BYTES);
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        sqd::mma_f8(tmem, adesc + 2 * k, bdesc + 2 * k, idesc_f8, (t == 0 && k == 0) ? 0u : 1u);
                    sqd::mma_commit(stg_empty(s));
                }
            }
            for (int u = 0; u < (DIRECT ? 0 : n_i) && ok; ++u) {  // INT4 blocks from the operand ring
                const int e = u % OPR;
                if (!sqd::mbar_wait(op_full(e), (u / OPR) & 1, abort_flag, SITE_SK_MMA)) { ok = false; break; }
                sqd::tc_fence_after();
                const uint64_t bdesc = sqd::make_sw128_desc(op_b(e));
                if constexpr (C::TA) {
                    // A: 32 TMEM columns of slot e, 8 columns (32 int8 K-elements) per MMA
                    const uint32_t at = tmem + static_cast<uint32_t>(C::TA_COL + 32 * e);
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        sqd::mma_s8_ta(tmem, at + 8 * k, bdesc + 2 * k, idesc_i8, (u == 0 && k == 0) ? 0u : 1u);
                } else {
                    const uint64_t adesc = sqd::make_sw128_desc(op_a(e));
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        sqd::mma_s8(tmem, adesc + 2 * k, bdesc + 2 * k, idesc_i8, (u == 0 && k == 0) ? 0u : 1u);
                }
                sqd::mma_commit(op_empty(e));
            }
            for (int t = ns_i; t < ns && ok; ++t) {  // bf16 blocks straight from the staging ring
                const int s = t % NST;
                if (!sqd::mbar_wait(stg_full(s), (t / NST) & 1, abort_flag, SITE_SK_MMA)) { ok = false; break; }
                sqd::tc_fence_after();
                const uint64_t adesc = sqd::make_sw128_desc(stg_a(s));
                const uint64_t bdesc = sqd::make_sw128_desc(stg_a(s) + C::A_BYTES);
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    // MX: the branch adds into the one accumulator (cleared by whichever MMA comes first)
                    const uint32_t acc = MX ? ((t == 0 && k == 0) ? 0u : 1u) : ((t == ns_i && k == 0) ? 0u : 1u);
                    sqd::mma_bf16(tmem + C::COL_F, adesc + 2 * k, bdesc + 2 * k, idesc_bf, acc);
                }
                sqd::mma_commit(stg_empty(s));
            }
            if (ok) {
                sqd::mma_commit(acc_full);  // also when this split has no blocks
            } else {
                sqd::mma_commit(drain);
                sqd::mbar_drain(drain, 0);
            }
        }
    } else {
        // ------------------------------------------------------------ INT4 expansion
        // Thread q of a stage handles 16-byte chunk q & 7 of row q >> 3: chunk
        // c holds packed K-block c >> 2 of the stage, and stored chunk c of
        // row r sits at position c ^ (r & 7) (128-byte swizzle).  Eight
        // threads read one whole row, so the loads are conflict-free.
        const int et = threadIdx.x - SK_PROD_WARP0 * 32;
        bool ok = true;
        for (int t = 0; t < (DIRECT ? 0 : ns_i) && ok; ++t) {
            const int s = t % NST;
            const int nblk = min(2, n_i - 2 * t);
            const int u0 = 2 * t;  // operand ring uses u0, u0 + 1
            if (!sqd::mbar_wait(stg_full(s), (t / NST) & 1, abort_flag, SITE_SK_OP)) { ok = false; break; }
            for (int j = 0; j < nblk; ++j) {
                if (!sqd::mbar_wait(op_empty((u0 + j) % OPR), (((u0 + j) / OPR) & 1) ^ 1u, abort_flag, SITE_SK_OP)) {
                    ok = false;
                    break;
                }
            }
            if (!ok) break;
            const uint32_t src = stg_a(s);
            auto ex = [&](uint32_t v) { return SQF ? clear_mask_code(v) : v; };
            if constexpr (C::TA) {
                // W row of this thread = its TMEM lane (warp quarter): its 128
                // packed bytes (both K-blocks) expanded into one 32-column slot
                // per K-block.  Eight consecutive rows read eight different
                // 16-byte positions (swizzle), so the loads are conflict-free.
                const int quarter = warp & 3;
                const int wr = quarter * 32 + lane;
                const uint32_t srow = src + wr * ROWB;
                const uint32_t tl = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + C::TA_COL;
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    if (j < nblk) {
                        uint4 c4[4];
#pragma unroll
                        for (int q = 0; q < 4; ++q) c4[q] = sqd::lds128(srow + (((4 * j + q) ^ (wr & 7)) << 4));
                        uint32_t v[32];
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            v[8 * q + 0] = ex((c4[q].x << 4) & 0xF0F0F0F0u);
                            v[8 * q + 1] = ex(c4[q].x & 0xF0F0F0F0u);
                            v[8 * q + 2] = ex((c4[q].y << 4) & 0xF0F0F0F0u);
                            v[8 * q + 3] = ex(c4[q].y & 0xF0F0F0F0u);
                            v[8 * q + 4] = ex((c4[q].z << 4) & 0xF0F0F0F0u);
                            v[8 * q + 5] = ex(c4[q].z & 0xF0F0F0F0u);
                            v[8 * q + 6] = ex((c4[q].w << 4) & 0xF0F0F0F0u);
                            v[8 * q + 7] = ex(c4[q].w & 0xF0F0F0F0u);
                        }
                        sqd::tmem_st_32x32b_x32(tl + 32u * static_cast<uint32_t>((u0 + j) % OPR), v);
                    }
                }
                // Token rows (staging rows 128 .. 128 + MP - 1): 16-byte chunk q
                // of the MP x 8 chunks, into the slot's swizzled token tile.
#pragma unroll
                for (int c = 0; c < C::MP * 8 / SK_PT; ++c) {
                    const int q = et + c * SK_PT;
                    const int tr = q >> 3;
                    const int ck = q & 7;
                    const int j = ck >> 2;
                    if (j < nblk) {
                        const uint4 w4 = sqd::lds128(src + (128 + tr) * ROWB + ((ck ^ (tr & 7)) << 4));
                        const uint32_t sw = static_cast<uint32_t>(tr & 7);
                        const uint32_t jj = static_cast<uint32_t>(ck & 3);
                        const uint32_t row = op_b((u0 + j) % OPR) + tr * ROWB;
                        sqd::sts128(row + (((2u * jj) ^ sw) << 4), ex((w4.x << 4) & 0xF0F0F0F0u), ex(w4.x & 0xF0F0F0F0u),
                                    ex((w4.y << 4) & 0xF0F0F0F0u), ex(w4.y & 0xF0F0F0F0u));
                        sqd::sts128(row + (((2u * jj + 1u) ^ sw) << 4), ex((w4.z << 4) & 0xF0F0F0F0u), ex(w4.z & 0xF0F0F0F0u),
                                    ex((w4.w << 4) & 0xF0F0F0F0u), ex(w4.w & 0xF0F0F0F0u));
                    }
                }
                sqd::tmem_wait_st();
                sqd::tc_fence_before();
            } else {
                uint4 w[EC];
#pragma unroll
                for (int c = 0; c < EC; ++c) {
                    const int q = et + c * SK_PT;
                    const int r = q >> 3;
                    w[c] = sqd::lds128(src + r * ROWB + (((q & 7) ^ (r & 7)) << 4));
                }
#pragma unroll
                for (int c = 0; c < EC; ++c) {
                    const int q = et + c * SK_PT;
                    const int r = q >> 3;
                    const int j = (q >> 2) & 1;  // K-block of the stage
                    if (j < nblk) {
                        const uint32_t sw = static_cast<uint32_t>(r & 7);
                        const uint32_t jj = static_cast<uint32_t>(q & 3);
                        const uint32_t row = op_a((u0 + j) % OPR) + r * ROWB;
                        const uint32_t a0 = row + (((2u * jj) ^ sw) << 4);
                        const uint32_t a1 = row + (((2u * jj + 1u) ^ sw) << 4);
                        const uint32_t lo0 = ex((w[c].x << 4) & 0xF0F0F0F0u), hi0 = ex(w[c].x & 0xF0F0F0F0u);
                        const uint32_t lo1 = ex((w[c].y << 4) & 0xF0F0F0F0u), hi1 = ex(w[c].y & 0xF0F0F0F0u);
                        const uint32_t lo2 = ex((w[c].z << 4) & 0xF0F0F0F0u), hi2 = ex(w[c].z & 0xF0F0F0F0u);
                        const uint32_t lo3 = ex((w[c].w << 4) & 0xF0F0F0F0u), hi3 = ex(w[c].w & 0xF0F0F0F0u);
                        // The two K-blocks' threads of a row store in opposite
                        // order, so the eight stores of a phase hit distinct banks.
                        if (j == 0) {
                            sqd::sts128(a0, lo0, hi0, lo1, hi1);
                            sqd::sts128(a1, lo2, hi2, lo3, hi3);
                        } else {
                            sqd::sts128(a1, lo2, hi2, lo3, hi3);
                            sqd::sts128(a0, lo0, hi0, lo1, hi1);
                        }
                    }
                }
            }
            sqd::fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                for (int j = 0; j < nblk; ++j) sqd::mbar_arrive(op_full((u0 + j) % OPR));
                // The stage is released by the last of the four warps to have
                // read it (a running count per slot, never reset).
                if ((atomicAdd(&stg_done[s], 1u) + 1u) % SK_PROD_WARPS == 0u) sqd::mbar_arrive(stg_empty(s));
            }
        }
        if (sqd::mbar_wait(acc_full, 0, abort_flag, SITE_SK_EPI)) sqd::tc_fence_after();
        // The rings are reused by the generic proxy below.
        sqd::fence_proxy_async_smem();
    }

    // ---------------------------------------------------------------- split reduction
    __syncwarp();
    sqd::tc_fence_before();
    sqd::cluster_sync();  // every MMA of every CTA of the cluster is complete: rings are free

    const int RP = (128 + S - 1) / S;
    if (warp >= SK_PROD_WARP0) {
        // Send this CTA's partial rows to their owners.  TMEM lane quarter
        // warp % 4 holds W rows t = 32 * (warp % 4) + lane.
        const int quarter = warp & 3;
        const int t = quarter * 32 + lane;
        const int owner = t / RP;
        const int rl = t - owner * RP;
        const uint32_t tl = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
        const uint32_t off = static_cast<uint32_t>(((rank * RP + rl) * C::RSTRIDE) * 4);
        const uint32_t dst_i = sqd::map_to_cta(sbase + C::OFF_RED_I + off, static_cast<uint32_t>(owner));
        const uint32_t dst_f = sqd::map_to_cta(sbase + C::OFF_RED_F + off, static_cast<uint32_t>(owner));
        // MX: one accumulator in [0, MP), sent as the "fp32" partial.
        const bool has_i = !MX && n_i > 0 && !*abort_flag;
        const bool has_f = (MX ? (n_i + n_o > 0) : n_o > 0) && !*abort_flag;
        const uint32_t col_f = static_cast<uint32_t>(C::COL_F);
#pragma unroll 1
        for (int ch = 0; ch < MP / 16; ++ch) {
            uint32_t vi[16] = {}, vf[16] = {};
            if (has_i) sqd::tmem_ld_32x32b_x16(tl + ch * 16, vi);
            if (has_f) sqd::tmem_ld_32x32b_x16(tl + col_f + ch * 16, vf);
            sqd::tmem_wait_ld_dep(vi, vf);
#pragma unroll
            for (int g = 0; g < 4; ++g) {
                sqd::st_cluster_v4(dst_i + (ch * 16 + 4 * g) * 4, vi[4 * g], vi[4 * g + 1], vi[4 * g + 2], vi[4 * g + 3]);
                sqd::st_cluster_v4(dst_f + (ch * 16 + 4 * g) * 4, vf[4 * g], vf[4 * g + 1], vf[4 * g + 2], vf[4 * g + 3]);
            }
        }
    }
    sqd::tc_fence_before();
    sqd::cluster_sync();  // all partials delivered

    if (warp >= SK_PROD_WARP0) {
        // Owned rows [rank * RP, rank * RP + R): sum the S partials, fuse, store.
        const int et = threadIdx.x - SK_PROD_WARP0 * 32;
        const int r0 = rank * RP;
        const int R = max(0, min(128 - r0, RP));
        const int32_t *red_i = reinterpret_cast<const int32_t *>(smem + C::OFF_RED_I);
        const float *red_f = reinterpret_cast<const float *>(smem + C::OFF_RED_F);
        // Thread et sums row rl = et % R for tokens m = et / R, + G, + 2G, ...
        // (one division per thread; rows of a warp are consecutive, so the Y
        // stores of one token coalesce).
        if (R > 0) {
            const int G = SK_PT / R;
            const int rl = et % R;
            const int mg = et / R;
            const int n = n0 + r0 + rl;
            const int mlim = min(args.M, MP);
            if (mg < G && n < args.N) {
                const float swn = scl_w[r0 + rl];
                const int wb = rl * C::RSTRIDE;
                const int sstep = RP * C::RSTRIDE;
#pragma unroll 4
                for (int m = mg; m < mlim; m += G) {
                    int32_t si = 0;
                    float sl = 0.0f, sf = 0.0f;
#pragma unroll
                    for (int s = 0; s < SK_MAX_SPLITS; ++s) {
                        if (s < S) {
                            const int w = wb + s * sstep + m;
                            if constexpr (FP8) sl = __fadd_rn(sl, __int_as_float(red_i[w]));
                            else si += red_i[w];
                            sf = __fadd_rn(sf, red_f[w]);
                        }
                    }
                    const int ai = si >> 8;
                    const float al = FP8 ? sl : static_cast<float>(ai);
                    const float add = SQF ? args.addend[static_cast<long long>(m) * args.N + n] : sf;
                    const float y = MX ? sf : __fadd_rn(__fmul_rn(__fmul_rn(al, scl_x[m]), swn), add);
                    args.Y[static_cast<long long>(m) * args.ldy + n] = __bfloat16_as_ushort(__float2bfloat16_rn(y));
                    if constexpr (DBG) {
                        if (args.dbg_i) args.dbg_i[static_cast<long long>(m) * args.N + n] = FP8 ? __float_as_int(sl) : ai;
                        if (args.dbg_f) args.dbg_f[static_cast<long long>(m) * args.N + n] = sf;
                    }
                }
            }
        }
    }
    if (warp == 1) {
        sqd::tc_fence_after();
        sqd::tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

}  // namespace sqg
