// Dual-path GEMM with fused epilogue on the sm_100a tensor cores (tcgen05).
//
// OSC (arXiv:2604.12782), abstract: inference runs a low-precision 4-bit GEMM
// path and a high-precision 16-bit branch GEMM on the compact outlier tensor,
// and fuses the two results.  Here both run inside one kernel per 128 x BN
// output tile, each into its own tensor-memory (TMEM) accumulator:
//
//   acc_f (fp32, TMEM columns [0, BN))   += X_O . W_O^T   (tcgen05 kind::f16, bf16 inputs)
//   acc_i (int32, TMEM columns [BN, 2BN)) += codes_X . codes_W^T  (tcgen05 kind::i8)
//   Y = bf16_rn( (float)acc_i * s_x[m] * s_w[n] + acc_f )         (one epilogue)
//
// Warp roles (6 warps):
//   warp 0      TMA producer: compact bf16 tiles straight into the operand
//               ring (128-byte swizzle, consumable by the MMA), packed INT4
//               tiles into a staging ring.
//   warp 1      allocates TMEM; one lane issues every MMA and commits.
//   warps 2..5  expand packed INT4 tiles into int8 operand tiles, then run
//               the epilogue (each warp owns one 32-lane TMEM sub-partition).
//
// INT4 expansion.  A packed 32-bit word holds 8 codes c0..c7 (c0 in the low
// nibble).  (w << 4) & 0xF0F0F0F0 gives the bytes 16*c0, 16*c2, 16*c4, 16*c6
// and w & 0xF0F0F0F0 gives 16*c1, 16*c3, 16*c5, 16*c7 as signed int8 --
// exact, two logic operations, no sign-extension step.  Both operands use the
// same within-8 order, so every product pairs matching channels, and each
// product is 256 * cx * cw.  The integer sum is therefore 256 * acc exactly
// (|256 * acc| <= 256 * 49 * 65536 < 2^31) and the epilogue shifts it right
// by 8.
#pragma once

#include <cuda_bf16.h>

#include "sq_device.cuh"

namespace sqg {

constexpr int BM = 128;         // tile rows (tokens) = TMEM lanes
constexpr int ROWB = 128;       // operand bytes per row per K-block (one 128-byte swizzle row)
constexpr int PROWB = 64;       // packed INT4 bytes per row per K-block
constexpr int KB_I8 = 128;      // int8 K elements per block
constexpr int KB_BF = 64;       // bf16 K elements per block
constexpr int NUM_THREADS = 192;
constexpr int NUM_EXP_WARPS = 4;

enum : unsigned {
    SITE_PROD_OP = 0x101, SITE_PROD_STG = 0x102, SITE_EXP_STG = 0x201, SITE_EXP_OP = 0x202,
    SITE_MMA = 0x301, SITE_EPI = 0x401
};

template <int BN_, int OPS_, int STG_>
struct Cfg {
    static constexpr int BN = BN_, OPS = OPS_, STG = STG_;
    static constexpr int A_BYTES = BM * ROWB;
    static constexpr int B_BYTES = BN * ROWB;
    static constexpr int OP_BYTES = A_BYTES + B_BYTES;
    static constexpr int PA_BYTES = BM * PROWB;
    static constexpr int PB_BYTES = BN * PROWB;
    static constexpr int STG_BYTES = PA_BYTES + PB_BYTES;
    static constexpr int OFF_OP = 0;
    static constexpr int OFF_STG = OPS * OP_BYTES;
    static constexpr int OFF_BAR = OFF_STG + STG * STG_BYTES;
    // barriers: stg_full[STG] stg_empty[STG] opx_full[OPS] opt_full[OPS] op_empty[OPS] acc_full drain
    static constexpr int NBAR = 2 * STG + 3 * OPS + 2;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;  // + slack for 1024-byte alignment
    static constexpr int TMEM_COLS = 2 * BN;
    static_assert(BN == 64 || BN == 128 || BN == 256, "BN");
    static_assert(OP_BYTES % 1024 == 0, "operand tiles must stay 1024-byte aligned");
    static_assert(SMEM_BYTES <= 232448, "shared memory");
};

struct GemmArgs {
    const float *s_x;
    const float *s_w;
    uint16_t *Y;
    int32_t *dbg_i;
    float *dbg_f;
    int M, N;
    long long ldy;
    int nkb_i;    // packed INT4 K-blocks (kn_pad / 128)
    int nkb_o;    // bf16 K-blocks (no_pad / 64)
    int tiles_m, tiles_n, group_m;
};

template <class C, bool DBG>
__global__ void __launch_bounds__(NUM_THREADS, 1)
dual_gemm_kernel(const __grid_constant__ CUtensorMap tm_xn, const __grid_constant__ CUtensorMap tm_wn,
                 const __grid_constant__ CUtensorMap tm_xo, const __grid_constant__ CUtensorMap tm_wo,
                 const GemmArgs args)
{
    constexpr int BN = C::BN, OPS = C::OPS, STG = C::STG;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = sqd::smem_u32(smem);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // Tile coordinates: groups of `group_m` M-tiles sweep all N-tiles so that a
    // wave of CTAs shares a few X tiles and a band of W tiles in L2.
    int tmi, tni;
    {
        const int bid = blockIdx.x;
        const int gsz = args.group_m * args.tiles_n;
        const int g = bid / gsz;
        const int first_m = g * args.group_m;
        const int gm = min(args.tiles_m - first_m, args.group_m);
        const int idx = bid - g * gsz;
        tmi = first_m + idx % gm;
        tni = idx / gm;
    }

    const uint32_t bar0 = sbase + C::OFF_BAR;
    auto stg_full = [&](int s) { return bar0 + 8u * s; };
    auto stg_empty = [&](int s) { return bar0 + 8u * (STG + s); };
    auto opx_full = [&](int e) { return bar0 + 8u * (2 * STG + e); };
    auto opt_full = [&](int e) { return bar0 + 8u * (2 * STG + OPS + e); };
    auto op_empty = [&](int e) { return bar0 + 8u * (2 * STG + 2 * OPS + e); };
    const uint32_t acc_full = bar0 + 8u * (2 * STG + 3 * OPS);
    const uint32_t drain = acc_full + 8u;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::OFF_MISC);
    volatile uint32_t *abort_flag = reinterpret_cast<volatile uint32_t *>(smem + C::OFF_MISC + 4);
    auto op_a = [&](int e) { return sbase + C::OFF_OP + e * C::OP_BYTES; };
    auto stg_a = [&](int s) { return sbase + C::OFF_STG + s * C::STG_BYTES; };

    if (threadIdx.x == 0) {
        for (int s = 0; s < STG; ++s) {
            sqd::mbar_init(stg_full(s), 1);
            sqd::mbar_init(stg_empty(s), NUM_EXP_WARPS);
        }
        for (int e = 0; e < OPS; ++e) {
            sqd::mbar_init(opx_full(e), NUM_EXP_WARPS);
            sqd::mbar_init(opt_full(e), 1);
            sqd::mbar_init(op_empty(e), 1);
        }
        sqd::mbar_init(acc_full, 1);
        sqd::mbar_init(drain, 1);
        *abort_flag = 0u;
        sqd::fence_barrier_init();
        sqd::fence_proxy_async_smem();
    }
    if (warp == 0 && lane == 0) {
        if (args.nkb_i > 0) { sqd::prefetch_tensormap(&tm_xn); sqd::prefetch_tensormap(&tm_wn); }
        if (args.nkb_o > 0) { sqd::prefetch_tensormap(&tm_xo); sqd::prefetch_tensormap(&tm_wo); }
    }
    if (warp == 1) {
        sqd::tmem_alloc(sqd::smem_u32(tmem_slot), C::TMEM_COLS);
        sqd::tmem_relinquish();
    }
    sqd::tc_fence_before();
    __syncthreads();
    sqd::tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    const int nkb_i = args.nkb_i, nkb_o = args.nkb_o;
    const int ntot = nkb_o + nkb_i;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            int i = 0;
            int armed_o = 0, armed_s = 0;
            bool ok = true;
            for (int kb = 0; kb < nkb_o && ok; ++kb, ++i) {
                const int e = i % OPS;
                const uint32_t ph = (i / OPS) & 1;
                if (!sqd::mbar_wait(op_empty(e), ph ^ 1u, abort_flag, SITE_PROD_OP)) { ok = false; break; }
                sqd::mbar_arrive_expect_tx(opt_full(e), C::OP_BYTES);
                sqd::tma_load_2d(op_a(e), &tm_xo, opt_full(e), kb * KB_BF, tmi * BM);
                sqd::tma_load_2d(op_a(e) + C::A_BYTES, &tm_wo, opt_full(e), kb * KB_BF, tni * BN);
                armed_o = kb + 1;
            }
            for (int kb = 0; kb < nkb_i && ok; ++kb) {
                const int s = kb % STG;
                const uint32_t ph = (kb / STG) & 1;
                if (!sqd::mbar_wait(stg_empty(s), ph ^ 1u, abort_flag, SITE_PROD_STG)) { ok = false; break; }
                sqd::mbar_arrive_expect_tx(stg_full(s), C::STG_BYTES);
                sqd::tma_load_2d(stg_a(s), &tm_xn, stg_full(s), kb * PROWB, tmi * BM);
                sqd::tma_load_2d(stg_a(s) + C::PA_BYTES, &tm_wn, stg_full(s), kb * PROWB, tni * BN);
                armed_s = kb + 1;
            }
            if (!ok) {
                // Let every copy that was issued land before the CTA exits.
                for (int kb = (armed_o > OPS ? armed_o - OPS : 0); kb < armed_o; ++kb)
                    sqd::mbar_drain(opt_full(kb % OPS), (kb / OPS) & 1);
                for (int kb = (armed_s > STG ? armed_s - STG : 0); kb < armed_s; ++kb)
                    sqd::mbar_drain(stg_full(kb % STG), (kb / STG) & 1);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_bf = sqd::make_idesc(false, BM, BN);
            constexpr uint32_t idesc_i8 = sqd::make_idesc(true, BM, BN);
            bool ok = true;
            for (int i = 0; i < ntot; ++i) {
                const int e = i % OPS;
                const bool is_bf = i < nkb_o;
                // opt_full(e) completes once per bf16 use of slot e and
                // opx_full(e) once per INT4 use, so each has its own phase.
                const uint32_t ph = is_bf ? ((i / OPS) & 1) : (((i - nkb_o) / OPS) & 1);
                if (!sqd::mbar_wait(is_bf ? opt_full(e) : opx_full(e), ph, abort_flag, SITE_MMA)) { ok = false; break; }
                sqd::tc_fence_after();
                const uint64_t adesc = sqd::make_sw128_desc(op_a(e));
                const uint64_t bdesc = sqd::make_sw128_desc(op_a(e) + C::A_BYTES);
                const uint32_t d = tmem + (is_bf ? 0u : static_cast<uint32_t>(BN));
                const bool first = is_bf ? (i == 0) : (i == nkb_o);
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    // each step advances 32 bytes along K inside the swizzle row
                    const uint32_t acc = (first && k == 0) ? 0u : 1u;
                    if (is_bf) sqd::mma_bf16(d, adesc + 2 * k, bdesc + 2 * k, idesc_bf, acc);
                    else sqd::mma_s8(d, adesc + 2 * k, bdesc + 2 * k, idesc_i8, acc);
                }
                sqd::mma_commit(op_empty(e));
            }
            if (ok) {
                sqd::mma_commit(acc_full);
            } else {
                sqd::mma_commit(drain);
                sqd::mbar_drain(drain, 0);
            }
        }
    } else {
        // ------------------------------------------------------------ expansion
        const int et = threadIdx.x - 64;  // 0..127
        constexpr int ROWS = BM + BN;
        for (int kb = 0; kb < nkb_i; ++kb) {
            const int s = kb % STG;
            const uint32_t sph = (kb / STG) & 1;
            const int i = nkb_o + kb;
            const int e = i % OPS;
            const uint32_t eph = (i / OPS) & 1;
            if (!sqd::mbar_wait(stg_full(s), sph, abort_flag, SITE_EXP_STG)) break;
            if (!sqd::mbar_wait(op_empty(e), eph ^ 1u, abort_flag, SITE_EXP_OP)) break;
            const uint32_t src = stg_a(s);
            const uint32_t dst = op_a(e);
            for (int q = et; q < ROWS * 4; q += NUM_EXP_WARPS * 32) {
                const int r = q >> 2;
                const int j = q & 3;
                const uint4 w = sqd::lds128(src + r * PROWB + j * 16);
                const uint32_t sw = static_cast<uint32_t>(r & 7);
                const uint32_t row = dst + r * ROWB;
                sqd::sts128(row + (((2u * j) ^ sw) << 4),
                            (w.x << 4) & 0xF0F0F0F0u, w.x & 0xF0F0F0F0u,
                            (w.y << 4) & 0xF0F0F0F0u, w.y & 0xF0F0F0F0u);
                sqd::sts128(row + (((2u * j + 1u) ^ sw) << 4),
                            (w.z << 4) & 0xF0F0F0F0u, w.z & 0xF0F0F0F0u,
                            (w.w << 4) & 0xF0F0F0F0u, w.w & 0xF0F0F0F0u);
            }
            sqd::fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                sqd::mbar_arrive(stg_empty(s));
                sqd::mbar_arrive(opx_full(e));
            }
        }

        // ------------------------------------------------------------ epilogue
        if (sqd::mbar_wait(acc_full, 0, abort_flag, SITE_EPI)) {
            sqd::tc_fence_after();
            const int sub = warp & 3;                 // TMEM lane sub-partition of this warp
            const int m = tmi * BM + sub * 32 + lane;
            const bool row_ok = m < args.M;
            const float sx = row_ok ? args.s_x[m] : 0.0f;
            const uint32_t tl = tmem + (static_cast<uint32_t>(sub * 32) << 16);
            const bool has_i = nkb_i > 0, has_o = nkb_o > 0;
#pragma unroll 1
            for (int c = 0; c < BN; c += 32) {
                uint32_t vi[32], vf[32];
                if (has_i) sqd::tmem_ld_32x32b_x32(tl + BN + c, vi);
                if (has_o) sqd::tmem_ld_32x32b_x32(tl + c, vf);
                sqd::tmem_wait_ld();
                const int n0 = tni * BN + c;
                if (!row_ok || n0 >= args.N) continue;
                uint16_t *yrow = args.Y + static_cast<long long>(m) * args.ldy;
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    const int n = n0 + 8 * g;
                    if (n >= args.N) break;
                    const float4 sw0 = __ldg(reinterpret_cast<const float4 *>(args.s_w + n));
                    const float4 sw1 = __ldg(reinterpret_cast<const float4 *>(args.s_w + n + 4));
                    const float swv[8] = {sw0.x, sw0.y, sw0.z, sw0.w, sw1.x, sw1.y, sw1.z, sw1.w};
                    uint32_t out[4];
#pragma unroll
                    for (int h = 0; h < 4; ++h) {
                        float y2[2];
#pragma unroll
                        for (int u = 0; u < 2; ++u) {
                            const int t = 8 * g + 2 * h + u;
                            const int ai = has_i ? (static_cast<int>(vi[t]) >> 8) : 0;
                            const float af = has_o ? __uint_as_float(vf[t]) : 0.0f;
                            y2[u] = __fadd_rn(__fmul_rn(__fmul_rn(static_cast<float>(ai), sx), swv[2 * h + u]), af);
                            if constexpr (DBG) {
                                if (args.dbg_i) args.dbg_i[static_cast<long long>(m) * args.N + n + 2 * h + u] = ai;
                                if (args.dbg_f) args.dbg_f[static_cast<long long>(m) * args.N + n + 2 * h + u] = af;
                            }
                        }
                        const __nv_bfloat162 b2 = __floats2bfloat162_rn(y2[0], y2[1]);
                        out[h] = *reinterpret_cast<const uint32_t *>(&b2);
                    }
                    *reinterpret_cast<uint4 *>(yrow + n) = make_uint4(out[0], out[1], out[2], out[3]);
                }
            }
        }
    }

    sqd::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        sqd::tc_fence_after();
        sqd::tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

}  // namespace sqg
