// Dual-path GEMM with fused epilogue on the sm_100a tensor cores (tcgen05).
//
// OSC (arXiv:2604.12782), abstract: inference runs a low-precision 4-bit GEMM
// path and a high-precision 16-bit branch GEMM on the compact outlier tensor,
// and fuses the two results.  Here both run inside one persistent kernel; each
// 128 x BN output tile owns two tensor-memory (TMEM) accumulators:
//
//   acc_f (fp32, TMEM columns [0, BN))    += X_O . W_O^T          (tcgen05 kind::f16, bf16 inputs)
//   acc_i (int32, TMEM columns [BN, 2BN)) += codes_X . codes_W^T  (tcgen05 kind::i8)
//   Y = bf16_rn( (float)acc_i * s_x[m] * s_w[n] + acc_f )           (one epilogue)
//
// Warp roles (14 warps, one CTA per SM, tiles handed out round-robin):
//   warp 0      idle after set-up.
//   warp 1      allocates TMEM; one lane issues every MMA and commits.
//   warps 2..5  epilogue: tcgen05.ld of both accumulators (each warp owns one
//               32-lane TMEM sub-partition), scale, fuse, bf16 stores.  They
//               hand TMEM back as soon as the last column block is read.
//   warps 6..13 operand producers, in the MMA's order of ring uses: for a
//               bf16 block one lane issues the two TMA tile loads (128-byte
//               swizzle, consumable by the MMA as they land); for an INT4
//               block every thread stores its share of the expanded int8
//               tile.  Packed INT4 rows come from global memory straight into
//               registers, two INT4 blocks ahead, so packed bytes never pass
//               through shared memory.  A single producer group keeps every
//               ring slot's uses strictly in order, which the mbarrier phase
//               parity protocol needs.
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
constexpr int NUM_EPI_WARPS = 4;
constexpr int NUM_EXP_WARPS = 8;
constexpr int EPI_WARP0 = 2;
constexpr int EXP_WARP0 = EPI_WARP0 + NUM_EPI_WARPS;
constexpr int NUM_THREADS = 32 * (EXP_WARP0 + NUM_EXP_WARPS);
constexpr int EXP_THREADS = 32 * NUM_EXP_WARPS;

enum : unsigned {
    SITE_EXP_OP = 0x202, SITE_MMA_FULL = 0x301, SITE_MMA_ACC = 0x302, SITE_EPI = 0x401
};

template <int BN_, int OPS_>
struct Cfg {
    static constexpr int BN = BN_, OPS = OPS_;
    static constexpr int A_BYTES = BM * ROWB;
    static constexpr int B_BYTES = BN * ROWB;
    static constexpr int OP_BYTES = A_BYTES + B_BYTES;
    static constexpr int OFF_OP = 0;
    static constexpr int OFF_BAR = OPS * OP_BYTES;
    // barriers: op_full[OPS] op_empty[OPS] acc_full acc_empty drain
    static constexpr int NBAR = 2 * OPS + 3;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;  // + slack for 1024-byte alignment
    static constexpr int TMEM_COLS = 2 * BN;
    // packed 16-byte chunks per K-block and per expansion thread
    static constexpr int EXP_CHUNKS = (BM + BN) * (PROWB / 16) / EXP_THREADS;
    static_assert(BN == 64 || BN == 128 || BN == 256, "BN");
    static_assert(OP_BYTES % 1024 == 0, "operand tiles must stay 1024-byte aligned");
    static_assert(SMEM_BYTES <= 232448, "shared memory");
    static_assert((BM + BN) * (PROWB / 16) % EXP_THREADS == 0, "expansion work split");
};

struct GemmArgs {
    const uint8_t *xn;   // packed X part [M, row_bytes]
    const uint8_t *wn;   // packed W part [N, row_bytes]
    long long row_bytes; // kn_pad / 2
    const float *s_x;
    const float *s_w;
    uint16_t *Y;
    int32_t *dbg_i;
    float *dbg_f;
    int M, N;
    long long ldy;
    int nkb_i;    // INT4 K-blocks per tile (kn_pad / 128)
    int nkb_o;    // bf16 K-blocks per tile (no_pad / 64)
    int tiles_m, tiles_n, group_m;
};

// Tile t -> (M-tile, N-tile): groups of `group_m` M-tiles sweep all N-tiles,
// so the CTAs working at the same time share a few X tiles and a band of W
// tiles in L2.
__device__ __forceinline__ void tile_coords(const GemmArgs &a, int t, int &tmi, int &tni)
{
    const int gsz = a.group_m * a.tiles_n;
    const int g = t / gsz;
    const int first_m = g * a.group_m;
    const int gm = min(a.tiles_m - first_m, a.group_m);
    const int idx = t - g * gsz;
    tmi = first_m + idx % gm;
    tni = idx / gm;
}

template <class C, bool DBG>
__global__ void __launch_bounds__(NUM_THREADS, 1)
dual_gemm_kernel(const __grid_constant__ CUtensorMap tm_xo, const __grid_constant__ CUtensorMap tm_wo,
                 const GemmArgs args)
{
    constexpr int BN = C::BN, OPS = C::OPS, EC = C::EXP_CHUNKS;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = sqd::smem_u32(smem);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    const uint32_t bar0 = sbase + C::OFF_BAR;
    auto op_full = [&](int e) { return bar0 + 8u * e; };
    auto op_empty = [&](int e) { return bar0 + 8u * (OPS + e); };
    const uint32_t acc_full = bar0 + 8u * (2 * OPS);
    const uint32_t acc_empty = acc_full + 8u;
    const uint32_t drain = acc_full + 16u;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::OFF_MISC);
    volatile uint32_t *abort_flag = reinterpret_cast<volatile uint32_t *>(smem + C::OFF_MISC + 4);
    auto op_a = [&](int e) { return sbase + C::OFF_OP + e * C::OP_BYTES; };

    if (threadIdx.x == 0) {
        for (int e = 0; e < OPS; ++e) {
            // One arrival per producer warp; for bf16 blocks the first
            // producer's arrival also carries the TMA byte count.
            sqd::mbar_init(op_full(e), NUM_EXP_WARPS);
            sqd::mbar_init(op_empty(e), 1);
        }
        sqd::mbar_init(acc_full, 1);
        sqd::mbar_init(acc_empty, NUM_EPI_WARPS);
        sqd::mbar_init(drain, 1);
        *abort_flag = 0u;
        sqd::fence_barrier_init();
        sqd::fence_proxy_async_smem();
    }
    if (warp == EXP_WARP0 && lane == 0 && args.nkb_o > 0) {
        sqd::prefetch_tensormap(&tm_xo);
        sqd::prefetch_tensormap(&tm_wo);
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
    const int per_tile = nkb_o + nkb_i;
    const int num_tiles = args.tiles_m * args.tiles_n;
    const int my_tiles = (num_tiles - static_cast<int>(blockIdx.x) + static_cast<int>(gridDim.x) - 1) /
                         static_cast<int>(gridDim.x);

    if (warp == 0) {
        // idle
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_bf = sqd::make_idesc(false, BM, BN);
            constexpr uint32_t idesc_i8 = sqd::make_idesc(true, BM, BN);
            bool ok = true;
            for (int lt = 0; lt < my_tiles && ok; ++lt) {
                // the epilogue must have read the previous tile's accumulators
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
                    const uint32_t d = tmem + (is_bf ? 0u : static_cast<uint32_t>(BN));
                    const bool first = (i == 0) || (i == nkb_o);
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        // each step advances 32 bytes along K inside the swizzle row
                        const uint32_t acc = (first && k == 0) ? 0u : 1u;
                        if (is_bf) sqd::mma_bf16(d, adesc + 2 * k, bdesc + 2 * k, idesc_bf, acc);
                        else sqd::mma_s8(d, adesc + 2 * k, bdesc + 2 * k, idesc_i8, acc);
                    }
                    sqd::mma_commit(op_empty(e));
                }
                if (ok) sqd::mma_commit(acc_full);
            }
            if (!ok) {
                sqd::mma_commit(drain);
                sqd::mbar_drain(drain, 0);
            }
        }
    } else if (warp >= EXP_WARP0) {
        // ------------------------------------------------------------ expansion
        const int et = threadIdx.x - EXP_WARP0 * 32;
        const int F = my_tiles * nkb_i;  // INT4 K-blocks this CTA expands, over all its tiles
        const long long rb = args.row_bytes;

        auto load = [&](int f, uint4 (&buf)[EC]) {
            const int lt = f / nkb_i;
            const int kb = f - lt * nkb_i;
            int tmi, tni;
            tile_coords(args, static_cast<int>(blockIdx.x) + lt * static_cast<int>(gridDim.x), tmi, tni);
#pragma unroll
            for (int c = 0; c < EC; ++c) {
                const int q = et + c * EXP_THREADS;
                const int r = q >> 2;
                const int j = q & 3;
                const uint8_t *p;
                bool ok;
                if (r < BM) {
                    const int row = tmi * BM + r;
                    ok = row < args.M;
                    p = args.xn + static_cast<long long>(row) * rb;
                } else {
                    const int row = tni * BN + (r - BM);
                    ok = row < args.N;
                    p = args.wn + static_cast<long long>(row) * rb;
                }
                buf[c] = ok ? sqd::ld_nc_v4(p + kb * PROWB + j * 16) : make_uint4(0, 0, 0, 0);
            }
        };
        auto store = [&](int f, const uint4 (&buf)[EC]) -> bool {
            const int lt = f / nkb_i;
            const int kb = f - lt * nkb_i;
            const int u = lt * per_tile + nkb_o + kb;
            const int e = u % OPS;
            if (!sqd::mbar_wait(op_empty(e), ((u / OPS) & 1) ^ 1u, abort_flag, SITE_EXP_OP)) return false;
            const uint32_t dst = op_a(e);
#pragma unroll
            for (int c = 0; c < EC; ++c) {
                const int q = et + c * EXP_THREADS;
                const int r = q >> 2;
                const uint32_t j = static_cast<uint32_t>(q & 3);
                const uint32_t sw = static_cast<uint32_t>(r & 7);
                const uint32_t row = dst + r * ROWB;
                const uint4 w = buf[c];
                sqd::sts128(row + (((2u * j) ^ sw) << 4),
                            (w.x << 4) & 0xF0F0F0F0u, w.x & 0xF0F0F0F0u,
                            (w.y << 4) & 0xF0F0F0F0u, w.y & 0xF0F0F0F0u);
                sqd::sts128(row + (((2u * j + 1u) ^ sw) << 4),
                            (w.z << 4) & 0xF0F0F0F0u, w.z & 0xF0F0F0F0u,
                            (w.w << 4) & 0xF0F0F0F0u, w.w & 0xF0F0F0F0u);
            }
            sqd::fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) sqd::mbar_arrive(op_full(e));
            return true;
        };

        // bf16 blocks of tile lt: the first producer thread issues the TMA
        // loads with the expected byte count; every other warp adds one plain
        // arrival (op_full counts one arrival per producer warp).
        const bool tma_thread = (et == 0);
        int last_armed = -1;
        auto produce_bf16 = [&](int lt) -> bool {
            int tmi, tni;
            tile_coords(args, static_cast<int>(blockIdx.x) + lt * static_cast<int>(gridDim.x), tmi, tni);
            for (int kb = 0; kb < nkb_o; ++kb) {
                const int u = lt * per_tile + kb;
                const int e = u % OPS;
                if (!sqd::mbar_wait(op_empty(e), ((u / OPS) & 1) ^ 1u, abort_flag, SITE_EXP_OP)) return false;
                if (tma_thread) {
                    sqd::mbar_arrive_expect_tx(op_full(e), C::OP_BYTES);
                    sqd::tma_load_2d(op_a(e), &tm_xo, op_full(e), kb * KB_BF, tmi * BM);
                    sqd::tma_load_2d(op_a(e) + C::A_BYTES, &tm_wo, op_full(e), kb * KB_BF, tni * BN);
                    last_armed = u;
                } else if (lane == 0) {
                    sqd::mbar_arrive(op_full(e));
                }
            }
            return true;
        };

        bool ok = true;
        if (nkb_i == 0) {
            for (int lt = 0; lt < my_tiles && ok; ++lt) ok = produce_bf16(lt);
        } else {
            // INT4 block f starts tile f / nkb_i when f % nkb_i == 0: its bf16
            // blocks come first in the ring.
            auto step = [&](int f, const uint4 (&buf)[EC]) -> bool {
                if (nkb_o > 0 && f % nkb_i == 0 && !produce_bf16(f / nkb_i)) return false;
                return store(f, buf);
            };
            uint4 b0[EC], b1[EC], b2[EC];
            if (F > 0) load(0, b0);
            if (F > 1) load(1, b1);
            for (int f = 0; f < F; f += 3) {
                if (f + 2 < F) load(f + 2, b2);
                if (!(ok = step(f, b0))) break;
                if (f + 1 >= F) break;
                if (f + 3 < F) load(f + 3, b0);
                if (!(ok = step(f + 1, b1))) break;
                if (f + 2 >= F) break;
                if (f + 4 < F) load(f + 4, b1);
                if (!(ok = step(f + 2, b2))) break;
            }
        }
        if (!ok && tma_thread && last_armed >= 0) {
            // Let the last copies that were issued land before the CTA exits.
            sqd::mbar_drain(op_full(last_armed % OPS), (last_armed / OPS) & 1);
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int sub = warp & 3;  // TMEM lane sub-partition of this warp
        const uint32_t tl = tmem + (static_cast<uint32_t>(sub * 32) << 16);
        const bool has_i = nkb_i > 0, has_o = nkb_o > 0;
        for (int lt = 0; lt < my_tiles; ++lt) {
            int tmi, tni;
            tile_coords(args, static_cast<int>(blockIdx.x) + lt * static_cast<int>(gridDim.x), tmi, tni);
            if (!sqd::mbar_wait(acc_full, lt & 1, abort_flag, SITE_EPI)) break;
            sqd::tc_fence_after();
            const int m = tmi * BM + sub * 32 + lane;
            const bool row_ok = m < args.M;
            const float sx = row_ok ? args.s_x[m] : 0.0f;
            uint16_t *yrow = args.Y + static_cast<long long>(row_ok ? m : 0) * args.ldy;
#pragma unroll 1
            for (int c = 0; c < BN; c += 32) {
                uint32_t vi[32], vf[32];
                if (has_i) sqd::tmem_ld_32x32b_x32(tl + BN + c, vi);
                if (has_o) sqd::tmem_ld_32x32b_x32(tl + c, vf);
                sqd::tmem_wait_ld();
                if (c + 32 == BN) {
                    // Accumulators fully read: the next tile's MMAs may start.
                    sqd::tc_fence_before();
                    __syncwarp();
                    if (lane == 0) sqd::mbar_arrive(acc_empty);
                }
                const int n0 = tni * BN + c;
                if (!row_ok || n0 >= args.N) continue;
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
