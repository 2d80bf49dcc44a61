// Element-level SQ-format weights on the sparse tensor cores.
//
// SQ-format (arXiv:2512.05409): the abstract (a sparse matrix is accelerated
// in high precision while the dense low-precision product is accelerated as
// usual); write-up section 3 (the low-precision part keeps its format with a
// mask value at the positions handled in high precision by a gather of
// sparse data), section 7 (banks with a fixed sparsity pattern), section 9
// (the unused top code of symmetric quantization is the mask; the top (1-s)
// of every bank by importance is high precision), section 8 (FP8/FP4).
//
// Format of a weight row (K channels, banks of `bank` = 4, 8 or 16 channels,
// `h` = 1 or 2 high entries per bank -- sparsity 50 % to 93.75 %):
//   - high set: per bank the h entries of largest |w|, ties to the lower index;
//   - low part W_N: packed INT4 (byte j = code 2j | code 2j+1 << 4), symmetric
//     codes clamp(rint(w / s_lo), -7, 7) with s_lo = (absmax over the low
//     entries) / 7, and the mask code -8 at every high position;
//   - high part: E4M3 codes of w / s_hi, s_hi = (absmax over the high
//     entries) / 448, stored 2:4-compressed: W_H [N, K/2] bytes, two per
//     aligned group of 4 channels (the group's high codes in channel order,
//     zero in free slots), and W_E [N, K/8] metadata bytes, group i in byte
//     i/2 (low nibble for even i), bits [1:0] / [3:2] = in-group index of the
//     first / second stored value (first < second; one high entry at p uses
//     (p, p+1), or (2, 3) with the zero first when p = 3; none uses (0, 1)).
// With h <= 2 per bank and banks of 4, 8 or 16, no aligned group of 4 holds
// more than two high entries, so the high part is exactly a 2:4 sparse matrix
// for tcgen05.mma.sp (kind::f8f6f4).  The metadata layout was confirmed on the
// device: a row-major [128 rows x 16 bytes] tile per 128 channels lands in
// TMEM lanes 0..127, 4 columns, by tcgen05.cp.128x128b, and an MMA of 64
// channels reads 2 of those columns.
#pragma once

#include <cuda_fp8.h>

#include "sq_gemm_common.cuh"

namespace sqf {

constexpr int kPrepThreads = 256;        // 8 warps, one weight row per warp at a time
constexpr int kChunk = 16;               // channels per lane per step (covers a bank of 16)

__device__ __forceinline__ float bf16f(uint32_t b) { return __uint_as_float(b << 16); }

// High mask (bit i = channel i is high) of 16 consecutive channels, banks of
// `bank` channels, h per bank, by rank: entry i is high when fewer than h
// entries of its bank are larger, or equal with a lower index.
__device__ __forceinline__ uint32_t chunk_high_mask(const float (&a)[kChunk], int bank, int h)
{
    uint32_t mask = 0;
#pragma unroll
    for (int i = 0; i < kChunk; ++i) {
        const int g0 = (i / bank) * bank;
        int rank = 0;
#pragma unroll
        for (int j = 0; j < kChunk; ++j) {
            const bool same_bank = j >= g0 && j < g0 + bank;
            rank += (same_bank && (a[j] > a[i] || (a[j] == a[i] && j < i))) ? 1 : 0;
        }
        mask |= (rank < h ? 1u : 0u) << i;
    }
    return mask;
}

__device__ __forceinline__ float warp_max(float v)
{
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, off));
    return v;
}

__device__ __forceinline__ uint32_t e4m3_of(float t)
{
    return static_cast<uint32_t>(__nv_cvt_float_to_fp8(t, __NV_SATFINITE, __NV_E4M3));
}

// Offline weight preparation: one warp per row (rows strided over the grid);
// each lane takes 16 consecutive channels per step.  Pass 1 finds the row's
// low and high absolute maxima, pass 2 writes the codes.  K % 16 == 0.
__global__ void __launch_bounds__(kPrepThreads) sqf_prep_kernel(const uint16_t *__restrict__ W, int N, int K,
                                                                 int64_t ldw, int bank, int h,
                                                                 uint8_t *__restrict__ W_N, float *__restrict__ s_lo,
                                                                 uint8_t *__restrict__ W_H, uint8_t *__restrict__ W_E,
                                                                 float *__restrict__ s_hi)
{
    const int lane = threadIdx.x & 31;
    const int warps = kPrepThreads / 32;
    const int nchunk = K / kChunk;
    for (int row = blockIdx.x * warps + (threadIdx.x >> 5); row < N; row += gridDim.x * warps) {
        const uint16_t *wr = W + static_cast<int64_t>(row) * ldw;
        auto load = [&](int c, float (&v)[kChunk]) {
            const uint4 p0 = *reinterpret_cast<const uint4 *>(wr + kChunk * c);
            const uint4 p1 = *reinterpret_cast<const uint4 *>(wr + kChunk * c + 8);
            const uint32_t w[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                v[2 * i] = bf16f(w[i] & 0xFFFFu);
                v[2 * i + 1] = bf16f(w[i] >> 16);
            }
        };
        // pass 1: maxima of the low and the high entries
        float amax_lo = 0.0f, amax_hi = 0.0f;
        for (int c = lane; c < nchunk; c += 32) {
            float v[kChunk], a[kChunk];
            load(c, v);
#pragma unroll
            for (int i = 0; i < kChunk; ++i) a[i] = fabsf(v[i]);
            const uint32_t hm = chunk_high_mask(a, bank, h);
#pragma unroll
            for (int i = 0; i < kChunk; ++i) {
                if ((hm >> i) & 1u) amax_hi = fmaxf(amax_hi, a[i]);
                else amax_lo = fmaxf(amax_lo, a[i]);
            }
        }
        amax_lo = warp_max(amax_lo);
        amax_hi = warp_max(amax_hi);
        const float sl = amax_lo == 0.0f ? 0.0f : __fdiv_rn(amax_lo, 7.0f);
        const float sh = amax_hi == 0.0f ? 0.0f : __fdiv_rn(amax_hi, 448.0f);
        if (lane == 0) {
            s_lo[row] = sl;
            s_hi[row] = sh;
        }
        // pass 2: codes, 2:4 values and metadata
        for (int c = lane; c < nchunk; c += 32) {
            float v[kChunk], a[kChunk];
            load(c, v);
#pragma unroll
            for (int i = 0; i < kChunk; ++i) a[i] = fabsf(v[i]);
            const uint32_t hm = chunk_high_mask(a, bank, h);
            uint32_t lo_w[2] = {0u, 0u};   // 16 nibbles
            uint32_t hv[2] = {0u, 0u};     // 8 value bytes (4 groups x 2)
            uint32_t meta = 0u;            // 4 nibbles
#pragma unroll
            for (int i = 0; i < kChunk; ++i) {
                uint32_t q;
                if ((hm >> i) & 1u) {
                    q = 8u;   // mask code -8
                } else if (amax_lo == 0.0f) {
                    q = 0u;
                } else {
                    const float t = rintf(__fdiv_rn(v[i], sl));
                    q = static_cast<uint32_t>(static_cast<int>(fminf(fmaxf(t, -7.0f), 7.0f))) & 15u;
                }
                lo_w[i >> 3] |= q << (4 * (i & 7));
            }
#pragma unroll
            for (int g = 0; g < kChunk / 4; ++g) {
                const uint32_t gm = (hm >> (4 * g)) & 15u;
                uint32_t i0, i1, c0 = 0u, c1 = 0u;
                const int n = __popc(gm);
                if (n == 2) {
                    i0 = __ffs(gm) - 1;
                    i1 = 31 - __clz(gm);
                } else if (n == 1) {
                    const uint32_t p = __ffs(gm) - 1;
                    i0 = p < 3 ? p : 2u;
                    i1 = p < 3 ? p + 1 : 3u;
                } else {
                    i0 = 0u;
                    i1 = 1u;
                }
                if (amax_hi != 0.0f) {
                    if ((gm >> i0) & 1u) c0 = e4m3_of(__fdiv_rn(v[4 * g + i0], sh));
                    if ((gm >> i1) & 1u) c1 = e4m3_of(__fdiv_rn(v[4 * g + i1], sh));
                }
                hv[g >> 1] |= (c0 | (c1 << 8)) << (16 * (g & 1));
                meta |= (i0 | (i1 << 2)) << (4 * g);
            }
            const int64_t rb = static_cast<int64_t>(row) * (K / 2) + 8 * c;
            *reinterpret_cast<uint2 *>(W_N + rb) = make_uint2(lo_w[0], lo_w[1]);
            *reinterpret_cast<uint2 *>(W_H + rb) = make_uint2(hv[0], hv[1]);
            *reinterpret_cast<uint16_t *>(W_E + static_cast<int64_t>(row) * (K / 8) + 2 * c) =
                static_cast<uint16_t>(meta);
        }
    }
}

// ---------------------------------------------------------------- high part
// P[m, n] = s_x8[m] * s_hi[n] * sum over the 2:4 structure of e(X)[m, k] e(W)[n, k]
// Swapped operands: the 128 W rows of a tile are the MMA's A side (the
// sparse operand), MT tokens its N side.  A stage holds 256 channels: the
// compressed W tile (128 bytes per row), two 128-channel boxes of E4M3
// tokens and two 16-byte metadata boxes.  TMEM: accumulator in [0, MT), the
// stage's metadata in [MT, MT + 8).
constexpr int kHiWarps = 6;                 // 0 TMA, 1 MMA, 2..5 epilogue
constexpr int kHiThreads = 32 * kHiWarps;
enum : unsigned { SITE_HI_STG = 0x601, SITE_HI_MMA = 0x602, SITE_HI_EPI = 0x603 };

// KS = 2: the K stages of a tile are split over a cluster of two CTAs; the
// second adds its fp32 accumulator into the first's through distributed shared
// memory (one fixed order, so P is deterministic).  Used when one CTA per tile
// would leave more than half of the SMs idle.
template <int MT_, int NST_, int KS_ = 1>
struct CfgHigh {
    static constexpr int MT = MT_;
    static constexpr int NST = NST_;
    static constexpr int KS = KS_;
    static_assert(KS == 1 || KS == 2, "K split");
    static constexpr int A_BYTES = 128 * 128;
    static constexpr int B_BYTES = MT * 128;          // one 128-channel box of tokens
    static constexpr int E_BYTES = 128 * 16;          // one 128-channel metadata box
    static constexpr int STAGE = A_BYTES + 2 * B_BYTES + 2 * E_BYTES;
    static constexpr int OFF_BAR = NST * STAGE;
    static constexpr int SMEM_BYTES = OFF_BAR + (2 * NST + 2) * 8 + 16 + 1024;
    // MT accumulator columns, then 8 metadata columns per stage (a stage's copy never waits
    // for the MMAs of the one before it)
    static constexpr int TMEM_USED = MT + 8 * NST;
    static constexpr int TMEM_COLS = TMEM_USED <= 32 ? 32 : TMEM_USED <= 64 ? 64 : TMEM_USED <= 128 ? 128 : 256;
    static_assert(TMEM_USED <= 256, "tensor memory columns");
    static_assert(STAGE % 1024 == 0, "stages stay 1024-byte aligned");
    static_assert(SMEM_BYTES <= 232448, "shared memory");
    static_assert(KS == 1 || MT * 128 * 4 <= NST * STAGE, "the partial accumulator fits in the staging ring");
};

struct HighArgs {
    const float *s_x8;
    const float *s_hi;
    float *P;
    int M, N, K;
    int group_m;   // pair kernel: tiles are handed out M-fastest in bands of group_m M-tiles
};

template <class C>
__global__ void __launch_bounds__(kHiThreads, 1)
sqf_high_kernel(const __grid_constant__ CUtensorMap tm_wh, const __grid_constant__ CUtensorMap tm_we,
                const __grid_constant__ CUtensorMap tm_x8, const HighArgs args)
{
    constexpr int MT = C::MT, NST = C::NST, KS = C::KS;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = sqd::smem_u32(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // KS = 2: CTAs 2j and 2j + 1 (one cluster) take the first and second half of tile j's stages
    const int kz = KS == 2 ? static_cast<int>(sqd::cluster_ctarank()) : 0;
    const int n0 = static_cast<int>(KS == 2 ? (blockIdx.x >> 1) : blockIdx.x) * 128;
    const int m0 = static_cast<int>(blockIdx.y) * MT;
    sqd::pdl_launch_dependents();

    const uint32_t bar0 = sbase + C::OFF_BAR;
    auto full = [&](int s) { return bar0 + 8u * s; };
    auto empty = [&](int s) { return bar0 + 8u * (NST + s); };
    const uint32_t acc_full = bar0 + 8u * (2 * NST);
    const uint32_t drain = acc_full + 8u;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::OFF_BAR + (2 * NST + 2) * 8);
    volatile uint32_t *abort_flag = reinterpret_cast<volatile uint32_t *>(tmem_slot + 1);
    auto stage = [&](int s) { return sbase + s * C::STAGE; };
    const int nst_all = args.K / 256;   // stages of the whole K range
    const int t_first = kz * nst_all / KS;   // this CTA's stages: [t_first, t_first + nst_k), nst_k >= 1
    const int nst_k = (kz + 1) * nst_all / KS - t_first;

    if (threadIdx.x == 0) {
        for (int s = 0; s < NST; ++s) {
            sqd::mbar_init(full(s), 1);
            sqd::mbar_init(empty(s), 1);
        }
        sqd::mbar_init(acc_full, 1);
        sqd::mbar_init(drain, 1);
        *abort_flag = 0u;
        sqd::fence_barrier_init();
        sqd::fence_proxy_async_smem();
    }
    if (warp == 0 && lane == 0) {
        sqd::prefetch_tensormap(&tm_wh);
        sqd::prefetch_tensormap(&tm_we);
        sqd::prefetch_tensormap(&tm_x8);
    }
    if (warp == 1) {
        sqd::tmem_alloc(sqd::smem_u32(tmem_slot), C::TMEM_COLS);
        sqd::tmem_relinquish();
    }
    sqd::tc_fence_before();
    __syncthreads();
    sqd::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    sqd::pdl_wait();

    if (warp == 0) {
        if (lane == 0) {
            int last = -1;
            bool ok = true;
            for (int u = 0; u < nst_k; ++u) {
                const int t = t_first + u;   // K stage
                const int s = u % NST;
                if (!sqd::mbar_wait(empty(s), ((u / NST) & 1) ^ 1u, abort_flag, SITE_HI_STG)) { ok = false; break; }
                const uint32_t st = stage(s);
                sqd::mbar_arrive_expect_tx(full(s), C::STAGE);
                sqd::tma_load_2d(st, &tm_wh, full(s), t * 128, n0);
                sqd::tma_load_2d(st + C::A_BYTES, &tm_x8, full(s), t * 256, m0);
                sqd::tma_load_2d(st + C::A_BYTES + C::B_BYTES, &tm_x8, full(s), t * 256 + 128, m0);
                sqd::tma_load_2d(st + C::A_BYTES + 2 * C::B_BYTES, &tm_we, full(s), t * 32, n0);
                sqd::tma_load_2d(st + C::A_BYTES + 2 * C::B_BYTES + C::E_BYTES, &tm_we, full(s), t * 32 + 16, n0);
                last = u;
            }
            if (!ok && last >= 0) sqd::mbar_drain(full(last % NST), (last / NST) & 1);
        }
        if constexpr (KS == 2) {
            __syncwarp();
            sqd::cluster_sync();   // the epilogue's two cluster barriers
            sqd::cluster_sync();
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // kind::f8f6f4, E4M3 x E4M3, fp32 D, sparse A (bit 2), M = 128, N = MT
            constexpr uint32_t idesc = (1u << 2) | (1u << 4) | (static_cast<uint32_t>(MT >> 3) << 17) |
                                       (static_cast<uint32_t>(128 >> 4) << 24);
            bool ok = true;
            for (int u = 0; u < nst_k && ok; ++u) {
                const int s = u % NST;
                if (!sqd::mbar_wait(full(s), (u / NST) & 1, abort_flag, SITE_HI_MMA)) { ok = false; break; }
                sqd::tc_fence_after();
                const uint32_t ecol = tmem + MT + 8 * s;
                const uint32_t st = stage(s);
                const uint32_t e0 = st + C::A_BYTES + 2 * C::B_BYTES;
                asm volatile("tcgen05.cp.cta_group::1.128x128b [%0], %1;" ::"r"(ecol), "l"(sqd::make_sf_desc(e0))
                             : "memory");
                asm volatile("tcgen05.cp.cta_group::1.128x128b [%0], %1;" ::"r"(ecol + 4),
                             "l"(sqd::make_sf_desc(e0 + C::E_BYTES))
                             : "memory");
                const uint64_t adesc = sqd::make_sw128_desc(st);
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint64_t bdesc = sqd::make_sw128_desc(st + C::A_BYTES + (j >> 1) * C::B_BYTES) + 4 * (j & 1);
                    asm volatile(
                        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                        "tcgen05.mma.sp.cta_group::1.kind::f8f6f4 [%0], %1, %2, [%5], %3, p;\n\t}\n" ::"r"(tmem),
                        "l"(adesc + 2 * j), "l"(bdesc), "r"(idesc), "r"((u == 0 && j == 0) ? 0u : 1u),
                        "r"(ecol + 2 * j)
                        : "memory");
                }
                sqd::mma_commit(empty(s));
            }
            if (ok) {
                sqd::mma_commit(acc_full);
            } else {
                sqd::mma_commit(drain);
                sqd::mbar_drain(drain, 0);
            }
        }
        if constexpr (KS == 2) {
            __syncwarp();
            sqd::cluster_sync();   // the epilogue's two cluster barriers
            sqd::cluster_sync();
        }
    } else if constexpr (KS == 2) {
        // epilogue of a split tile.  The second CTA's accumulator goes into the first's staging
        // ring (free once the first CTA's MMAs are done: first barrier), column-major
        // ([MT][128 rows], conflict-free); after the second barrier the first CTA adds it.
        const int q = warp & 3;
        const int row = 32 * q + lane;   // TMEM lane = W row n0 + row
        const int n = n0 + row;
        const bool n_ok = n < args.N;
        const float sh = n_ok ? args.s_hi[n] : 0.0f;
        const uint32_t tl = tmem + (static_cast<uint32_t>(32 * q) << 16);
        const bool have = sqd::mbar_wait(acc_full, 0, abort_flag, SITE_HI_EPI);
        if (have) sqd::tc_fence_after();
        __syncwarp();
        sqd::cluster_sync();
        if (kz == 1 && have) {
            const uint32_t buf0 = sqd::map_to_cta(sbase, 0);
            for (int c = 0; c < MT; c += 16) {
                uint32_t v[16];
                sqd::tmem_ld_32x32b_x16(tl + c, v);
                sqd::tmem_wait_ld_dep1(v);
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    sqd::st_cluster_f32(buf0 + 4u * static_cast<uint32_t>((c + i) * 128 + row), __uint_as_float(v[i]));
            }
        }
        __syncwarp();
        sqd::cluster_sync();
        if (kz == 0 && have) {
            const float *part = reinterpret_cast<const float *>(smem);
            for (int c = 0; c < MT; c += 16) {
                uint32_t v[16];
                sqd::tmem_ld_32x32b_x16(tl + c, v);
                sqd::tmem_wait_ld_dep1(v);
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int m = m0 + c + i;
                    const float acc = __fadd_rn(__uint_as_float(v[i]), part[(c + i) * 128 + row]);
                    if (n_ok && m < args.M)
                        args.P[static_cast<int64_t>(m) * args.N + n] = __fmul_rn(__fmul_rn(acc, args.s_x8[m]), sh);
                }
            }
        }
    } else {
        // epilogue: TMEM lane quarter warp % 4 = W rows n0 + 32 (warp % 4) + lane
        const int q = warp & 3;
        const int n = n0 + 32 * q + lane;
        const bool n_ok = n < args.N;
        const float sh = n_ok ? args.s_hi[n] : 0.0f;
        if (sqd::mbar_wait(acc_full, 0, abort_flag, SITE_HI_EPI)) {
            sqd::tc_fence_after();
            const uint32_t tl = tmem + (static_cast<uint32_t>(32 * q) << 16);
            for (int c = 0; c < MT; c += 16) {
                uint32_t v[16];
                sqd::tmem_ld_32x32b_x16(tl + c, v);
                sqd::tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int m = m0 + c + i;
                    if (n_ok && m < args.M)
                        args.P[static_cast<int64_t>(m) * args.N + n] =
                            __fmul_rn(__fmul_rn(__uint_as_float(v[i]), args.s_x8[m]), sh);
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

// ---------------------------------------------------------------- high part, CTA pairs
// The same product on 256 W rows x 256 tokens per cluster of two CTAs
// (tcgen05 cta_group::2): each CTA supplies its 128 W rows (the sparse A
// operand), their metadata and 128 of the 256 token rows (half of B), and
// receives its 128 W rows x 256 tokens of D.  Per CTA a stage carries the same
// 52 KB as the single-CTA kernel for twice the products, which halves the L2
// traffic per product.  The metadata copy of a pair moves each CTA's own
// shared memory into its own tensor memory.
//
// Persistent: one cluster per SM pair takes tiles t = pair, pair + pairs, ...
// (M-fastest in bands of group_m M-tiles, so the token band stays in L2 while
// the W tiles stream).  The staging ring runs on across tiles, so the next
// tile's operands load while the current one's epilogue writes P; the MMAs of
// the next tile wait for the epilogue to have read the accumulator.
template <int NST_, int EPI_WARPS_>
struct CfgHighPair {
    static constexpr int NST = NST_;
    // epilogue warps: 4 (one per TMEM lane quarter, all 256 columns, streamed through two
    // 16-column buffers) or 8 (two per quarter, 128 columns each, held in registers so the
    // accumulator goes back to the next tile's MMAs before P is stored)
    static constexpr int EPI_WARPS = EPI_WARPS_;
    static constexpr int THREADS = 32 * (2 + EPI_WARPS);
    static_assert(EPI_WARPS == 4 || EPI_WARPS == 8, "epilogue warps");
    static constexpr int A_BYTES = 128 * 128;   // this CTA's 128 W rows, 256 channels (2:4)
    static constexpr int B_BYTES = 128 * 128;   // this CTA's 128 tokens, one 128-channel box
    static constexpr int E_BYTES = 128 * 16;    // metadata of this CTA's W rows, 128 channels
    static constexpr int STAGE = A_BYTES + 2 * B_BYTES + 2 * E_BYTES;
    static constexpr int OFF_BAR = NST * STAGE;
    // barriers: full[NST] empty[NST] acc_full acc_empty drain; then the TMEM slot and the abort flag
    static constexpr int NBAR = 2 * NST + 3;
    static constexpr int SMEM_BYTES = OFF_BAR + NBAR * 8 + 16 + 1024;
    static constexpr int TMEM_COLS = 512;       // 256 accumulator columns + 8 metadata columns per stage
    static_assert(256 + 8 * NST <= TMEM_COLS, "tensor memory columns");
    static_assert(STAGE % 1024 == 0, "stages stay 1024-byte aligned");
    static_assert(SMEM_BYTES <= 232448, "shared memory");
};

template <class C>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(C::THREADS, 1)
sqf_high_pair_kernel(const __grid_constant__ CUtensorMap tm_wh, const __grid_constant__ CUtensorMap tm_we,
                     const __grid_constant__ CUtensorMap tm_x8, const HighArgs args)
{
    constexpr int NST = C::NST;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = sqd::smem_u32(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = sqd::cluster_ctarank();
    const bool leader = rank == 0;
    const int tiles_n = (args.N + 255) / 256;
    const int tiles_m = (args.M + 255) / 256;
    const int num_tiles = tiles_n * tiles_m;
    const int pair = static_cast<int>(blockIdx.x >> 1);
    const int num_pairs = static_cast<int>(gridDim.x >> 1);
    const int my_tiles = (num_tiles - pair + num_pairs - 1) / num_pairs;
    // tile t -> (M-tile, N-tile): bands of group_m M-tiles, M-fastest inside a band
    auto coords = [&](int t, int &mi, int &ni) {
        const int gsz = args.group_m * tiles_n;
        const int g = t / gsz;
        const int first_m = g * args.group_m;
        const int gm = min(tiles_m - first_m, args.group_m);
        const int idx = t - g * gsz;
        mi = first_m + idx % gm;
        ni = idx / gm;
    };
    sqd::pdl_launch_dependents();

    const uint32_t bar0 = sbase + C::OFF_BAR;
    auto full = [&](int s) { return bar0 + 8u * s; };
    auto empty = [&](int s) { return bar0 + 8u * (NST + s); };
    const uint32_t acc_full = bar0 + 8u * (2 * NST);
    const uint32_t acc_empty = acc_full + 8u;
    const uint32_t drain = acc_full + 16u;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::OFF_BAR + C::NBAR * 8);
    volatile uint32_t *abort_flag = reinterpret_cast<volatile uint32_t *>(tmem_slot + 1);
    auto stage = [&](int s) { return sbase + s * C::STAGE; };
    const int nst_k = args.K / 256;

    if (threadIdx.x == 0) {
        for (int s = 0; s < NST; ++s) {
            sqd::mbar_init(full(s), 2);    // both CTAs' producers (the first CTA's copy is used)
            sqd::mbar_init(empty(s), 1);   // multicast commit
        }
        sqd::mbar_init(acc_full, 1);       // multicast commit
        sqd::mbar_init(acc_empty, 2 * C::EPI_WARPS);   // the epilogue warps of both CTAs (the first CTA's copy)
        sqd::mbar_init(drain, 1);
        *abort_flag = 0u;
        sqd::fence_barrier_init();
        sqd::fence_proxy_async_smem();
    }
    if (warp == 0 && lane == 0) {
        sqd::prefetch_tensormap(&tm_wh);
        sqd::prefetch_tensormap(&tm_we);
        sqd::prefetch_tensormap(&tm_x8);
    }
    if (warp == 1) {
        sqd::tmem_alloc_pair(sqd::smem_u32(tmem_slot), C::TMEM_COLS);
        sqd::tmem_relinquish_pair();
    }
    sqd::tc_fence_before();
    sqd::cluster_sync();
    sqd::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    sqd::pdl_wait();

    if (warp == 0) {
        if (lane == 0) {
            int last = -1;
            bool ok = true;
            for (int lt = 0; lt < my_tiles && ok; ++lt) {
                int mi, ni;
                coords(pair + lt * num_pairs, mi, ni);
                const int n0 = ni * 256 + static_cast<int>(rank) * 128;   // this CTA's W rows
                const int mt = mi * 256 + static_cast<int>(rank) * 128;   // this CTA's tokens
                for (int t = 0; t < nst_k; ++t) {
                    const int u = lt * nst_k + t;
                    const int s = u % NST;
                    if (!sqd::mbar_wait(empty(s), ((u / NST) & 1) ^ 1u, abort_flag, SITE_HI_STG)) { ok = false; break; }
                    const uint32_t st = stage(s);
                    const uint32_t fl = sqd::map_to_cta(full(s), 0);
                    sqd::mbar_arrive_expect_tx_cluster(fl, C::STAGE);
                    sqd::tma_load_2d_pair(st, &tm_wh, fl, t * 128, n0);
                    sqd::tma_load_2d_pair(st + C::A_BYTES, &tm_x8, fl, t * 256, mt);
                    sqd::tma_load_2d_pair(st + C::A_BYTES + C::B_BYTES, &tm_x8, fl, t * 256 + 128, mt);
                    sqd::tma_load_2d_pair(st + C::A_BYTES + 2 * C::B_BYTES, &tm_we, fl, t * 32, n0);
                    sqd::tma_load_2d_pair(st + C::A_BYTES + 2 * C::B_BYTES + C::E_BYTES, &tm_we, fl, t * 32 + 16, n0);
                    last = u;
                }
            }
            if (!ok && last >= 0 && leader) sqd::mbar_drain(full(last % NST), (last / NST) & 1);
        }
    } else if (warp == 1) {
        if (leader && lane == 0) {
            // kind::f8f6f4, E4M3 x E4M3, fp32 D, sparse A (bit 2), M = 256 (pair), N = 256
            constexpr uint32_t idesc = (1u << 2) | (1u << 4) | (static_cast<uint32_t>(256 >> 3) << 17) |
                                       (static_cast<uint32_t>(256 >> 4) << 24);
            bool ok = true;
            for (int lt = 0; lt < my_tiles && ok; ++lt) {
                // the accumulator of the previous tile has been read
                if (!sqd::mbar_wait(acc_empty, (lt & 1) ^ 1u, abort_flag, SITE_HI_MMA)) { ok = false; break; }
                sqd::tc_fence_after();
                for (int t = 0; t < nst_k; ++t) {
                    const int u = lt * nst_k + t;
                    const int s = u % NST;
                    if (!sqd::mbar_wait(full(s), (u / NST) & 1, abort_flag, SITE_HI_MMA)) { ok = false; break; }
                    sqd::tc_fence_after();
                    const uint32_t ecol = tmem + 256 + 8 * s;   // this stage's metadata columns
                    const uint32_t st = stage(s);
                    const uint32_t e0 = st + C::A_BYTES + 2 * C::B_BYTES;
                    asm volatile("tcgen05.cp.cta_group::2.128x128b [%0], %1;" ::"r"(ecol), "l"(sqd::make_sf_desc(e0))
                                 : "memory");
                    asm volatile("tcgen05.cp.cta_group::2.128x128b [%0], %1;" ::"r"(ecol + 4),
                                 "l"(sqd::make_sf_desc(e0 + C::E_BYTES))
                                 : "memory");
                    const uint64_t adesc = sqd::make_sw128_desc(st);
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const uint64_t bdesc = sqd::make_sw128_desc(st + C::A_BYTES + (j >> 1) * C::B_BYTES) + 4 * (j & 1);
                        asm volatile(
                            "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                            "tcgen05.mma.sp.cta_group::2.kind::f8f6f4 [%0], %1, %2, [%5], %3, p;\n\t}\n" ::"r"(tmem),
                            "l"(adesc + 2 * j), "l"(bdesc), "r"(idesc), "r"((t == 0 && j == 0) ? 0u : 1u),
                            "r"(ecol + 2 * j)
                            : "memory");
                    }
                    sqd::mma_commit_pair_multicast(empty(s), 0x3);
                }
                if (ok) sqd::mma_commit_pair_multicast(acc_full, 0x3);
            }
            if (!ok) {
                sqd::mma_commit_pair(drain);
                sqd::mbar_drain(drain, 0);
            }
        }
    } else {
        // epilogue (each CTA): TMEM lane quarter warp % 4 = W rows n0 + 32 (warp % 4) + lane;
        // with 8 warps the second four take the upper 128 columns
        const int q = warp & 3;
        constexpr int NCOL = 256 / (C::EPI_WARPS / 4);
        const int c_lo = ((warp - 2) >> 2) * NCOL;
        const uint32_t empty_leader = sqd::map_to_cta(acc_empty, 0);
        const uint32_t tl = tmem + (static_cast<uint32_t>(32 * q) << 16);
        for (int lt = 0; lt < my_tiles; ++lt) {
            int mi, ni;
            coords(pair + lt * num_pairs, mi, ni);
            const int n = ni * 256 + static_cast<int>(rank) * 128 + 32 * q + lane;
            const int m0 = mi * 256;
            const bool n_ok = n < args.N;
            const float sh = n_ok ? args.s_hi[n] : 0.0f;
            if (!sqd::mbar_wait(acc_full, lt & 1, abort_flag, SITE_HI_EPI)) break;
            sqd::tc_fence_after();
            const int64_t row0 = static_cast<int64_t>(m0) * args.N + n;
            auto put = [&](const uint32_t (&v)[16], int c) {
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int m = m0 + c + i;
                    if (n_ok && m < args.M)
                        args.P[row0 + static_cast<int64_t>(c + i) * args.N] =
                            __fmul_rn(__fmul_rn(__uint_as_float(v[i]), args.s_x8[m]), sh);
                }
            };
            if constexpr (NCOL == 128) {
                // all 128 columns into registers, hand the accumulator back, then store: the
                // next tile's MMAs run while P is written
                uint32_t v[8][16];
#pragma unroll
                for (int j = 0; j < 8; ++j) sqd::tmem_ld_32x32b_x16(tl + c_lo + 16 * j, v[j]);
#pragma unroll
                for (int j = 0; j < 8; ++j) sqd::tmem_wait_ld_dep1(v[j]);
                sqd::tc_fence_before();
                __syncwarp();
                if (lane == 0) sqd::mbar_arrive_cluster(empty_leader);
#pragma unroll
                for (int j = 0; j < 8; ++j) put(v[j], c_lo + 16 * j);
            } else {
                // two 16-column buffers: the next chunk loads while this one is stored
                uint32_t va[16], vb[16];
                sqd::tmem_ld_32x32b_x16(tl + c_lo, va);
                sqd::tmem_wait_ld_dep1(va);
#pragma unroll 1
                for (int c = c_lo; c < c_lo + NCOL; c += 32) {
                    sqd::tmem_ld_32x32b_x16(tl + c + 16, vb);
                    put(va, c);
                    sqd::tmem_wait_ld_dep1(vb);
                    if (c + 32 < c_lo + NCOL) {
                        sqd::tmem_ld_32x32b_x16(tl + c + 32, va);
                    } else {
                        // every accumulator column this warp reads has been read
                        sqd::tc_fence_before();
                        __syncwarp();
                        if (lane == 0) sqd::mbar_arrive_cluster(empty_leader);
                    }
                    put(vb, c + 16);
                    if (c + 32 < c_lo + NCOL) sqd::tmem_wait_ld_dep1(va);
                }
            }
        }
    }
    sqd::tc_fence_before();
    sqd::cluster_sync();   // every pair MMA and TMEM read of both CTAs is done
    if (warp == 1) {
        sqd::tc_fence_after();
        sqd::tmem_dealloc_pair(tmem, C::TMEM_COLS);
    }
}

}  // namespace sqf
