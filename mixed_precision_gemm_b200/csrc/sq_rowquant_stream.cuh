// Quantize-and-gather with rows streamed through shared memory (K <= 16384).
// Same computation and output layout as rowquant_kernel (sq_rowquant.cuh);
// the difference is how rows reach the threads.
//
// A persistent CTA (one per SM) owns rows b, b + grid, b + 2 grid, ...  One
// thread of warp 0 copies whole rows (2K bytes, one bulk asynchronous copy
// each) into a ring of shared-memory slots, completion counted on an
// mbarrier per slot; NGRP groups of G consumer warps take the CTA's rows in
// turn (row i of the CTA goes to group i % NGRP), SPG slots per group, so a
// group's next rows are in flight while it works on the current one.
//
// A group works on a row in this order: (0) the compact outlier row is
// gathered from the slot and the outlier channels are set to zero there;
// (1) each thread loads its chunks of the row into registers and takes their
// absolute maximum (zeros cannot raise it, so no masking is needed), the
// group-wide maximum follows (shuffles; a named barrier when G > 1) -- the
// slot is handed back at this point, as the row now lives in registers;
// (2) scale, then the codes of every chunk, the normal channels' codes packed
// and OR-ed into the group's packed row (as in rowquant_kernel); the packed
// row is then written out.
//
// Every wait is bounded; after a timeout the abort flag makes the remaining
// waits return at once, and every group still walks through the same rows
// and named barriers, so the CTA always finishes.
#pragma once

#include "sq_rowquant.cuh"

namespace sqq {

constexpr int kStreamMaxK = 16384;
constexpr int kStreamChunks = 8;  // most 8-channel chunks per thread and row: K <= 2048 G

enum : unsigned { SITE_RQ_PROD = 0x601, SITE_RQ_CONS = 0x602 };

// Shared-memory layout, computed identically on the host and the device.
// The table is the packing half of QuantTables (pack[256][4]).
struct StreamLayout {
    int row_bytes;   // 2K, rounded up to 128
    int pk_alloc;    // code bytes per row (kn_pad / 2 INT4, kn_pad E4M3) + 16
    int nslot;       // ring slots (spg per group)
    int off_pl, off_olist, off_pbuf, off_bar, off_misc, off_ring, bytes;

    __host__ __device__ StreamLayout(int K, int kn_pad, int no_pad, int ngrp, int spg, bool fp8)
    {
        row_bytes = (2 * K + 127) & ~127;
        pk_alloc = (fp8 ? kn_pad : kn_pad / 2) + 16;
        nslot = spg * ngrp;
        off_pl = static_cast<int>(sizeof(QuantTables::pack));
        off_olist = off_pl + ((4 * (K / 8) + 15) & ~15);
        off_pbuf = off_olist + ((2 * no_pad + 15) & ~15);
        off_bar = off_pbuf + ngrp * ((pk_alloc + 15) & ~15);
        off_misc = off_bar + 2 * nslot * 8;
        off_ring = (off_misc + 16 + 8 * ngrp * 4 + 127) & ~127;   // + per-group reduction words
        bytes = off_ring + nslot * row_bytes;
    }
};

__device__ __forceinline__ void named_bar_sync(int id, int threads)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// Most consumer groups per CTA for G warps per row (more warps per row
// raise the warps per SM without more shared memory; every thread holds its
// chunks of the row in registers).
__host__ __device__ constexpr int stream_max_groups(int G) { return G <= 2 ? 8 : G == 4 ? 6 : 3; }

// FP8: E4M3 codes (one byte per normal channel, scale absmax / 448) in place
// of INT4 codes (OSC's FP8 fallback for the inputs of W2).
template <int G, bool FP8>
__global__ void __launch_bounds__(32 * (1 + stream_max_groups(G) * G), 1) rowquant_stream_kernel(
    const uint16_t *__restrict__ src, int64_t rows, int K, int64_t ld,
    const uint32_t *__restrict__ chan_tab, int nO, int kn_pad, int no_pad,
    uint8_t *__restrict__ dst_n, float *__restrict__ dst_s, uint16_t *__restrict__ dst_o, int ngrp, int spg)
{
    extern __shared__ __align__(128) uint8_t rs_smem[];
    const StreamLayout L(K, kn_pad, no_pad, ngrp, spg, FP8);
    uint32_t (*pack_tab)[4] = reinterpret_cast<uint32_t (*)[4]>(rs_smem);
    uint32_t *pl_tab = reinterpret_cast<uint32_t *>(rs_smem + L.off_pl);
    uint16_t *olist = reinterpret_cast<uint16_t *>(rs_smem + L.off_olist);
    const uint32_t sbase = sqd::smem_u32(rs_smem);
    const int nslot = L.nslot;
    auto full = [&](int s) { return sbase + L.off_bar + 8u * s; };
    auto empty = [&](int s) { return sbase + L.off_bar + 8u * (nslot + s); };
    volatile uint32_t *abort_flag = reinterpret_cast<volatile uint32_t *>(rs_smem + L.off_misc);
    uint32_t *red = reinterpret_cast<uint32_t *>(rs_smem + L.off_misc + 16);   // [ngrp][8]

    const int tid = threadIdx.x;
    const int nthr = blockDim.x;
    const int nchunk = K >> 3;
    sqd::pdl_launch_dependents();

    // ---------------------------------------------------------------- set-up
    // (runs while the previous kernel in the stream may still be finishing)
    if (tid == 0) {
        for (int s = 0; s < nslot; ++s) {
            sqd::mbar_init(full(s), 1);   // producer's expect-tx arrival + the copy's bytes
            sqd::mbar_init(empty(s), G);  // one arrival per warp of the consuming group
        }
        *abort_flag = 0u;
        sqd::fence_barrier_init();
    }
    for (int i = tid; i < static_cast<int>(sizeof(QuantTables::pack) / 16); i += nthr)
        reinterpret_cast<uint4 *>(rs_smem)[i] = __ldg(reinterpret_cast<const uint4 *>(&g_qtab.pack[0][0]) + i);
    for (int i = tid; i < ngrp * ((L.pk_alloc + 15) / 16); i += nthr)
        reinterpret_cast<uint4 *>(rs_smem + L.off_pbuf)[i] = make_uint4(0, 0, 0, 0);
    for (int j = nO + tid; j < no_pad; j += nthr) olist[j] = kNoChannel;
    // Per chunk: outlier mask, packed word and position inside it of its
    // first code (a nibble for INT4, a byte for E4M3; see rowquant_kernel);
    // its outliers enter the list O.
    for (int c = tid; c < nchunk; c += nthr) {
        const uint32_t tb = __ldg(chan_tab + c);
        const uint32_t below = tb >> 8;
        const uint32_t p = 8u * static_cast<uint32_t>(c) - below;
        pl_tab[c] = FP8 ? ((tb & 0xFFu) | ((p & 3u) << 8) | ((p >> 2) << 11))
                        : ((tb & 0xFFu) | ((p & 7u) << 8) | ((p >> 3) << 11));
        for (uint32_t mm = tb & 0xFFu, j = below; mm; mm &= mm - 1, ++j)
            olist[j] = static_cast<uint16_t>(8 * c + __ffs(mm) - 1);
    }
    __syncthreads();
    sqd::pdl_wait();  // X and the outputs may belong to the previous kernel

    const int warp = tid >> 5;
    const int lane = tid & 31;
    if (warp == 0) {
        // ------------------------------------------------------------ row copies
        if (lane == 0) {
            int64_t issued = 0;
            for (int64_t i = 0;; ++i) {
                const int64_t r = blockIdx.x + i * gridDim.x;
                if (r >= rows) break;
                const int s = static_cast<int>(i % nslot);
                if (!sqd::mbar_wait(empty(s), static_cast<uint32_t>((i / nslot) & 1) ^ 1u, abort_flag, SITE_RQ_PROD))
                    break;
                sqd::mbar_arrive_expect_tx(full(s), static_cast<uint32_t>(2 * K));
                sqd::bulk_load(sbase + L.off_ring + s * L.row_bytes, src + r * ld, static_cast<uint32_t>(2 * K), full(s));
                issued = i + 1;
            }
            if (*abort_flag) {
                // Let the copies still in flight land before the CTA exits.
                for (int64_t i = issued > nslot ? issued - nslot : 0; i < issued; ++i)
                    sqd::mbar_drain(full(static_cast<int>(i % nslot)), static_cast<uint32_t>((i / nslot) & 1));
            }
        }
        return;
    }

    // ---------------------------------------------------------------- consumer groups
    const int gi = (warp - 1) / G;       // group
    const int gt = tid - 32 - gi * 32 * G;  // thread index inside the group
    const int GT = 32 * G;
    const int bar_id = 1 + gi;
    auto group_sync = [&] {
        if constexpr (G > 1) named_bar_sync(bar_id, GT);
        else __syncwarp();
    };
    uint32_t *pbuf = reinterpret_cast<uint32_t *>(rs_smem + L.off_pbuf + gi * L.pk_alloc);
    const uint32_t *ol2 = reinterpret_cast<const uint32_t *>(olist);
    const int pk_bytes = FP8 ? kn_pad : (kn_pad >> 1);
    constexpr float kDiv = FP8 ? 448.0f : 7.0f;  // largest code magnitude
    const float ydiv = __frcp_rn(kDiv);
    const RowScale rs_const = [] {
        RowScale r{};
        r.magic2 = f2_pack(__float_as_uint(kMagic), __float_as_uint(kMagic));
        r.up2 = f2_pack(__float_as_uint(kUpScale), __float_as_uint(kUpScale));
        return r;
    }();
    // Packing of a chunk without outliers: codes 0, 2, 4, 6 / 1, 3, 5, 7, all 8 kept.
    const uint4 pk_plain = make_uint4(pack_tab[0][0], pack_tab[0][1], pack_tab[0][2], pack_tab[0][3]);

    // Row i = gi + j ngrp of the CTA (the group's j-th row) sits in slot i % nslot =
    // gi + ngrp (j % spg) with phase parity (i / nslot) & 1 = (j / spg) & 1; both are
    // kept as counters (no 64-bit division per row).
    int sj = 0;
    uint32_t ph = 0u;
    const int64_t rstep = static_cast<int64_t>(ngrp) * gridDim.x;
    for (int64_t r = blockIdx.x + static_cast<int64_t>(gi) * gridDim.x; r < rows; r += rstep) {
        const int s = gi + ngrp * sj;
        // A timed-out wait only raises the abort flag: the group goes on with
        // whatever the slot holds, so that every barrier below is still met.
        sqd::mbar_wait(full(s), ph, abort_flag, SITE_RQ_CONS);
        if (++sj == spg) { sj = 0; ph ^= 1u; }
        uint16_t *xrow = reinterpret_cast<uint16_t *>(rs_smem + L.off_ring + s * L.row_bytes);

        // 0. compact outlier row X_O[r, j] = X[r, O[j]], then the outlier channels set to zero
        if (nO > 0) {
            uint32_t *out_o = reinterpret_cast<uint32_t *>(dst_o + r * static_cast<int64_t>(no_pad));
#pragma unroll 4
            for (int jp = gt; jp < (no_pad >> 1); jp += GT) {
                const uint32_t e2 = ol2[jp];
                const uint32_t e0 = e2 & 0xFFFFu, e1 = e2 >> 16;
                const uint32_t x0 = e0 != kNoChannel ? xrow[e0] : 0u;
                const uint32_t x1 = e1 != kNoChannel ? xrow[e1] : 0u;
                out_o[jp] = x0 | (x1 << 16);
                if (e0 != kNoChannel) xrow[e0] = 0;
                if (e1 != kNoChannel) xrow[e1] = 0;
            }
            group_sync();   // the zeros are in place for every warp of the group
        }

        // 1. the row's chunks into registers; absolute maximum (outliers are zero now)
        uint4 v[kStreamChunks];
        uint32_t am = 0u;
#pragma unroll
        for (int k = 0; k < kStreamChunks; ++k) {
            const int c = gt + k * GT;
            v[k] = c < nchunk ? *reinterpret_cast<const uint4 *>(rs_smem + L.off_ring + s * L.row_bytes + 16 * c)
                              : make_uint4(0u, 0u, 0u, 0u);
            am = maxabs_bf16x2(am, maxabs_bf16x2(maxabs_bf16x2(v[k].x, v[k].y), maxabs_bf16x2(v[k].z, v[k].w)));
        }
        // The slot has been read by this warp: hand it back (after the zeros it
        // wrote, which the next bulk copy into the slot must not overtake).
        if (nO > 0) sqd::fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) sqd::mbar_arrive(empty(s));
        uint32_t amax = max(am & 0x7FFFu, (am >> 16) & 0x7FFFu);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) amax = max(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, off));
        if constexpr (G > 1) {
            if (lane == 0) red[gi * 8 + (gt >> 5)] = amax;
            named_bar_sync(bar_id, GT);
            amax = red[gi * 8];
#pragma unroll
            for (int w = 1; w < G; ++w) amax = max(amax, red[gi * 8 + w]);
        }

        // 2. scale and quantizer constants
        const bool zero = (amax == 0u);
        const float sc = zero ? 0.0f : row_scale(__uint_as_float(amax << 16), kDiv, ydiv);
        const bool up = !zero && sc < kTinyScale;
        const float s1 = up ? sc * kUpScale : sc;
        const float inv_s = zero ? 0.0f : __frcp_rn(s1);
        if (gt == 0) dst_s[r] = sc;
        RowScale rs = rs_const;
        rs.inv2 = f2_pack(__float_as_uint(inv_s), __float_as_uint(inv_s));
        rs.negs2 = f2_pack(__float_as_uint(-s1), __float_as_uint(-s1));

        // 3. codes of each chunk, normal ones packed and OR-ed into the row
#pragma unroll
        for (int k = 0; k < kStreamChunks; ++k) {
            const int c = gt + k * GT;
            if (c >= nchunk) break;
            const uint32_t pl = pl_tab[c];
            uint32_t lo, hi;
            uint4 pk = pk_plain;
            if (chunk_mask(pl)) pk = *reinterpret_cast<const uint4 *>(pack_tab[chunk_mask(pl)]);
            if constexpr (!FP8) {
                if (!up) quant8_pairs<false>(v[k], rs, lo, hi);
                else quant8_pairs<true>(v[k], rs, lo, hi);
                const uint32_t ev = __byte_perm(lo, hi, pk.x);  // normal codes 0, 2, 4, 6
                const uint32_t od = __byte_perm(lo, hi, pk.y);  // normal codes 1, 3, 5, 7
                const uint32_t V = ((ev & 0x0F0F0F0Fu) | ((od << 4) & 0xF0F0F0F0u)) & pk.z;
                const uint32_t sh = 4u * chunk_nib(pl);
                uint32_t *dst = pbuf + chunk_word(pl);
                atomicOr(dst, V << sh);
                if (sh) atomicOr(dst + 1, V >> (32u - sh));
            } else {
                if (zero) {
                    lo = hi = 0u;  // a zero row has all-zero codes
                } else if (!up) {
                    quant8_fp8_pairs<false>(v[k], rs, lo, hi);
                } else {
                    quant8_fp8_pairs<true>(v[k], rs, lo, hi);
                }
                // normal codes in channel order: A = codes 0..3, B = 4..7, the
                // bytes past the n normal channels cleared
                const uint32_t ev = __byte_perm(lo, hi, pk.x);
                const uint32_t od = __byte_perm(lo, hi, pk.y);
                const uint32_t n = pk.w;
                const uint32_t A = __byte_perm(ev, od, 0x5140) & (n >= 4 ? 0xFFFFFFFFu : (1u << (8 * n)) - 1u);
                const uint32_t B = __byte_perm(ev, od, 0x7362) &
                                   (n >= 8 ? 0xFFFFFFFFu : n > 4 ? (1u << (8 * (n - 4))) - 1u : 0u);
                const uint32_t sh = 8u * chunk_nib(pl);
                uint32_t *dst = pbuf + chunk_word(pl);
                atomicOr(dst, A << sh);
                atomicOr(dst + 1, __funnelshift_l(A, B, sh));
                if (sh) atomicOr(dst + 2, __funnelshift_l(B, 0u, sh));
            }
        }
        group_sync();   // the packed row is complete

        // 4. packed row out, cleared for the group's next row
        uint4 *pk16 = reinterpret_cast<uint4 *>(pbuf);
        uint4 *out_n = reinterpret_cast<uint4 *>(dst_n + r * static_cast<int64_t>(pk_bytes));
        for (int j = gt; j < (L.pk_alloc >> 4); j += GT) {
            if (j < (pk_bytes >> 4)) out_n[j] = pk16[j];
            pk16[j] = make_uint4(0, 0, 0, 0);
        }
        // Cleared before the group's next row ORs into it: with G > 1 the next
        // row's named barriers order it; a single warp only needs its own lanes.
        if constexpr (G == 1) __syncwarp();
    }
}

}  // namespace sqq
