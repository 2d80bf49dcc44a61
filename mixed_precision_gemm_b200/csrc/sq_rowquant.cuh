// Quantize-and-gather of bf16 rows: the online activation step of the OSC
// page (arXiv:2604.12782, technical framework: "structured sub-tensor
// extraction" coalesces the scattered outlier channels into a compact dense
// tensor) and, applied to weight rows, the offline weight step (SQ-format
// write-up, section 9: symmetric quantization, columns reordered by the
// static mask).
//
// One group of G warps (G = 1 for K <= 2048) handles one row at a time
// (grid-stride over rows, the next row's loads in flight while the current
// one is processed); thread t holds chunks t, t + 32G, ... of 8
// channels (16 bytes each, 8 chunks per thread up to K = 32768).  The outlier set is
// the same for every row, so each thread computes once, per chunk, where the
// chunk's codes land in the packed row (word and nibble shift) and keeps its
// 8-bit outlier mask.  Per row:
//   1. outliers copied to a shared compact buffer at their rank in O and
//      cleared from the chunk (keep masks from a constant table, copied to
//      shared memory once per CTA); absolute
//      maximum over what is left;
//   2. reduction of the maximum over the group (shuffles; one block barrier
//      when G > 1), s = a / 7 and the per-row quantizer constants;
//   3. codes of every chunk (quant8_pairs), the normal channels' codes
//      gathered in channel order -- even-numbered ones into one word and
//      odd-numbered ones into another, by two byte permutations from the
//      constant table -- so that one shift and one logic operation pack them
//      into a nibble word, which two shared atomics OR into the packed row;
//   4. both rows written out with 16-byte stores.
// Shared buffers alternate between consecutive rows, so one barrier per row
// suffices (two when G > 1).  Memory-bound: bytes per row = 2K read +
// kn_pad/2 + 2 no_pad + 4 written.
#pragma once

#include <cuda_fp8.h>

#include "sq_device.cuh"

namespace sqq {

constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23: x + kMagic rounds x to an integer (ties to even)
constexpr int kChunksPerThread = 8;   // target; the widest rows (K > 32768) take up to 16

// ---------------------------------------------------------------- constant tables
// For the 8-bit outlier mask m of a chunk (bit e set: channel e of the chunk
// is an outlier):
//   keep[m][p]   clears the bf16 halves of word p that are outliers;
//   pack[m][0]   byte-permutation selector gathering the codes of the normal
//                channels number 0, 2, 4, 6 (in channel order) from the 8
//                code bytes of the chunk;
//   pack[m][1]   the same for normal channels number 1, 3, 5, 7;
//   pack[m][2]   mask of the 4n low bits, n = number of normal channels;
//   pack[m][3]   n.
struct QuantTables {
    uint32_t keep[256][4];
    uint32_t pack[256][4];
};

constexpr QuantTables make_quant_tables()
{
    QuantTables t{};
    for (int m = 0; m < 256; ++m) {
        for (int p = 0; p < 4; ++p)
            t.keep[m][p] = (((m >> (2 * p)) & 1) ? 0u : 0x0000FFFFu) | (((m >> (2 * p + 1)) & 1) ? 0u : 0xFFFF0000u);
        uint32_t sel[2] = {0u, 0u};
        int n = 0;
        for (int e = 0; e < 8; ++e) {
            if (!((m >> e) & 1)) {
                sel[n & 1] |= static_cast<uint32_t>(e) << (4 * (n >> 1));
                ++n;
            }
        }
        t.pack[m][0] = sel[0];
        t.pack[m][1] = sel[1];
        t.pack[m][2] = n == 8 ? 0xFFFFFFFFu : ((1u << (4 * n)) - 1u);
        t.pack[m][3] = static_cast<uint32_t>(n);
    }
    return t;
}

__device__ const QuantTables g_qtab = make_quant_tables();

// ---------------------------------------------------------------- element helpers
// |a| vs |b| per bf16 half, larger magnitude kept (its sign bit is replaced
// by the xor of the signs; callers clear it).  bf16 max handles subnormals.
__device__ __forceinline__ uint32_t maxabs_bf16x2(uint32_t a, uint32_t b)
{
    uint32_t d;
    asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}


// Low bytes of four words -> one word (byte i = low byte of word i).
__device__ __forceinline__ uint32_t low_bytes4(uint32_t a, uint32_t b, uint32_t c, uint32_t d)
{
    return __byte_perm(__byte_perm(a, b, 0x0040), __byte_perm(c, d, 0x0040), 0x5410);
}

// ---------------------------------------------------------------- paired fp32 arithmetic
// sm_100 executes two fp32 operations per instruction on register pairs.
__device__ __forceinline__ uint64_t f2_pack(uint32_t lo, uint32_t hi)
{
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "r"(lo), "r"(hi));
    return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, uint32_t &lo, uint32_t &hi)
{
    asm("mov.b64 {%0, %1}, %2;" : "=r"(lo), "=r"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b)
{
    uint64_t r;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c)
{
    uint64_t r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b)
{
    uint64_t r;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}

// Per-row quantizer constants, as fp32 pairs.  For a row whose scale s is
// below 2^-100, both x and s are first multiplied by 2^64: exact for every
// fp32 value in range (a power-of-two scaling of a normal or subnormal
// number), the quotient x / s is unchanged, and the scaled operands are far
// enough from the underflow range for the correction step below.
constexpr float kTinyScale = 7.888609052210118e-31f;  // 2^-100
constexpr float kUpScale = 18446744073709551616.0f;  // 2^64

struct RowScale {
    uint64_t inv2;   // (fl(1/s'), fl(1/s')), s' = s or s * 2^64
    uint64_t negs2;  // (-s', -s')
    uint64_t magic2; // (1.5 * 2^23, 1.5 * 2^23)
    uint64_t up2;    // (2^64, 2^64), used when s' = s * 2^64
};

// Codes of the 8 channels of a chunk as int8 bytes (lo: channels 0..3, hi:
// 4..7).  The fp32 quotient fl(x / s) is obtained with Markstein's correction
// (P. Markstein, "Computation of elementary functions on the IBM RISC
// System/6000 processor", IBM J. Res. Dev. 34(1), 1990; restated as the
// "correcting the quotient" theorem in Muller et al., Handbook of
// Floating-Point Arithmetic): with y = fl(1/s) and q0 = fl(x * y), which is
// within one ulp of x / s, the residual r = x - s * q0 is exact in one fused
// multiply-add and fl(q0 + r * y) is the correctly rounded quotient.  Adding
// 1.5 * 2^23 then rounds it to the nearest integer, ties to even, and the
// low byte of the sum is that integer as int8.  Needs 1/s finite and no
// underflow near a rounding tie (tiny |x / s| rounds to 0 either way); rows
// with s < 2^-100 run on operands scaled by 2^64 (UP).  |x| <= 7 s keeps the
// code within [-7, 7].
template <bool UP>
__device__ __forceinline__ void quant8_pairs(const uint4 &v, const RowScale &rs, uint32_t &lo, uint32_t &hi)
{
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t t[8];
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        uint64_t x = f2_pack(w[p] << 16, w[p] & 0xFFFF0000u);
        if constexpr (UP) x = f2_mul(x, rs.up2);
        const uint64_t q0 = f2_mul(x, rs.inv2);
        const uint64_t r = f2_fma(q0, rs.negs2, x);
        const uint64_t q1 = f2_fma(r, rs.inv2, q0);
        f2_unpack(f2_add(q1, rs.magic2), t[2 * p], t[2 * p + 1]);
    }
    lo = low_bytes4(t[0], t[1], t[2], t[3]);
    hi = low_bytes4(t[4], t[5], t[6], t[7]);
}

// E4M3 codes of the 8 channels of a chunk (lo: channels 0..3, hi: 4..7, one
// byte each): the same correctly rounded fp32 quotient t = fl(x / s) as
// quant8_pairs, then the hardware conversion to E4M3 (round to nearest even,
// magnitudes above 448 saturate to 448, the sign of t kept).
template <bool UP>
__device__ __forceinline__ void quant8_fp8_pairs(const uint4 &v, const RowScale &rs, uint32_t &lo, uint32_t &hi)
{
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t b[4];
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        uint64_t x = f2_pack(w[p] << 16, w[p] & 0xFFFF0000u);
        if constexpr (UP) x = f2_mul(x, rs.up2);
        const uint64_t q0 = f2_mul(x, rs.inv2);
        const uint64_t r = f2_fma(q0, rs.negs2, x);
        const uint64_t q1 = f2_fma(r, rs.inv2, q0);
        uint32_t t0, t1;
        f2_unpack(q1, t0, t1);
        b[p] = static_cast<uint32_t>(
            __nv_cvt_float2_to_fp8x2(make_float2(__uint_as_float(t0), __uint_as_float(t1)), __NV_SATFINITE, __NV_E4M3));
    }
    // The correction step turns x = -0 into +0 (r = fma(-0, -s, -0) = +0 and
    // +0 + -0 = +0), while fl(-0 / s) = -0.  For s > 0 the sign of every code
    // is the sign of x, so it is copied from the bf16 inputs: byte i of the
    // byte permutation holds the high byte (sign bit 7) of channel i.
    lo = (b[0] | (b[1] << 16)) & 0x7F7F7F7Fu;
    hi = (b[2] | (b[3] << 16)) & 0x7F7F7F7Fu;
    lo |= __byte_perm(v.x, v.y, 0x7531) & 0x80808080u;
    hi |= __byte_perm(v.z, v.w, 0x7531) & 0x80808080u;
}

// Group-wide maximum of a 32-bit value: warp shuffles, then (G > 1) the
// warps' results through shared memory and one block barrier.
template <int G>
__device__ __forceinline__ uint32_t group_max(uint32_t v, uint32_t *red)
{
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v = max(v, __shfl_xor_sync(0xFFFFFFFFu, v, off));
    if constexpr (G > 1) {
        if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
        __syncthreads();
        v = red[0];
#pragma unroll
        for (int w = 1; w < G; ++w) v = max(v, red[w]);
    }
    return v;
}


// Scale of a row, s = fl(a / d) (d = 7 for INT4 codes, 448 for E4M3).  For
// a >= 2^-100 Markstein's correction (see quant8_pairs) with yd = fl(1/d)
// gives the correctly rounded quotient in three operations; smaller a takes
// the division.
__device__ __forceinline__ float row_scale(float a, float d, float yd)
{
    if (a < kTinyScale) return __fdiv_rn(a, d);
    const float q0 = __fmul_rn(a, yd);
    const float r = __fmaf_rn(-d, q0, a);
    return __fmaf_rn(r, yd, q0);
}

// Row-invariant facts about one chunk, packed into a word: outlier mask in
// bits [0, 8), nibble offset of its first code inside its packed word in
// [8, 11), index of that packed word in [11, 32).
__device__ __forceinline__ uint32_t chunk_mask(uint32_t pl) { return pl & 0xFFu; }
__device__ __forceinline__ uint32_t chunk_nib(uint32_t pl) { return (pl >> 8) & 7u; }
__device__ __forceinline__ uint32_t chunk_word(uint32_t pl) { return pl >> 11; }

// 16-byte load of a row chunk: kept in L1 when the row's outliers are read
// back from it, streamed past L1 otherwise.
template <bool KEEP_L1>
__device__ __forceinline__ uint4 load_chunk(const uint16_t *p)
{
    if constexpr (KEEP_L1) return __ldg(reinterpret_cast<const uint4 *>(p));
    else return sqd::ld_nc_v4(p);
}

constexpr uint16_t kNoChannel = 0xFFFFu;  // outlier-list padding (K <= 65536 keeps real indices below it)

template <int G, int CPT>
__global__ void __launch_bounds__(32 * G, 512 / (32 * G)) rowquant_kernel(
    const uint16_t *__restrict__ src, int64_t rows, int K, int64_t ld,
    const uint32_t *__restrict__ chan_tab, int nO, int kn_pad, int no_pad,
    uint8_t *__restrict__ dst_n, float *__restrict__ dst_s, uint16_t *__restrict__ dst_o)
{
    constexpr int T = 32 * G;
    static_assert(CPT >= 1 && CPT <= 16, "chunks per thread");
    // Shared memory: the constant tables; the outlier channel list O (u16,
    // no_pad entries, padded with kNoChannel); two alternating packed code
    // rows of kn_pad/2 + 16 bytes.
    extern __shared__ __align__(16) uint8_t rq_smem[];
    __shared__ uint32_t red[2][G];
    QuantTables *tabs = reinterpret_cast<QuantTables *>(rq_smem);
    uint16_t *olist = reinterpret_cast<uint16_t *>(rq_smem + sizeof(QuantTables));
    uint8_t *bufs = rq_smem + sizeof(QuantTables) + ((2 * no_pad + 15) & ~15);
    const int pk_bytes = kn_pad >> 1;
    const int pk_alloc = pk_bytes + 16;  // room for the second OR of the last chunk

    const int tid = threadIdx.x;
    const int nchunk = K >> 3;
    const bool has_o = nO > 0;

    sqd::pdl_launch_dependents();
    constexpr bool kPrefetch = CPT <= 8;  // registers allow holding the next row too
    uint4 nxt[kPrefetch ? CPT : 1];
    auto load_row = [&](int64_t r, uint4 *dst) {
        const uint16_t *row = src + r * ld;
#pragma unroll
        for (int i = 0; i < CPT; ++i) {
            const int c = tid + i * T;
            dst[i] = c >= nchunk ? make_uint4(0, 0, 0, 0)
                     : has_o     ? load_chunk<true>(row + 8 * c)
                                 : load_chunk<false>(row + 8 * c);
        }
    };
    // Set-up (runs while the previous kernel in the stream may still be finishing).
    for (int i = tid; i < static_cast<int>(sizeof(QuantTables) / 16); i += T)
        reinterpret_cast<uint4 *>(tabs)[i] = __ldg(reinterpret_cast<const uint4 *>(&g_qtab) + i);
    for (int i = tid; i < 2 * pk_alloc / 16; i += T)
        reinterpret_cast<uint4 *>(bufs)[i] = make_uint4(0, 0, 0, 0);
    for (int j = nO + tid; j < no_pad; j += T) olist[j] = kNoChannel;

    // Where each of this thread's chunks goes: the rank p of its first normal
    // channel among the normal channels is 8c minus the outliers below it.
    // The chunk's outliers, at ranks below, below + 1, ..., enter the list O.
    uint32_t pl[CPT];
#pragma unroll
    for (int i = 0; i < CPT; ++i) {
        const int c = tid + i * T;
        pl[i] = 0u;
        if (c < nchunk) {
            const uint32_t tb = __ldg(chan_tab + c);
            const uint32_t below = tb >> 8;
            const uint32_t p = 8u * static_cast<uint32_t>(c) - below;
            pl[i] = (tb & 0xFFu) | ((p & 7u) << 8) | ((p >> 3) << 11);
            for (uint32_t mm = tb & 0xFFu, j = below; mm; mm &= mm - 1, ++j)
                olist[j] = static_cast<uint16_t>(8 * c + __ffs(mm) - 1);
        }
    }
    const float y7 = __frcp_rn(7.0f);
    __syncthreads();  // tables, outlier list and zeroed buffers visible
    sqd::pdl_wait();  // X and the outputs may belong to the previous kernel
    if constexpr (kPrefetch) {
        if (blockIdx.x < rows) load_row(blockIdx.x, nxt);
    }

    int parity = 0;
    for (int64_t r = blockIdx.x; r < rows; r += gridDim.x, parity ^= 1) {
        uint4 v[CPT];
        if constexpr (kPrefetch) {
#pragma unroll
            for (int i = 0; i < CPT; ++i) v[i] = nxt[i];
            if (r + gridDim.x < rows) load_row(r + gridDim.x, nxt);
        } else {
            load_row(r, v);
        }
        uint32_t *pbuf = reinterpret_cast<uint32_t *>(bufs + parity * pk_alloc);  // packed codes

        // 1. outlier channels cleared from the chunks; absolute maximum over
        //    what is left
        uint32_t am = 0u;
#pragma unroll
        for (int i = 0; i < CPT; ++i) {
            const uint4 kp = *reinterpret_cast<const uint4 *>(tabs->keep[chunk_mask(pl[i])]);
            v[i].x &= kp.x;
            v[i].y &= kp.y;
            v[i].z &= kp.z;
            v[i].w &= kp.w;
            am = maxabs_bf16x2(am, maxabs_bf16x2(maxabs_bf16x2(v[i].x, v[i].y), maxabs_bf16x2(v[i].z, v[i].w)));
        }
        const uint32_t amax = group_max<G>(max(am & 0x7FFFu, (am >> 16) & 0x7FFFu), red[parity]);

        // 2. per-row scale and quantizer constants
        const bool zero = (amax == 0u);
        const float s = zero ? 0.0f : row_scale(__uint_as_float(amax << 16), 7.0f, y7);
        const bool up = !zero && s < kTinyScale;
        const float s1 = up ? s * kUpScale : s;
        const float inv_s = zero ? 0.0f : __frcp_rn(s1);
        if (tid == 0) dst_s[r] = s;
        RowScale rs;
        rs.inv2 = f2_pack(__float_as_uint(inv_s), __float_as_uint(inv_s));
        rs.negs2 = f2_pack(__float_as_uint(-s1), __float_as_uint(-s1));
        rs.magic2 = f2_pack(__float_as_uint(kMagic), __float_as_uint(kMagic));
        rs.up2 = f2_pack(__float_as_uint(kUpScale), __float_as_uint(kUpScale));

        // 3. codes of each chunk, normal ones packed and OR-ed into the row
#pragma unroll
        for (int i = 0; i < CPT; ++i) {
            const int c = tid + i * T;
            if (c >= nchunk) continue;
            uint32_t lo, hi;
            if (!up) quant8_pairs<false>(v[i], rs, lo, hi);
            else quant8_pairs<true>(v[i], rs, lo, hi);
            const uint4 pk = *reinterpret_cast<const uint4 *>(tabs->pack[chunk_mask(pl[i])]);
            const uint32_t ev = __byte_perm(lo, hi, pk.x);  // normal codes 0, 2, 4, 6
            const uint32_t od = __byte_perm(lo, hi, pk.y);  // normal codes 1, 3, 5, 7
            const uint32_t V = ((ev & 0x0F0F0F0Fu) | ((od << 4) & 0xF0F0F0F0u)) & pk.z;
            const uint32_t sh = 4u * chunk_nib(pl[i]);
            uint32_t *dst = pbuf + chunk_word(pl[i]);
            atomicOr(dst, V << sh);
            if (sh) atomicOr(dst + 1, V >> (32u - sh));
        }

        // 4. compact outlier row X_O[r, j] = X[r, O[j]], two entries per
        //    thread and step, read back from the row (L1, else L2)
        if (has_o) {
            const uint16_t *row = src + r * ld;
            uint32_t *out_o = reinterpret_cast<uint32_t *>(dst_o + r * static_cast<int64_t>(no_pad));
            const uint32_t *ol2 = reinterpret_cast<const uint32_t *>(olist);
#pragma unroll 4
            for (int jp = tid; jp < (no_pad >> 1); jp += T) {
                const uint32_t e2 = ol2[jp];
                const uint32_t e0 = e2 & 0xFFFFu, e1 = e2 >> 16;
                const uint32_t x0 = e0 != kNoChannel ? __ldg(row + e0) : 0u;
                const uint32_t x1 = e1 != kNoChannel ? __ldg(row + e1) : 0u;
                out_o[jp] = x0 | (x1 << 16);
            }
        }
        if constexpr (G == 1) __syncwarp();
        else __syncthreads();

        // 5. packed row out, cleared for its next use (two rows on)
        uint4 *pk16 = reinterpret_cast<uint4 *>(pbuf);
        uint4 *out_n = reinterpret_cast<uint4 *>(dst_n + r * static_cast<int64_t>(pk_bytes));
        for (int j = tid; j < (pk_alloc >> 4); j += T) {
            if (j < (pk_bytes >> 4)) out_n[j] = pk16[j];
            pk16[j] = make_uint4(0, 0, 0, 0);
        }
        // No barrier here: the next row uses the other buffer; this one is
        // reused two rows later, after that row's barrier.
    }
}

}  // namespace sqq
