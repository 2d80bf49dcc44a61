// Quantize-and-gather of bf16 rows: the online activation step of the OSC
// page (arXiv:2604.12782, technical framework: "structured sub-tensor
// extraction" coalesces the scattered outlier channels into a compact dense
// tensor) and, applied to weight rows, the offline weight step (SQ-format
// write-up, section 9: symmetric quantization, columns reordered by the
// static mask).
//
// One small CTA (64 threads for K <= 4096) handles one row at a time
// (grid-stride over rows), so each thread holds up to 8 chunks of 8 channels
// and the per-row fixed work (reduction, scale, barriers, packing set-up) is
// spread over many elements; with few chunks per thread it also prefetches
// its next row into registers.  Per row:
//   1. absolute maximum over the normal channels, on packed bf16 magnitude
//      bits (exact; outlier channels masked out), block reduction;
//   2. codes of every 8-channel chunk (see quant8_pairs below) packed into one
//      32-bit nibble word -- the normal channels' codes first moved to the
//      front with a byte permutation from a 256-entry table, the same steps
//      for every chunk -- and OR-ed into a packed row in shared memory at
//      their rank among the normal channels (two shared atomics, so
//      neighbouring chunks never race); outliers go to a shared compact
//      buffer at their rank in O (in step 1, before the maximum);
//   3. both rows written out with 16-byte stores.
// Shared buffers alternate between consecutive rows, so two block barriers
// per row suffice.  Memory-bound: bytes per row = 2K read + kn_pad/2 +
// 2 no_pad + 4 written.
#pragma once

#include "sq_device.cuh"

namespace sqq {

constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23: x + kMagic rounds x to an integer (ties to even)

__device__ __forceinline__ uint32_t max_u16x2(uint32_t a, uint32_t b)
{
    uint32_t d;
    asm("max.u16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Low bytes of four words -> one word (byte i = low byte of word i).
__device__ __forceinline__ uint32_t low_bytes4(uint32_t a, uint32_t b, uint32_t c, uint32_t d)
{
    return __byte_perm(__byte_perm(a, b, 0x0040), __byte_perm(c, d, 0x0040), 0x5410);
}

// Exact code: clamp(rint(fl(x / s)), -7, 7) with the IEEE fp32 quotient.
__device__ __forceinline__ uint32_t exact_code_byte(float x, float s)
{
    int q = __float2int_rn(__fdiv_rn(x, s));
    q = q > 7 ? 7 : (q < -7 ? -7 : q);
    return static_cast<uint32_t>(q) & 0xFFu;
}

__device__ __forceinline__ float bf16_lo(uint32_t w);
__device__ __forceinline__ float bf16_hi(uint32_t w);
__device__ __forceinline__ uint32_t low_bytes4(uint32_t a, uint32_t b, uint32_t c, uint32_t d);

// The 8 codes of a chunk by correctly rounded division (rare path, kept out
// of line so that the common path stays small).
__device__ __noinline__ uint2 quant8_exact(uint4 v, float s)
{
    const float x[8] = {bf16_lo(v.x), bf16_hi(v.x), bf16_lo(v.y), bf16_hi(v.y),
                        bf16_lo(v.z), bf16_hi(v.z), bf16_lo(v.w), bf16_hi(v.w)};
    uint32_t t[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) t[e] = exact_code_byte(x[e], s);
    return make_uint2(low_bytes4(t[0], t[1], t[2], t[3]), low_bytes4(t[4], t[5], t[6], t[7]));
}

// Codes of the 8 channels of one chunk as 8 int8 bytes (lo: channels 0..3,
// hi: 4..7).  Fast path: t = fma(x, inv_s, 1.5*2^23) rounds the exact product
// x * fl(1/s) to the nearest integer q, whose int8 value is the low byte of t.
// |x*fl(1/s) - x/s| and |fl(x/s) - x/s| are both below 7 * 2^-24 for
// |x/s| <= 7, so when the residual x*fl(1/s) - q stays 2^-16 away from +-1/2
// no half-integer separates x*fl(1/s) from fl(x/s) and q = rint(fl(x/s)).
// Otherwise (or when 1/s is not safely finite) the correctly rounded
// division decides.  Codes of outlier channels in the chunk are computed but
// never used.  For |x| <= a = 7s the result never exceeds 7 in magnitude.
__device__ __forceinline__ void quant8(const uint4 &v, float s, float inv_s, bool fast_ok, uint32_t &lo,
                                       uint32_t &hi)
{
    const float x[8] = {bf16_lo(v.x), bf16_hi(v.x), bf16_lo(v.y), bf16_hi(v.y),
                        bf16_lo(v.z), bf16_hi(v.z), bf16_lo(v.w), bf16_hi(v.w)};
    uint32_t t[8];
    float worst = 0.0f;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        const float tf = fmaf(x[e], inv_s, kMagic);
        const float q = tf - kMagic;
        worst = fmaxf(worst, fabsf(fmaf(x[e], inv_s, -q)));
        t[e] = __float_as_uint(tf);
    }
    if (!fast_ok || worst > 0.49998474121f) {  // 1/2 - 2^-16
        const uint2 ex = quant8_exact(v, s);
        lo = ex.x;
        hi = ex.y;
        return;
    }
    lo = low_bytes4(t[0], t[1], t[2], t[3]);
    hi = low_bytes4(t[4], t[5], t[6], t[7]);
}

// Packs 8 code bytes (lo4: codes 0..3, hi4: codes 4..7) into 4 bytes, two
// codes per byte, the even code in the low nibble.
__device__ __forceinline__ uint32_t pack8_codes(uint32_t lo4, uint32_t hi4)
{
    const uint32_t a = lo4 & 0x0F0F0F0Fu;
    const uint32_t b = hi4 & 0x0F0F0F0Fu;
    const uint32_t pa = (a & 0x000F000Fu) | ((a & 0x0F000F00u) >> 4);  // bytes 0, 2: c0|c1<<4, c2|c3<<4
    const uint32_t pb = (b & 0x000F000Fu) | ((b & 0x0F000F00u) >> 4);
    return __byte_perm(pa, pb, 0x6420);
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

// Per-row quantizer constants, as fp32 pairs.
struct RowScale {
    uint64_t inv2;   // (fl(1/s), fl(1/s))
    uint64_t negs2;  // (-s, -s)
    uint64_t magic2; // (1.5 * 2^23, 1.5 * 2^23)
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
// with s < 2^-100 take the division path instead.  |x| <= 7 s keeps the code
// within [-7, 7].
__device__ __forceinline__ void quant8_pairs(const uint4 &v, const RowScale &rs, uint32_t &lo, uint32_t &hi)
{
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t t[8];
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        const uint64_t x = f2_pack(w[p] << 16, w[p] & 0xFFFF0000u);
        const uint64_t q0 = f2_mul(x, rs.inv2);
        const uint64_t r = f2_fma(q0, rs.negs2, x);
        const uint64_t q1 = f2_fma(r, rs.inv2, q0);
        f2_unpack(f2_add(q1, rs.magic2), t[2 * p], t[2 * p + 1]);
    }
    lo = low_bytes4(t[0], t[1], t[2], t[3]);
    hi = low_bytes4(t[4], t[5], t[6], t[7]);
}

// Byte-compaction selectors: for an 8-bit outlier mask m, the byte_perm
// selectors (low word, high word) that move the codes of the normal channels
// of a chunk to the front, in channel order.
__device__ __forceinline__ uint2 compaction_selectors(uint32_t m)
{
    uint32_t sel[2] = {0u, 0u};
    int t = 0;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        if (!((m >> e) & 1u)) {
            sel[t >> 2] |= static_cast<uint32_t>(e) << (4 * (t & 3));
            ++t;
        }
    }
    return make_uint2(sel[0], sel[1]);
}

// Keep masks for an 8-bit outlier mask: word p clears the bf16 halves of
// pair p that are outliers.
__device__ __forceinline__ uint4 keep_words(uint32_t m)
{
    uint32_t k[4];
#pragma unroll
    for (int p = 0; p < 4; ++p)
        k[p] = (((m >> (2 * p)) & 1u) ? 0u : 0x0000FFFFu) | (((m >> (2 * p + 1)) & 1u) ? 0u : 0xFFFF0000u);
    return make_uint4(k[0], k[1], k[2], k[3]);
}

template <int T, int CPT>
__global__ void __launch_bounds__(T, (T >= 512 ? 1 : 512 / T)) rowquant_kernel(
    const uint16_t *__restrict__ src, int64_t rows, int K, int64_t ld,
    const uint32_t *__restrict__ chan_tab, int nO, int kn_pad, int no_pad,
    uint8_t *__restrict__ dst_n, float *__restrict__ dst_s, uint16_t *__restrict__ dst_o)
{
    // Shared memory: two alternating (packed code row [kn_pad/2 + 16 bytes] +
    // outlier row [2 no_pad bytes]) pairs, then 256 compaction selectors and
    // 256 keep masks.
    extern __shared__ __align__(16) uint8_t rq_smem[];
    __shared__ uint32_t red[2][T / 32];
    const int pk_bytes = kn_pad >> 1;
    const int pk_alloc = pk_bytes + 16;  // room for the second OR of the last chunk
    const int buf_bytes = pk_alloc + 2 * no_pad;
    uint2 *sel_tab = reinterpret_cast<uint2 *>(rq_smem + 2 * buf_bytes);
    uint4 *keep_tab = reinterpret_cast<uint4 *>(rq_smem + 2 * buf_bytes + 256 * 8);

    const int tid = threadIdx.x;
    const int nchunk = K >> 3;

    for (int i = tid; i < 2 * buf_bytes / 16; i += T)
        reinterpret_cast<uint4 *>(rq_smem)[i] = make_uint4(0, 0, 0, 0);
    for (int m = tid; m < 256; m += T) {
        sel_tab[m] = compaction_selectors(static_cast<uint32_t>(m));
        keep_tab[m] = keep_words(static_cast<uint32_t>(m));
    }

    // The channel table is the same for every row: keep this thread's words.
    uint32_t tb[CPT];
#pragma unroll
    for (int i = 0; i < CPT; ++i) {
        const int c = tid + i * T;
        tb[i] = c < nchunk ? __ldg(chan_tab + c) : 0xFFu;
    }

    constexpr bool kPrefetch = CPT <= 4;  // registers allow holding the next row too
    uint4 nxt[kPrefetch ? CPT : 1];
    auto load_row = [&](int64_t r, uint4 *dst) {
        const uint16_t *row = src + r * ld;
#pragma unroll
        for (int i = 0; i < CPT; ++i) {
            const int c = tid + i * T;
            dst[i] = c < nchunk ? sqd::ld_nc_v4(row + 8 * c) : make_uint4(0, 0, 0, 0);
        }
    };

    int64_t r = blockIdx.x;
    if constexpr (kPrefetch) {
        if (r < rows) load_row(r, nxt);
    }
    __syncthreads();  // zeroed buffers and tables visible
    int parity = 0;
    for (; r < rows; r += gridDim.x, parity ^= 1) {
        uint4 v[CPT];
        if constexpr (kPrefetch) {
#pragma unroll
            for (int i = 0; i < CPT; ++i) v[i] = nxt[i];
            if (r + gridDim.x < rows) load_row(r + gridDim.x, nxt);
        } else {
            load_row(r, v);
        }

        uint32_t *pbuf = reinterpret_cast<uint32_t *>(rq_smem + parity * buf_bytes);          // packed codes
        uint16_t *obuf = reinterpret_cast<uint16_t *>(rq_smem + parity * buf_bytes + pk_alloc);  // outliers

        // 1. outliers to obuf at their rank in O and cleared from the chunk;
        //    absolute maximum over what is left (bf16 magnitude bits)
        uint32_t am2 = 0;
#pragma unroll
        for (int i = 0; i < CPT; ++i) {
            const uint32_t mask = tb[i] & 0xFFu;
            if (mask && tid + i * T < nchunk) {
                const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
                uint32_t mm = mask;
                int j = static_cast<int>(tb[i] >> 8);
                while (mm) {
                    const int e = __ffs(mm) - 1;
                    mm &= mm - 1;
                    obuf[j++] = static_cast<uint16_t>(w[e >> 1] >> ((e & 1) * 16));
                }
                const uint4 kp = keep_tab[mask];
                v[i].x &= kp.x;
                v[i].y &= kp.y;
                v[i].z &= kp.z;
                v[i].w &= kp.w;
            }
            am2 = max_u16x2(am2, max_u16x2(max_u16x2(v[i].x & 0x7FFF7FFFu, v[i].y & 0x7FFF7FFFu),
                                           max_u16x2(v[i].z & 0x7FFF7FFFu, v[i].w & 0x7FFF7FFFu)));
        }
        uint32_t amax = max(am2 & 0xFFFFu, am2 >> 16);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) amax = max(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, off));
        if ((tid & 31) == 0) red[parity][tid >> 5] = amax;
        __syncthreads();
        amax = red[parity][0];
#pragma unroll
        for (int wi = 1; wi < T / 32; ++wi) amax = max(amax, red[parity][wi]);

        const float a = __uint_as_float(amax << 16);
        const float s = __fdiv_rn(a, 7.0f);
        const bool zero = (amax == 0u);
        const float inv_s = zero ? 0.0f : __frcp_rn(s);
        const bool fast_ok = zero || s >= 7.888609052210118e-31f;  // 2^-100: 1/s stays finite
        if (tid == 0) dst_s[r] = zero ? 0.0f : s;
        RowScale rs;
        rs.inv2 = f2_pack(__float_as_uint(inv_s), __float_as_uint(inv_s));
        rs.negs2 = f2_pack(__float_as_uint(-s), __float_as_uint(-s));
        rs.magic2 = f2_pack(__float_as_uint(kMagic), __float_as_uint(kMagic));

        // 2. each chunk: codes, normal codes moved to the front, packed into
        //    one nibble word, OR-ed into the packed row at their rank
#pragma unroll
        for (int i = 0; i < CPT; ++i) {
            const int c = tid + i * T;
            if (c >= nchunk) continue;
            const uint32_t mask = tb[i] & 0xFFu;
            const int below = static_cast<int>(tb[i] >> 8);
            uint32_t lo, hi;
            if (fast_ok) {
                quant8_pairs(v[i], rs, lo, hi);
            } else {
                const uint2 ex = quant8_exact(v[i], s);
                lo = ex.x;
                hi = ex.y;
            }
            const uint2 sel = sel_tab[mask];
            const uint32_t clo = __byte_perm(lo, hi, sel.x);
            const uint32_t chi = __byte_perm(lo, hi, sel.y);
            const int n = 8 - __popc(mask);
            const uint32_t V = pack8_codes(clo, chi) & static_cast<uint32_t>((1ull << (4 * n)) - 1ull);
            const int p = 8 * c - below;   // rank of the chunk's first normal channel
            const int sh = (p & 7) * 4;
            uint32_t *dst = pbuf + (p >> 3);
            atomicOr(dst, V << sh);
            atomicOr(dst + 1, sh ? (V >> (32 - sh)) : 0u);
        }
        __syncthreads();

        // 3. copy out, clearing the packed row for its next use (two rows on)
        uint4 *pk16 = reinterpret_cast<uint4 *>(pbuf);
        uint4 *out_n = reinterpret_cast<uint4 *>(dst_n + r * static_cast<int64_t>(pk_bytes));
        for (int j = tid; j < (pk_alloc >> 4); j += T) {
            if (j < (pk_bytes >> 4)) out_n[j] = pk16[j];
            pk16[j] = make_uint4(0, 0, 0, 0);
        }
        uint16_t *out_o = dst_o + r * static_cast<int64_t>(no_pad);
        for (int j = tid; j < (no_pad >> 3); j += T)
            *reinterpret_cast<uint4 *>(out_o + 8 * j) = *reinterpret_cast<const uint4 *>(obuf + 8 * j);
        // No barrier here: the next row uses the other buffers; these are
        // reused two rows later, after that row's two barriers.
    }
}

}  // namespace sqq
