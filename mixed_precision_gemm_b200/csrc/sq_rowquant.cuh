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
//   2. codes of every 8-channel chunk (see quant8 below) scattered as bytes
//      into shared memory at their rank among the normal channels, outliers
//      copied to a shared compact buffer at their rank in O;
//   3. codes packed two per byte and both parts written with 16-byte stores.
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

template <int T, int CPT>
__global__ void __launch_bounds__(T, (T >= 512 ? 1 : 512 / T)) rowquant_kernel(
    const uint16_t *__restrict__ src, int64_t rows, int K, int64_t ld,
    const uint32_t *__restrict__ chan_tab, int nO, int kn_pad, int no_pad,
    uint8_t *__restrict__ dst_n, float *__restrict__ dst_s, uint16_t *__restrict__ dst_o)
{
    extern __shared__ __align__(16) uint8_t rq_smem[];
    __shared__ uint32_t red[2][T / 32];
    const int buf_bytes = kn_pad + 2 * no_pad;  // one code buffer + one outlier buffer

    const int tid = threadIdx.x;
    const int KN = K - nO;
    const int nchunk = K >> 3;

    // Padding positions are never written by the row loop: zero them once in both buffers.
    for (int b = 0; b < 2; ++b) {
        int8_t *qb = reinterpret_cast<int8_t *>(rq_smem + b * buf_bytes);
        uint16_t *ob = reinterpret_cast<uint16_t *>(rq_smem + b * buf_bytes + kn_pad);
        for (int i = KN + tid; i < kn_pad; i += T) qb[i] = 0;
        for (int i = nO + tid; i < no_pad; i += T) ob[i] = 0;
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

        int8_t *qbuf = reinterpret_cast<int8_t *>(rq_smem + parity * buf_bytes);
        uint16_t *obuf = reinterpret_cast<uint16_t *>(rq_smem + parity * buf_bytes + kn_pad);

        // 1. absolute maximum over the normal channels (bf16 magnitude bits)
        uint32_t am2 = 0;
#pragma unroll
        for (int i = 0; i < CPT; ++i) {
            const uint32_t mask = tb[i] & 0xFFu;
            uint32_t w[4] = {v[i].x & 0x7FFF7FFFu, v[i].y & 0x7FFF7FFFu, v[i].z & 0x7FFF7FFFu, v[i].w & 0x7FFF7FFFu};
            if (mask) {
#pragma unroll
                for (int p = 0; p < 4; ++p) {
                    const uint32_t keep = (((mask >> (2 * p)) & 1u) ? 0u : 0x0000FFFFu) |
                                          (((mask >> (2 * p + 1)) & 1u) ? 0u : 0xFFFF0000u);
                    w[p] &= keep;
                }
            }
            am2 = max_u16x2(am2, max_u16x2(max_u16x2(w[0], w[1]), max_u16x2(w[2], w[3])));
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

        // 2. codes -> qbuf at their normal rank, outliers -> obuf at their rank in O
#pragma unroll
        for (int i = 0; i < CPT; ++i) {
            const int c = tid + i * T;
            if (c >= nchunk) continue;
            const uint32_t mask = tb[i] & 0xFFu;
            const int below = static_cast<int>(tb[i] >> 8);
            uint32_t lo, hi;
            quant8(v[i], s, inv_s, fast_ok, lo, hi);
            const int p = 8 * c - below;
            if (mask == 0u) {
                if ((p & 7) == 0) {
                    *reinterpret_cast<uint2 *>(qbuf + p) = make_uint2(lo, hi);
                } else if ((p & 3) == 0) {
                    *reinterpret_cast<uint32_t *>(qbuf + p) = lo;
                    *reinterpret_cast<uint32_t *>(qbuf + p + 4) = hi;
                } else if ((p & 1) == 0) {
                    *reinterpret_cast<uint16_t *>(qbuf + p) = static_cast<uint16_t>(lo);
                    *reinterpret_cast<uint16_t *>(qbuf + p + 2) = static_cast<uint16_t>(lo >> 16);
                    *reinterpret_cast<uint16_t *>(qbuf + p + 4) = static_cast<uint16_t>(hi);
                    *reinterpret_cast<uint16_t *>(qbuf + p + 6) = static_cast<uint16_t>(hi >> 16);
                } else {
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        qbuf[p + e] = static_cast<int8_t>(((e < 4 ? lo : hi) >> (8 * (e & 3))) & 0xFFu);
                }
            } else {
                const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
                int nlow = 0;  // outliers of this chunk before element e
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    if ((mask >> e) & 1u) {
                        obuf[below + nlow] = static_cast<uint16_t>(w[e >> 1] >> ((e & 1) * 16));
                        ++nlow;
                    } else {
                        qbuf[p + e - nlow] = static_cast<int8_t>(((e < 4 ? lo : hi) >> (8 * (e & 3))) & 0xFFu);
                    }
                }
            }
        }
        __syncthreads();

        // 3. pack and store: 32 codes -> 16 bytes per item; outliers 8 per item
        uint8_t *out_n = dst_n + r * static_cast<int64_t>(kn_pad >> 1);
        for (int j = tid; j < (kn_pad >> 5); j += T) {
            const uint4 c0 = *reinterpret_cast<const uint4 *>(qbuf + 32 * j);
            const uint4 c1 = *reinterpret_cast<const uint4 *>(qbuf + 32 * j + 16);
            uint4 o;
            o.x = pack8_codes(c0.x, c0.y);
            o.y = pack8_codes(c0.z, c0.w);
            o.z = pack8_codes(c1.x, c1.y);
            o.w = pack8_codes(c1.z, c1.w);
            *reinterpret_cast<uint4 *>(out_n + 16 * j) = o;
        }
        uint16_t *out_o = dst_o + r * static_cast<int64_t>(no_pad);
        for (int j = tid; j < (no_pad >> 3); j += T)
            *reinterpret_cast<uint4 *>(out_o + 8 * j) = *reinterpret_cast<const uint4 *>(obuf + 8 * j);
        // No barrier here: the next row fills the other buffers; this row's
        // buffers are reused two rows later, after that row's two barriers.
    }
}

}  // namespace sqq
