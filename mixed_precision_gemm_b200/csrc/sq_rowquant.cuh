// Quantize-and-gather of bf16 rows: the online activation step of the OSC
// page (arXiv:2604.12782, technical framework: "structured sub-tensor
// extraction" coalesces the scattered outlier channels into a compact dense
// tensor) and, applied to weight rows, the offline weight step (SQ-format
// write-up, section 9: symmetric quantization, columns reordered by the
// static mask).
//
// One CTA handles one row at a time (grid-stride over rows).  The row is read
// once from HBM with 16-byte loads held in registers; a block reduction gives
// the absolute maximum over the normal channels; each element then goes
// either to a code byte in shared memory (at its rank among the normal
// channels) or to the compact outlier buffer (at its rank in O); finally the
// codes are packed two per byte and both parts are written with 16-byte
// stores.  Memory-bound: bytes per row = 2K read + kn_pad/2 + 2 no_pad + 4
// written.
#pragma once

#include "sq_device.cuh"

namespace sqq {

// Code of x for scale s (s > 0): clamp(rint(fl(x / s)), -7, 7) with the IEEE
// fp32 quotient fl(x / s).  The quotient is first estimated as x * fl(1/s),
// which is within 2^-19 of fl(x / s) for |x / s| <= 7.  When the estimate is
// farther than 2^-16 from every half-integer, both round to the same integer
// and the estimate is used; otherwise the correctly rounded division decides.
__device__ __forceinline__ int quant_code(float x, float s, float inv_s, bool fast_ok)
{
    float t;
    if (fast_ok) {
        const float r = x * inv_s;
        const float fr = r - floorf(r);
        if (fabsf(fr - 0.5f) > 1.52587890625e-05f) {  // 2^-16
            t = r;
        } else {
            t = __fdiv_rn(x, s);
        }
    } else {
        t = __fdiv_rn(x, s);
    }
    int q = __float2int_rn(t);
    q = q > 7 ? 7 : q;
    q = q < -7 ? -7 : q;
    return q;
}

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t b)
{
    return __uint_as_float(b << 16);
}

// Packs 32 code bytes (int8, values in [-7, 7]) into 16 bytes, two codes per
// byte, even code in the low nibble.
__device__ __forceinline__ uint32_t pack8_codes(uint32_t lo4, uint32_t hi4)
{
    // lo4 holds codes 0..3 (one per byte), hi4 codes 4..7.
    uint32_t a = lo4 & 0x0F0F0F0Fu;           // nibbles in the low half of each byte
    uint32_t b = hi4 & 0x0F0F0F0Fu;
    // byte k of a: code k.  Want nibble 2i = code 2i (low), 2i+1 = code 2i+1 (high).
    uint32_t pa = (a & 0x000F000Fu) | ((a & 0x0F000F00u) >> 4);  // bytes 0,2: code0|code1<<4, code2|code3<<4
    uint32_t pb = (b & 0x000F000Fu) | ((b & 0x0F000F00u) >> 4);
    // pa: byte0 = c0|c1<<4, byte2 = c2|c3<<4 ; pb similarly for c4..c7
    return __byte_perm(pa, pb, 0x6420);
}

template <int T, int CPT>
__global__ void __launch_bounds__(T) rowquant_kernel(
    const uint16_t *__restrict__ src, int64_t rows, int K, int64_t ld,
    const uint32_t *__restrict__ chan_tab, int nO, int kn_pad, int no_pad,
    uint8_t *__restrict__ dst_n, float *__restrict__ dst_s, uint16_t *__restrict__ dst_o)
{
    extern __shared__ __align__(16) uint8_t rq_smem[];
    int8_t *qbuf = reinterpret_cast<int8_t *>(rq_smem);                  // [kn_pad] codes
    uint16_t *obuf = reinterpret_cast<uint16_t *>(rq_smem + kn_pad);     // [no_pad] bf16 bits
    __shared__ uint32_t red[T / 32];

    const int tid = threadIdx.x;
    const int KN = K - nO;
    const int nchunk = K >> 3;

    // Padding positions are never written by the row loop: zero them once.
    for (int i = KN + tid; i < kn_pad; i += T) qbuf[i] = 0;
    for (int i = nO + tid; i < no_pad; i += T) obuf[i] = 0;

    for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
        const uint16_t *row = src + r * ld;
        uint4 v[CPT];
        uint32_t tb[CPT];
#pragma unroll
        for (int i = 0; i < CPT; ++i) {
            const int c = tid + i * T;
            if (c < nchunk) {
                v[i] = sqd::ld_nc_v4(row + 8 * c);
                tb[i] = __ldg(chan_tab + c);
            } else {
                v[i] = make_uint4(0, 0, 0, 0);
                tb[i] = 0xFFu;  // all outliers: excluded from everything below
            }
        }

        // Absolute maximum over the normal channels, on bf16 magnitude bits
        // (monotone in the value for finite inputs, and exact).
        uint32_t amax = 0;
#pragma unroll
        for (int i = 0; i < CPT; ++i) {
            const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const uint32_t bits = (w[e >> 1] >> ((e & 1) * 16)) & 0x7FFFu;
                if (!((tb[i] >> e) & 1u)) amax = bits > amax ? bits : amax;
            }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const uint32_t o = __shfl_xor_sync(0xFFFFFFFFu, amax, off);
            amax = o > amax ? o : amax;
        }
        if ((tid & 31) == 0) red[tid >> 5] = amax;
        __syncthreads();
        amax = red[0];
#pragma unroll
        for (int wi = 1; wi < T / 32; ++wi) amax = red[wi] > amax ? red[wi] : amax;

        const float a = bf16_bits_to_f32(amax);
        const float s = __fdiv_rn(a, 7.0f);
        const bool zero = (amax == 0u);
        const float inv_s = zero ? 0.0f : __frcp_rn(s);
        const bool fast_ok = s >= 7.888609052210118e-31f;  // 2^-100: 1/s stays finite
        if (tid == 0) dst_s[r] = zero ? 0.0f : s;

        // Scatter: codes to qbuf at their normal rank, outliers to obuf at
        // their rank in O.
#pragma unroll
        for (int i = 0; i < CPT; ++i) {
            const int c = tid + i * T;
            if (c >= nchunk) continue;
            const uint32_t mask = tb[i] & 0xFFu;
            const int below = static_cast<int>(tb[i] >> 8);
            const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
            if (mask == 0u) {
                // No outlier in this chunk: 8 consecutive normal ranks.
                uint32_t packed_lo = 0, packed_hi = 0;
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float x = bf16_bits_to_f32((w[e >> 1] >> ((e & 1) * 16)) & 0xFFFFu);
                    const int q = zero ? 0 : quant_code(x, s, inv_s, fast_ok);
                    const uint32_t byte = static_cast<uint32_t>(q) & 0xFFu;
                    if (e < 4) packed_lo |= byte << (8 * e);
                    else packed_hi |= byte << (8 * (e - 4));
                }
                const int p = 8 * c - below;
                if ((p & 7) == 0) {
                    *reinterpret_cast<uint2 *>(qbuf + p) = make_uint2(packed_lo, packed_hi);
                } else {
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        qbuf[p + e] = static_cast<int8_t>(((e < 4 ? packed_lo : packed_hi) >> (8 * (e & 3))) & 0xFFu);
                }
            } else {
                int nlow = 0;  // outliers of this chunk before element e
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const uint32_t bits = (w[e >> 1] >> ((e & 1) * 16)) & 0xFFFFu;
                    if ((mask >> e) & 1u) {
                        obuf[below + nlow] = static_cast<uint16_t>(bits);
                        ++nlow;
                    } else {
                        const int q = zero ? 0 : quant_code(bf16_bits_to_f32(bits), s, inv_s, fast_ok);
                        qbuf[8 * c - below + (e - nlow)] = static_cast<int8_t>(q);
                    }
                }
            }
        }
        __syncthreads();

        // Pack and store: 32 codes -> 16 bytes per thread-iteration.
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
        for (int j = tid; j < (no_pad >> 3); j += T) {
            *reinterpret_cast<uint4 *>(out_o + 8 * j) = *reinterpret_cast<const uint4 *>(obuf + 8 * j);
        }
        __syncthreads();  // qbuf, obuf and red are reused by the next row
    }
}

}  // namespace sqq
