// Quantize-and-gather for the micro-scaling FP4 (MXFP4) low path.
//
// OSC (arXiv:2604.12782), abstract: the channel split is meant for 4-bit
// micro-scaling hardware; SQ-format write-up of arXiv:2512.05409, section 8:
// the format also works with FP4 data.  The block format is the open MX
// definition of FP4:
//   - the normal channels of a row, compacted in ascending channel order, are
//     cut into blocks of 32 entries;
//   - block scale 2^E, stored as the E8M0 byte e8 = E + 127, with
//     E = floor(log2 a) - 2 (a = the block's absolute maximum), clamped to
//     [-127, 127]; for a bf16 a this is e8 = max(exponent field of a - 2, 0);
//   - codes: E2M1 (magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6) nearest to x / 2^E,
//     ties to even, saturating, sign kept.
// x / 2^E is computed as x * 2^-E in fp32, which is exact whenever the result
// is normal; a result below 2^-126 lies far below the first rounding point
// (0.25) and becomes a signed zero code either way.  The hardware conversion
// cvt.rn.satfinite.e2m1x2.f32 does the rounding.
//
// One CTA works on one row at a time (rows strided by the grid):
//   1. the row is read with coalesced 16-byte loads and split in shared
//      memory: normal channels to `cbuf` (compacted), outlier channels to
//      `obuf` (the channel table gives every chunk of 8 channels its place);
//   2. each thread takes one chunk of 8 compacted entries: the four threads
//      of a block combine their partial maxima by shuffles, every thread
//      converts its 8 entries to one 32-bit word of codes, and the first
//      thread of every 4 blocks writes their 4 scale bytes as one word;
//   3. the compact outlier row is written from `obuf`.
// Outputs:
//   Xn  [rows, kn_pad / 2] bytes, byte j = code 2j (low nibble) | code 2j+1;
//   S   block scales in tiles of 128 rows x 4 blocks (512 bytes each, tiles
//       ordered by row band then block group): row r, block b at byte
//       ((r / 128) * (kn_pad / 128) + b / 4) * 512 + 16 (r % 32)
//       + 4 ((r % 128) / 32) + b % 4 -- the order in which tcgen05.cp moves
//       scale factors into tensor memory; rows in [rows, rows_pad) get 0;
//   Xo  [rows, no_pad] bf16 compact outlier channels.
// Padding entries (compacted positions >= kn, outlier columns >= nO) are 0.
#pragma once

#include "sq_rowquant.cuh"

namespace sqq {

constexpr int kMxThreads = 256;
constexpr int kMxLoadBatch = 4;   // row chunks loaded per thread before they are split

// Eight fp32 values -> eight E2M1 codes in one word (value i in nibble i).
__device__ __forceinline__ uint32_t e2m1x8(uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t a4,
                                           uint32_t a5, uint32_t a6, uint32_t a7)
{
    uint32_t r;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(r)
        : "f"(__uint_as_float(a0)), "f"(__uint_as_float(a1)), "f"(__uint_as_float(a2)), "f"(__uint_as_float(a3)),
          "f"(__uint_as_float(a4)), "f"(__uint_as_float(a5)), "f"(__uint_as_float(a6)), "f"(__uint_as_float(a7)));
    return r;
}

// Codes of 8 bf16 entries (one 16-byte chunk) for the block scale 2^E, given
// as the fp32 pair {2^-E, 2^-E}.
__device__ __forceinline__ uint32_t mx_codes8(const uint4 &v, uint64_t inv2)
{
    uint32_t t[8];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint64_t p = f2_mul(f2_pack(w[i] << 16, w[i] & 0xFFFF0000u), inv2);
        f2_unpack(p, t[2 * i], t[2 * i + 1]);
    }
    return e2m1x8(t[0], t[1], t[2], t[3], t[4], t[5], t[6], t[7]);
}

// Bit pattern of the largest |entry| of a chunk of 8 bf16 values.
__device__ __forceinline__ uint32_t chunk_absmax_bits(const uint4 &v)
{
    const uint32_t m = maxabs_bf16x2(maxabs_bf16x2(v.x, v.y), maxabs_bf16x2(v.z, v.w)) & 0x7FFF7FFFu;
    return max(m & 0xFFFFu, m >> 16);
}

__global__ void __launch_bounds__(kMxThreads) mx_quant_kernel(const uint16_t *__restrict__ X, int rows, int rows_pad,
                                                              int K, int64_t ldx, const uint32_t *__restrict__ chan_tab,
                                                              int nO, int kn, int kn_pad, int no_pad,
                                                              uint8_t *__restrict__ Xn, uint8_t *__restrict__ S,
                                                              uint16_t *__restrict__ Xo)
{
    sqd::pdl_launch_dependents();
    extern __shared__ uint4 mx_smem[];
    uint16_t *cbuf = reinterpret_cast<uint16_t *>(mx_smem);   // [kn_pad]
    uint16_t *obuf = cbuf + kn_pad;                          // [no_pad]; kn_pad is a multiple of 256
    const int tid = threadIdx.x;
    for (int j = kn + tid; j < kn_pad; j += kMxThreads) cbuf[j] = 0;
    for (int j = nO + tid; j < no_pad; j += kMxThreads) obuf[j] = 0;
    sqd::pdl_wait();  // X may come from, and the outputs may still be read by, the previous kernel

    const int nchunk = K / 8;
    const int ncode_chunks = kn_pad / 8;     // multiple of 32: whole warps, whole 16-lane block groups
    const int na = kn_pad / 128;             // scale tiles per 128-row band
    const int64_t code_bytes = kn_pad / 2;
    const int lane = tid & 31;

    for (int row = blockIdx.x; row < rows_pad; row += gridDim.x) {
        uint8_t *srow = S + static_cast<int64_t>(row >> 7) * na * 512 + 16 * (row & 31) + 4 * ((row & 127) >> 5);
        if (row >= rows) {   // padding row of the last band: zero scales (the same for every thread)
            for (int g = tid; g < na; g += kMxThreads) *reinterpret_cast<uint32_t *>(srow + g * 512) = 0u;
            continue;
        }
        const uint16_t *xr = X + static_cast<int64_t>(row) * ldx;

        // 1. split the row into cbuf (normal, compacted) and obuf (outliers)
        for (int c0 = tid; c0 < nchunk; c0 += kMxThreads * kMxLoadBatch) {
            uint4 v[kMxLoadBatch];
            uint32_t w[kMxLoadBatch];
#pragma unroll
            for (int i = 0; i < kMxLoadBatch; ++i) {
                const int c = c0 + i * kMxThreads;
                if (c < nchunk) {
                    v[i] = sqd::ld_nc_v4(xr + 8 * c);
                    w[i] = __ldg(chan_tab + c);
                }
            }
#pragma unroll
            for (int i = 0; i < kMxLoadBatch; ++i) {
                const int c = c0 + i * kMxThreads;
                if (c >= nchunk) break;
                const uint32_t mask = w[i] & 0xFFu, below = w[i] >> 8;
                const int nb = 8 * c - static_cast<int>(below);   // compacted position of the chunk's first normal entry
                if (mask == 0u && (nb & 7) == 0) {
                    *reinterpret_cast<uint4 *>(cbuf + nb) = v[i];
                } else {
                    const uint32_t e[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const uint16_t x = static_cast<uint16_t>(k & 1 ? e[k >> 1] >> 16 : e[k >> 1] & 0xFFFFu);
                        const int before = __popc(mask & ((1u << k) - 1u));   // outliers of the chunk before entry k
                        if ((mask >> k) & 1u) obuf[below + before] = x;
                        else cbuf[nb + k - before] = x;
                    }
                }
            }
        }
        __syncthreads();

        // 2. one chunk of 8 compacted entries per thread; 4 lanes per block
        for (int q = tid; q < ncode_chunks; q += kMxThreads) {
            const uint4 v = *reinterpret_cast<const uint4 *>(cbuf + 8 * q);
            uint32_t am = chunk_absmax_bits(v);
            am = max(am, __shfl_xor_sync(0xFFFFFFFFu, am, 1));
            am = max(am, __shfl_xor_sync(0xFFFFFFFFu, am, 2));
            const int e8 = max(static_cast<int>(am >> 7) - 2, 0);
            const uint32_t inv = static_cast<uint32_t>(254 - e8) << 23;   // 2^-E, a normal fp32 for e8 in [0, 252]
            const uint32_t codes = mx_codes8(v, f2_pack(inv, inv));
            *reinterpret_cast<uint32_t *>(Xn + static_cast<int64_t>(row) * code_bytes + 4 * q) = codes;
            // Scale bytes of the 4 blocks of this 16-lane group (lanes 0, 4, 8, 12 of the group hold them).
            const uint32_t s1 = __shfl_down_sync(0xFFFFFFFFu, static_cast<uint32_t>(e8), 4);
            const uint32_t s2 = __shfl_down_sync(0xFFFFFFFFu, static_cast<uint32_t>(e8), 8);
            const uint32_t s3 = __shfl_down_sync(0xFFFFFFFFu, static_cast<uint32_t>(e8), 12);
            if ((lane & 15) == 0)
                *reinterpret_cast<uint32_t *>(srow + (q >> 4) * 512) =
                    static_cast<uint32_t>(e8) | (s1 << 8) | (s2 << 16) | (s3 << 24);
        }

        // 3. compact outlier row
        for (int i = tid; i < no_pad / 8; i += kMxThreads)
            *reinterpret_cast<uint4 *>(Xo + static_cast<int64_t>(row) * no_pad + 8 * i) =
                *reinterpret_cast<const uint4 *>(obuf + 8 * i);
        __syncthreads();   // cbuf / obuf are refilled by the next row
    }
}

}  // namespace sqq
