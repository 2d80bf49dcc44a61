// Definitions shared by the two dual-path GEMM kernels (sq_gemm_pair.cuh for
// M > 128, sq_gemm_skinny.cuh for M <= 128).
//
// OSC (arXiv:2604.12782), abstract: inference runs a low-precision 4-bit GEMM
// path and a high-precision 16-bit branch GEMM on the compact outlier tensor,
// and fuses the two results.  Both kernels keep two tensor-memory (TMEM)
// accumulators per output tile:
//
//   acc_f (fp32)  += X_O . W_O^T          (tcgen05 kind::f16, bf16 inputs)
//   acc_i (int32) += codes_X . codes_W^T  (tcgen05 kind::i8)
//   Y = bf16_rn( (float)acc_i * s_x[m] * s_w[n] + acc_f )   (one epilogue)
//
// K-blocks.  An INT4 K-block is 128 channels: 64 packed bytes per row, 128
// int8 bytes per row once expanded.  A bf16 K-block is 64 outlier channels:
// 128 bytes per row.  Either way an operand row of one K-block is one
// 128-byte row of the 128-byte swizzle layout, so both MMA kinds read their
// tiles through the same shared-memory descriptors.
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

constexpr int ROWB = 128;       // operand bytes per row per K-block (one 128-byte swizzle row)
constexpr int PROWB = 64;       // packed INT4 bytes per row per K-block
constexpr int KB_I8 = 128;      // int8 K elements per block
constexpr int KB_BF = 64;       // bf16 K elements per block
constexpr int NUM_EXP_WARPS = 8;  // operand-producer warps of the pair kernel

// Low-path formats.  INT4: packed codes expanded to int8 (kind::i8), one
// fp32 scale per row.  FP8: E4M3 bytes (kind::f8f6f4), one fp32 scale per
// row.  MX: packed E2M1 codes (kind::mxf4) with one E8M0 scale per 32
// K-elements of each row; the tensor core applies the scales, so the low path
// and the 16-bit branch accumulate into one fp32 accumulator.
// SQF: the element-level SQ-format (sq_sqf.cuh): INT4 low part whose mask code
// -8 the expansion turns into 0, plus a precomputed fp32 high part added in
// the epilogue (GemmArgs::addend).
enum : int { kLowInt4 = 0, kLowFp8 = 1, kLowMx = 2, kLowSqf = 3 };

// Expanded INT4 word (bytes 16*c) with the bytes of code -8 (0x80) cleared:
// a byte is 0x80 exactly when bit 7 is set and bits 6..4 are clear.
__device__ __forceinline__ uint32_t clear_mask_code(uint32_t x)
{
    const uint32_t nz = ((x & 0x70707070u) + 0x70707070u) & 0x80808080u;  // bit 7: bits 6..4 not all clear
    return x ^ (x & ~nz & 0x80808080u);
}
constexpr int KB_MX = 256;        // E2M1 K elements per block (128 packed bytes per row)
constexpr int MX_SF_BYTES = 3072; // scale bytes per ring slot: 2 tiles of X rows, 4 of W rows
constexpr int MX_SFA_COL = 256;   // TMEM columns of the X-row scales (2 K-tiles x 4)
constexpr int MX_SFB_COL = 264;   // TMEM columns of the W-row scales (2 K-tiles x 8)
constexpr int MX_SF_SLOT = 24;    // pair kernel: ring slot e keeps its scales at the columns above + 24 e

// Site codes stored in the device error word by a bounded wait that ran out.
enum : unsigned {
    SITE_EXP_OP = 0x202, SITE_MMA_FULL = 0x301, SITE_MMA_ACC = 0x302, SITE_EPI = 0x401
};

struct GemmArgs {
    const float *s_x;
    const float *s_w;
    uint16_t *Y;
    int32_t *dbg_i;
    float *dbg_f;
    int M, N;
    long long ldy;
    int nkb_i;    // low-path K-blocks per tile (kn_pad / 128; MX: kn_pad / 256)
    int nkb_o;    // bf16 K-blocks per tile (no_pad / 64)
    int tiles_m, tiles_n, group_m;
    const float *addend;   // SQF: fp32 [M, N] added to the low part in place of the 16-bit branch
    int y_tma = 0;         // pair kernel: Y written by bulk tensor stores (tm_y) instead of per-lane stores
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

}  // namespace sqg
