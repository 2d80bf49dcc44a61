/*
 * sq.h -- C ABI of the dual-path sparse-quantized linear layer on B200 (sm_100a).
 *
 *   Y[m,n] = s_x[m] * s_w[n] * sum_{k not in O} q4(X)[m,k] * q4(W)[n,k]
 *          +                   sum_{k in O}     X[m,k]    * W[n,k]
 *
 * The layer follows two pages:
 *   - OSC: Hardware Efficient W4A4 Quantization via Outlier Separation in
 *     Channel Dimension (arXiv:2604.12782), abstract and technical framework:
 *     an offline step fixes the outlier channels O; online, the scattered
 *     outlier channels are coalesced into a compact dense tensor for a 16-bit
 *     branch GEMM while all other channels take a 4-bit GEMM; the two results
 *     are fused.
 *   - SQ-format (arXiv:2512.05409) write-up, section 9: symmetric quantization
 *     of the low-precision part (INT4 codes in [-7, 7]) and reordering of the
 *     weight columns by the static mask; section 5: the static mask is chosen
 *     offline so no runtime top-k is needed.
 *
 * Scales: one fp32 scale per token row of X (computed online by
 * sq_quant_gather) and one per output channel of W (computed offline by
 * sq_prepare_weights): s = max_{k not in O} |x_k| / 7 (IEEE fp32 division),
 * code = clamp(rint(x / s), -7, 7) with the fp32 quotient, ties to even;
 * a row whose normal channels are all zero gets s = 0 and zero codes.
 *
 * Conventions for every call
 *   - Memory: every buffer is allocated by the caller; no call allocates
 *     device memory.  The library's own device state is a per-device error
 *     word and the fixed SQ_NOALLOC_WS_BYTES scratch array of
 *     sq_linear_noalloc (below), both module variables that every device
 *     holds from the moment it loads the library.
 *   - Pointers named "dev" are device pointers, "host" host pointers.  All
 *     device pointers must be 16-byte aligned (SQ_ERR_MISALIGNED otherwise).
 *   - Matrices are row-major.  bf16 buffers are passed as void* holding IEEE
 *     bfloat16 bit patterns (uint16).
 *   - Asynchrony: calls enqueue work on `stream` (a cudaStream_t; NULL is the
 *     legacy default stream) and return without waiting, except
 *     sq_prepare_weights, which waits for its own work (it is an offline step).
 *     Argument errors are returned before anything is enqueued.
 *   - Errors: SQ_ERR_INVALID_ARG / SQ_ERR_MISALIGNED / SQ_ERR_UNSUPPORTED are
 *     returned synchronously; SQ_ERR_CUDA reports a failed launch or copy.
 *     A kernel whose bounded wait ran out records it in the device error word
 *     and exits cleanly; sq_check() reports it as SQ_ERR_TIMEOUT.
 *     sq_last_error_detail() returns a text for the last failing call on the
 *     calling thread.
 *
 * Storage formats (all produced by this library, all zero-padded; padding is
 * exact because zero codes and zero bf16 values add nothing):
 *   - KN = K - nO normal channels, ascending channel order; kn_pad = sq_kn_pad.
 *   - Packed INT4 part, [rows, kn_pad/2] bytes: byte j holds code 2j in its
 *     low nibble and code 2j+1 in its high nibble, 4-bit two's complement;
 *     code -8 is never produced.
 *   - Compact outlier part, [rows, no_pad] bf16: column j is channel O[j].
 *   - Channel table, [K/8] uint32 ("static mask"): word c holds
 *     (number of channels of O below 8c) << 8 | (bit e set when channel
 *     8c+e is in O).
 */
#ifndef SQ_B200_H
#define SQ_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t. */
typedef struct CUstream_st *sq_stream_t;

typedef enum {
    SQ_OK = 0,
    SQ_ERR_INVALID_ARG = 1,  /* a size, a stride or the outlier set is invalid */
    SQ_ERR_UNSUPPORTED = 2,  /* no sm_100 device, or a size beyond the limits below */
    SQ_ERR_MISALIGNED = 3,   /* a device pointer is not 16-byte aligned */
    SQ_ERR_CUDA = 4,         /* a CUDA launch or copy failed */
    SQ_ERR_TIMEOUT = 5       /* a kernel's bounded wait ran out (see sq_check) */
} sq_status;

/* Limits: 8 <= K <= 65536, K % 8 == 0, 0 <= nO <= K, N % 8 == 0, M >= 0. */
#define SQ_MAX_K 65536

const char *sq_status_string(sq_status status);
const char *sq_last_error_detail(void);

/* Layout queries (pure functions, no device access). */
int64_t sq_kn_pad(int64_t K, int64_t nO);            /* roundup(K - nO, 128) codes   */
int64_t sq_no_pad(int64_t nO);                       /* roundup(nO, 64) bf16 columns */
int64_t sq_chan_table_words(int64_t K);              /* K / 8                        */
/* Bytes of the sq_linear workspace: packed X part, s_x and compact X_O, each
 * 256-byte aligned. */
size_t sq_linear_workspace_bytes(int64_t M, int64_t K, int64_t nO);

/*
 * Offline step (SQ-format write-up sections 5 and 9; OSC "offline grouping"):
 * from the outlier channel list and the bf16 weights, build the static
 * channel table and the weight operands of both paths.
 *
 *   W        dev  bf16 [N, ldw]     weights, one row per output channel
 *   O        host int32 [nO]        strictly increasing channels in [0, K)
 *   W_N      dev  u8   [N, kn_pad/2] packed INT4 codes of the normal channels
 *   s_w      dev  f32  [N]          per-output-channel scales
 *   W_O      dev  bf16 [N, no_pad]  compact outlier columns (may be NULL if nO == 0)
 *   chan_tab dev  u32  [K/8]        static channel table
 * Waits for the stream before returning (the table is copied from host memory).
 */
sq_status sq_prepare_weights(const void *W, int64_t N, int64_t K, int64_t ldw,
                             const int32_t *O, int64_t nO,
                             void *W_N, float *s_w, void *W_O, uint32_t *chan_tab,
                             sq_stream_t stream);

/*
 * Online quantize-and-gather of the activations (OSC technical framework:
 * "structured sub-tensor extraction" of the outlier channels into a compact
 * dense tensor; the rest quantized to INT4 with a per-token scale).  One pass
 * over X; memory-bound.
 *
 *   X        dev bf16 [M, ldx]       activations, ldx >= K, ldx % 8 == 0
 *   chan_tab dev u32  [K/8]          from sq_prepare_weights
 *   X_N      dev u8   [M, kn_pad/2]  packed INT4 codes (may be NULL if kn_pad == 0)
 *   s_x      dev f32  [M]            per-token scales
 *   X_O      dev bf16 [M, no_pad]    compact outlier channels (may be NULL if nO == 0)
 */
sq_status sq_quant_gather(const void *X, int64_t M, int64_t K, int64_t ldx,
                          const uint32_t *chan_tab, int64_t nO,
                          void *X_N, float *s_x, void *X_O, sq_stream_t stream);

/*
 * Dual-path GEMM with fused epilogue (OSC abstract: 4-bit GEMM path plus a
 * 16-bit branch GEMM, results fused):
 *   acc_i[m,n] = sum_j codeX[m,j] * codeW[n,j]         (exact, int32)
 *   acc_f[m,n] = sum_j X_O[m,j] * W_O[n,j]             (fp32 accumulate)
 *   Y[m,n]     = bf16_rn( (float)acc_i * s_x[m] * s_w[n] + acc_f )
 *
 *   Y            dev bf16 [M, ldy]   ldy >= N, ldy % 8 == 0
 *   dbg_acc_i32  dev i32  [M, N]     optional (NULL): the exact integer sums
 *   dbg_acc_f32  dev f32  [M, N]     optional (NULL): the 16-bit branch sums
 * Other operands as produced by the two calls above.
 */
sq_status sq_gemm(const void *X_N, const float *s_x, const void *X_O,
                  const void *W_N, const float *s_w, const void *W_O,
                  int64_t M, int64_t N, int64_t K, int64_t nO,
                  void *Y, int64_t ldy,
                  int32_t *dbg_acc_i32, float *dbg_acc_f32, sq_stream_t stream);

/*
 * The whole online layer: sq_quant_gather into `workspace`, then sq_gemm,
 * both on `stream`.  workspace: dev, ws_bytes >= sq_linear_workspace_bytes.
 */
sq_status sq_linear(const void *X, int64_t M, int64_t K, int64_t ldx,
                    const uint32_t *chan_tab,
                    const void *W_N, const float *s_w, const void *W_O,
                    int64_t N, int64_t nO, void *Y, int64_t ldy,
                    void *workspace, size_t ws_bytes, sq_stream_t stream);

/*
 * sq_linear without a caller workspace.  (No counterpart in the papers: this
 * is a deployment convenience of this library.)
 *
 * Some callers cannot allocate device memory for the workspace sq_linear
 * needs: a plugin or inference server that hands out all device memory from
 * its own pool and forbids allocations once it has started, or a
 * latency-bound serving loop where cudaMalloc/cudaFree would synchronize the
 * device and stall other streams.  This entry point takes the same inputs and
 * outputs as sq_linear but keeps its scratch in a fixed array inside the
 * library, so it allocates nothing and calls no allocating routine.
 *
 *   - Limit: sq_linear_workspace_bytes(M, K, nO) must not exceed
 *     SQ_NOALLOC_WS_BYTES (16 MiB; e.g. M <= 4096 tokens at K = 4096, nO = 256);
 *     larger requests return SQ_ERR_UNSUPPORTED before anything is enqueued.
 *   - Every device that loads the library holds this 16 MiB until the process
 *     exits.
 *   - The first call on a device looks up the array's device address once
 *     (again only after a device reset has replaced the device's context);
 *     make that first call before any stream capture begins.
 *   - All calls share the one array and it keeps the previous call's
 *     contents.  Nothing in it has to start at zero (the quantize-and-gather
 *     kernel writes every byte the GEMM reads), but calls whose work overlaps
 *     on the GPU (different streams, or different host threads) race on it:
 *     serialize them.
 */
#define SQ_NOALLOC_WS_BYTES (16u * 1024u * 1024u)
sq_status sq_linear_noalloc(const void *X, int64_t M, int64_t K, int64_t ldx,
                            const uint32_t *chan_tab,
                            const void *W_N, const float *s_w, const void *W_O,
                            int64_t N, int64_t nO, void *Y, int64_t ldy,
                            sq_stream_t stream);

/* ------------------------------------------------------------------------
 * FP8 low path.
 *
 * OSC (arXiv:2604.12782), abstract and "technical framework": for the inputs
 * of W2 (the down projection), where outlier clustering is less pronounced,
 * the 4-bit path falls back to FP8.  These calls are the four above with the
 * normal (non-outlier) channels in FP8 E4M3 instead of INT4:
 *
 *   Y[m,n] = s_x[m] * s_w[n] * sum_{k not in O} e(X)[m,k] * e(W)[n,k]
 *          +                   sum_{k in O}     X[m,k]   * W[n,k]
 *
 *   - s = a / 448 (fp32, IEEE), a = absolute maximum over the normal
 *     channels of the row; a == 0 gives s = 0 and all-zero codes.
 *   - e(x) = the E4M3 code nearest to the fp32 quotient x / s, ties to the
 *     even code, magnitudes above 448 saturated to 448, the sign kept (a
 *     negative value that rounds to zero gives -0, byte 0x80).
 *   - Layout: W_N8 / X_N8 are u8 [rows, sq_kn_pad(K, nO)], one E4M3 byte per
 *     normal channel in ascending channel order, zero bytes past K - nO.
 *     s_w, s_x, W_O, X_O and the channel table are as for INT4.
 *   - The products run on the tensor cores as E4M3 x E4M3 with fp32
 *     accumulation (tcgen05 kind::f8f6f4); the epilogue is
 *     Y = bf16_rn(((float)acc_8 * s_x) * s_w + acc_f).
 *   - Supported for K <= 16384 (SQ_ERR_UNSUPPORTED above).
 *   - dbg_acc_8 (nullable, [M, N] fp32): the low-path accumulator.
 * Error behaviour, ownership and stream ordering are those of the INT4 calls.
 * ------------------------------------------------------------------------ */
size_t sq_linear_workspace_bytes_fp8(int64_t M, int64_t K, int64_t nO);

sq_status sq_prepare_weights_fp8(const void *W, int64_t N, int64_t K, int64_t ldw,
                                 const int32_t *O, int64_t nO,
                                 void *W_N8, float *s_w, void *W_O, uint32_t *chan_tab,
                                 sq_stream_t stream);

sq_status sq_quant_gather_fp8(const void *X, int64_t M, int64_t K, int64_t ldx,
                              const uint32_t *chan_tab, int64_t nO,
                              void *X_N8, float *s_x, void *X_O, sq_stream_t stream);

sq_status sq_gemm_fp8(const void *X_N8, const float *s_x, const void *X_O,
                      const void *W_N8, const float *s_w, const void *W_O,
                      int64_t M, int64_t N, int64_t K, int64_t nO,
                      void *Y, int64_t ldy,
                      float *dbg_acc_8, float *dbg_acc_f32, sq_stream_t stream);

sq_status sq_linear_fp8(const void *X, int64_t M, int64_t K, int64_t ldx,
                        const uint32_t *chan_tab,
                        const void *W_N8, const float *s_w, const void *W_O,
                        int64_t N, int64_t nO, void *Y, int64_t ldy,
                        void *workspace, size_t ws_bytes, sq_stream_t stream);

/* ------------------------------------------------------------------------
 * Micro-scaling FP4 (MXFP4) low path.
 *
 * OSC (arXiv:2604.12782), abstract: the channel split fits 4-bit
 * micro-scaling hardware; SQ-format write-up of arXiv:2512.05409, section 8:
 * the format also works with FP4 data.  These calls run the normal channels
 * as MXFP4 (the open MX block format: E2M1 codes, one E8M0 power-of-two scale
 * per block of 32 normal channels) and keep the 16-bit branch:
 *
 *   Y[m,n] = sum_b 2^(Ex[m,b] + Ew[n,b]) * sum_{j in block b} e(X)[m,j] * e(W)[n,j]
 *          + sum_{k in O} X[m,k] * W[n,k]
 *
 *   - Blocks: the normal channels of a row in ascending channel order, cut
 *     into blocks of 32 (the last one may be partial).
 *   - Scale: E = floor(log2 a) - 2 with a the block's absolute maximum,
 *     clamped to [-127, 127] (a == 0 gives -127); stored as the byte E + 127.
 *   - e(x) = the E2M1 code (sign bit 3; magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6)
 *     nearest to x / 2^E, ties to the even code, saturating at 6, the sign
 *     kept (-0 and negative values that round to zero give code 8).
 *   - Codes, [rows, kn_pad_mx / 2] bytes with kn_pad_mx = sq_kn_pad_mx(K, nO):
 *     byte j = code 2j (low nibble) | code 2j+1 (high nibble); zero past K - nO.
 *   - Scales, sq_mx_scale_bytes(rows, K, nO) bytes, in tiles of 128 rows x 4
 *     blocks: row r, block b at byte ((r / 128) * (kn_pad_mx / 128) + b / 4)
 *     * 512 + 16 * (r % 32) + 4 * ((r % 128) / 32) + b % 4; entries for rows
 *     past the matrix and blocks past K - nO are 0.
 *   - W_O, X_O and the channel table are as for INT4.
 *   - The products run on the tensor cores (tcgen05 kind::mxf4, block
 *     scales applied in hardware) and accumulate in fp32 together with the
 *     16-bit branch; Y = bf16_rn(accumulator).
 *   - dbg_acc (nullable, [M, N] fp32): that accumulator.
 * Error behaviour, ownership and stream ordering are those of the INT4 calls.
 * ------------------------------------------------------------------------ */
int64_t sq_kn_pad_mx(int64_t K, int64_t nO);                   /* roundup(K - nO, 256) codes */
size_t sq_mx_scale_bytes(int64_t rows, int64_t K, int64_t nO);  /* roundup(rows, 128) * kn_pad_mx / 32 */
/* Workspace of sq_linear_mx: codes, scales and compact X_O, each 256-byte aligned. */
size_t sq_linear_workspace_bytes_mx(int64_t M, int64_t K, int64_t nO);

/* W_N4 dev u8 [N, kn_pad_mx / 2]; S_W dev u8 [sq_mx_scale_bytes(N, K, nO)];
 * W_O and chan_tab as sq_prepare_weights.  Waits for its own work. */
sq_status sq_prepare_weights_mx(const void *W, int64_t N, int64_t K, int64_t ldw,
                                const int32_t *O, int64_t nO,
                                void *W_N4, void *S_W, void *W_O, uint32_t *chan_tab,
                                sq_stream_t stream);

/* X_N4 dev u8 [M, kn_pad_mx / 2]; S_X dev u8 [sq_mx_scale_bytes(M, K, nO)]. */
sq_status sq_quant_gather_mx(const void *X, int64_t M, int64_t K, int64_t ldx,
                             const uint32_t *chan_tab, int64_t nO,
                             void *X_N4, void *S_X, void *X_O, sq_stream_t stream);

sq_status sq_gemm_mx(const void *X_N4, const void *S_X, const void *X_O,
                     const void *W_N4, const void *S_W, const void *W_O,
                     int64_t M, int64_t N, int64_t K, int64_t nO,
                     void *Y, int64_t ldy, float *dbg_acc, sq_stream_t stream);

sq_status sq_linear_mx(const void *X, int64_t M, int64_t K, int64_t ldx,
                       const uint32_t *chan_tab,
                       const void *W_N4, const void *S_W, const void *W_O,
                       int64_t N, int64_t nO, void *Y, int64_t ldy,
                       void *workspace, size_t ws_bytes, sq_stream_t stream);

/* ------------------------------------------------------------------------
 * Element-level SQ-format weights (no outlier channels).
 *
 * SQ-format (arXiv:2512.05409): abstract (the sparse part is accelerated in
 * high precision, the dense low-precision part as a low-precision GEMM);
 * write-up sections 3, 7, 8, 9 (a mask value in the low-precision format
 * marks the high-precision positions; banks with a fixed sparsity; the top
 * (1-s) of every bank by importance; FP8/FP4 combinations).
 *
 *   Y[m,n] = s_x4[m] s_lo[n] sum_{k low(n)}  q4(X)[m,k] q4(W)[n,k]
 *          + s_x8[m] s_hi[n] sum_{k high(n)} e(X)[m,k]  e(W)[n,k]
 *
 *   - Banks: `bank` (4, 8 or 16) consecutive channels of a weight row; in each
 *     the `h` (1 or 2) entries of largest |w| are high, ties to the lower
 *     index (sparsity 1 - h/bank: 50 % to 93.75 %).
 *   - Low part W_N [N, K/2]: packed INT4 as for sq_prepare_weights, s_lo =
 *     (absmax over the row's low entries) / 7, mask code -8 at high positions
 *     (the GEMM reads it as 0).
 *   - High part: E4M3 codes of w / s_hi, s_hi = (absmax over the row's high
 *     entries) / 448, stored 2:4: W_H [N, K/2] (two value bytes per aligned
 *     group of 4 channels, the group's high codes in channel order, 0 in free
 *     slots) and W_E [N, K/8] metadata (group i in byte i/2, low nibble for
 *     even i; bits [1:0] and [3:2] = in-group indices of the two stored values,
 *     first < second; one high entry at p < 3 uses (p, p+1), at 3 uses (2, 3);
 *     none uses (0, 1)).
 *   - Tokens: INT4 codes over all K channels (X_N [M, K/2], s_x4 = absmax/7)
 *     and E4M3 codes over all K channels (X_8 [M, K], s_x8 = absmax/448).
 *   - GEMM: the high part runs on the 2:4 sparse tensor cores (tcgen05.mma.sp,
 *     kind::f8f6f4) into P [M, N] fp32 = s_x8 s_hi (e(X) e(W_hi)^T); the low
 *     part is the INT4 GEMM with P added before the bf16 rounding:
 *     Y = bf16_rn((float)acc_lo s_x4 s_lo + P).  dbg_acc_lo (nullable,
 *     [M, N] int32): the exact low-part sums.
 *   - Limits: K a multiple of 256 in [256, 16384]; N % 8 == 0.
 * Error behaviour, ownership and stream ordering are those of the INT4 calls.
 * ------------------------------------------------------------------------ */
/* Workspace of sq_linear_sqf: X_N, s_x4, X_8, s_x8 and P, each 256-byte aligned. */
size_t sq_linear_workspace_bytes_sqf(int64_t M, int64_t N, int64_t K);

/* W: dev bf16 [N, ldw].  Writes W_N, s_lo, W_H, W_E, s_hi and chan_tab (K/8
 * words, all zero: no outlier channels).  Waits for its own work. */
sq_status sq_prepare_weights_sqf(const void *W, int64_t N, int64_t K, int64_t ldw, int bank, int h,
                                 void *W_N, float *s_lo, void *W_H, void *W_E, float *s_hi,
                                 uint32_t *chan_tab, sq_stream_t stream);

sq_status sq_quant_gather_sqf(const void *X, int64_t M, int64_t K, int64_t ldx, const uint32_t *chan_tab,
                              void *X_N, float *s_x4, void *X_8, float *s_x8, sq_stream_t stream);

/* P: dev fp32 [M, N] scratch (the high part). */
sq_status sq_gemm_sqf(const void *X_N, const float *s_x4, const void *X_8, const float *s_x8,
                      const void *W_N, const float *s_lo, const void *W_H, const void *W_E, const float *s_hi,
                      int64_t M, int64_t N, int64_t K, void *Y, int64_t ldy, float *P,
                      int32_t *dbg_acc_lo, sq_stream_t stream);

sq_status sq_linear_sqf(const void *X, int64_t M, int64_t K, int64_t ldx, const uint32_t *chan_tab,
                        const void *W_N, const float *s_lo, const void *W_H, const void *W_E, const float *s_hi,
                        int64_t N, void *Y, int64_t ldy, void *workspace, size_t ws_bytes, sq_stream_t stream);

/* ------------------------------------------------------------------------
 * Static outlier-channel selection (the offline step that chooses O).
 *
 * SQ-format write-up of arXiv:2512.05409, section 5 (static strategy: mean
 * activation per channel on calibration data) and section 9 (activation
 * importance = activation times its contribution through the weights); OSC
 * (arXiv:2604.12782) selects the outlier channels offline, group-wise.
 *
 *   score[k] = mean_m |Xc[m,k]| * ||W[:,k]||_2   (fp64)
 *   O = the channels of the nO / group groups of `group` consecutive
 *       channels with the largest summed score, ties to the lower index,
 *       in ascending order.
 *
 * Row sums are taken in consecutive blocks of 256 rows, each block summed in
 * row order and the block sums added in block order; the result is therefore
 * reproducible bit for bit.
 *
 *   Xc        calibration activations, bf16 [Mc, ldx] (dev), row-major
 *   W         weights, bf16 [N, ldw] (dev), row-major
 *   nO, group 0 <= nO <= K, group >= 1 divides K and nO
 *   O         out: int32 [nO] (dev), ascending; feed it (copied to the host)
 *             to sq_prepare_weights / sq_prepare_weights_fp8
 *   scores    out (nullable): fp64 [K] (dev, 8-byte aligned)
 *   workspace dev, ws_bytes >= sq_select_outliers_workspace_bytes(Mc, N, K, group)
 * Asynchronous on `stream`; argument errors return SQ_ERR_INVALID_ARG before
 * any launch.
 * ------------------------------------------------------------------------ */
size_t sq_select_outliers_workspace_bytes(int64_t Mc, int64_t N, int64_t K, int64_t group);

sq_status sq_select_outliers(const void *Xc, int64_t Mc, int64_t K, int64_t ldx,
                             const void *W, int64_t N, int64_t ldw,
                             int64_t nO, int64_t group, int32_t *O, double *scores,
                             void *workspace, size_t ws_bytes, sq_stream_t stream);

/*
 * Waits for `stream`, then reports (and clears) the device error word of the
 * current device: SQ_ERR_TIMEOUT if a kernel's bounded wait ran out,
 * SQ_ERR_CUDA on a pending CUDA error, SQ_OK otherwise.
 */
sq_status sq_check(sq_stream_t stream);

/*
 * Failure-detection self test: launches one single-thread kernel that waits
 * on a barrier nothing will ever complete, with a bounded wait of about
 * `timeout_ms` milliseconds (1..10000).  The kernel records the timeout in
 * the device error word and exits; sq_check() then returns SQ_ERR_TIMEOUT
 * and the context stays usable.
 */
sq_status sq_selftest_watchdog(int timeout_ms, sq_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* SQ_B200_H */
