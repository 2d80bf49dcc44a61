// Static outlier-channel selection from calibration statistics: the offline
// step that chooses O.  SQ-format write-up of arXiv:2512.05409, section 5
// (static strategy: mean activation per channel on calibration data) and
// section 9 (activation importance = activation times its contribution through
// the weights); OSC (arXiv:2604.12782) selects the channels offline,
// group-wise.
//
//   score[k] = mean_m |X[m,k]| * ||W[:,k]||_2            (fp64)
//   group g  = channels g*G .. g*G+G-1, score sum_j score[g*G+j]
//   O        = the channels of the nO/G best groups (ties to the lower index),
//              ascending.
//
// Each column sum is taken here in consecutive blocks of kSelBlock rows, each
// block summed in row order and the block sums added in block order, for
// parallelism.  The plain statement sums in row order; any order of adding n
// nonnegative fp64 terms lies within (n-1)*2^-53 of the exact sum, relative,
// so the scores agree with it to that bound and the selection can differ
// only between channels whose scores tie within it.  Kernel 1
// computes the block sums (one thread per channel pair and block, loads
// coalesced across channels), kernel 2 adds them in order and forms the score,
// kernel 3 the group scores, kernel 4 (one CTA) selects by an 8-pass radix
// select on the 64-bit score bits (non-negative doubles order like unsigned
// integers), breaks ties at the threshold by index and writes O.
#pragma once

#include <stdint.h>

#include "sq_device.cuh"

namespace sqs {

constexpr int kSelBlock = 256;    // rows per partial sum
constexpr int kColThreads = 256;
constexpr int kTopThreads = 1024;
constexpr int kTopKeys = 16;      // keys per thread held in registers by the top-k kernel

__device__ __forceinline__ double bf16_to_f64(uint16_t b) { return static_cast<double>(__uint_as_float(static_cast<uint32_t>(b) << 16)); }

// part[b * K + k] = sum over rows [b*kSelBlock, ...) of |A[r,k]| (square = 0) or A[r,k]^2.
// PAIR: each thread sums channels k and k+1 from one 4-byte load per row
// (K and ld even, A 4-byte aligned), so more bytes are in flight per load.
template <bool PAIR>
__global__ void __launch_bounds__(kColThreads) colsum_blocks_kernel(const uint16_t *__restrict__ A, int64_t rows,
                                                                    int K, int64_t ld, int square,
                                                                    double *__restrict__ part)
{
    sqd::pdl_launch_dependents();
    sqd::pdl_wait();
    constexpr int C = PAIR ? 2 : 1;
    const int k = (blockIdx.x * kColThreads + threadIdx.x) * C;
    const int64_t r0 = static_cast<int64_t>(blockIdx.y) * kSelBlock;
    if (k >= K) return;
    const int64_t r1 = min(rows, r0 + kSelBlock);
    double a0 = 0.0, a1 = 0.0;
    if constexpr (PAIR) {
        const uint32_t *p = reinterpret_cast<const uint32_t *>(A + r0 * ld + k);
        const int64_t step = ld / 2;
#pragma unroll 32
        for (int64_t r = r0; r < r1; ++r, p += step) {
            const uint32_t w = __ldg(p);
            const double v0 = static_cast<double>(__uint_as_float(w << 16));
            const double v1 = static_cast<double>(__uint_as_float(w & 0xFFFF0000u));
            if (square) {
                a0 = __dadd_rn(a0, __dmul_rn(v0, v0));
                a1 = __dadd_rn(a1, __dmul_rn(v1, v1));
            } else {
                a0 = __dadd_rn(a0, fabs(v0));
                a1 = __dadd_rn(a1, fabs(v1));
            }
        }
    } else {
        const uint16_t *p = A + r0 * ld + k;
#pragma unroll 16
        for (int64_t r = r0; r < r1; ++r, p += ld) {
            const double v = bf16_to_f64(__ldg(p));
            a0 = __dadd_rn(a0, square ? __dmul_rn(v, v) : fabs(v));
        }
    }
    double *out = part + static_cast<int64_t>(blockIdx.y) * K + k;
    out[0] = a0;
    if constexpr (PAIR) out[1] = a1;
}

// score[k] = (sum_b partX[b,k] / Mc) * sqrt(sum_b partW[b,k]), sums in block order.
__global__ void __launch_bounds__(kColThreads) score_kernel(const double *__restrict__ partX, int nbx, int64_t Mc,
                                                            const double *__restrict__ partW, int nbw, int K,
                                                            double *__restrict__ score)
{
    sqd::pdl_launch_dependents();
    sqd::pdl_wait();
    const int k = blockIdx.x * kColThreads + threadIdx.x;
    if (k >= K) return;
    double sx = 0.0, sw = 0.0;
    for (int b = 0; b < nbx; ++b) sx = __dadd_rn(sx, partX[static_cast<int64_t>(b) * K + k]);
    for (int b = 0; b < nbw; ++b) sw = __dadd_rn(sw, partW[static_cast<int64_t>(b) * K + k]);
    score[k] = __dmul_rn(__ddiv_rn(sx, static_cast<double>(Mc)), __dsqrt_rn(sw));
}

// gscore[g] = sum_j score[g*G + j], in channel order.
__global__ void __launch_bounds__(kColThreads) group_score_kernel(const double *__restrict__ score, int ng, int G,
                                                                  double *__restrict__ gscore)
{
    sqd::pdl_launch_dependents();
    sqd::pdl_wait();
    const int g = blockIdx.x * kColThreads + threadIdx.x;
    if (g >= ng) return;
    double t = 0.0;
    for (int j = 0; j < G; ++j) t = __dadd_rn(t, score[static_cast<int64_t>(g) * G + j]);
    gscore[g] = t;
}

// Exclusive prefix sum of one value per thread over the CTA (kTopThreads
// threads); also returns the total.
__device__ __forceinline__ int cta_exclusive_scan(int v, int *sm, int &total)
{
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    int x = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xFFFFFFFFu, x, off);
        if (lane >= off) x += y;
    }
    if (lane == 31) sm[w] = x;
    __syncthreads();
    if (w == 0) {
        int s = (lane < kTopThreads / 32) ? sm[lane] : 0;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(0xFFFFFFFFu, s, off);
            if (lane >= off) s += y;
        }
        sm[32 + lane] = s;  // inclusive prefix of warp totals
    }
    __syncthreads();
    total = sm[32 + kTopThreads / 32 - 1];
    const int before = (w > 0 ? sm[32 + w - 1] : 0) + x - v;
    __syncthreads();
    return before;
}

// One CTA: the `pick` groups with the largest gscore (ties to the lower
// index); writes O = their channels in ascending order (pick * G entries).
__global__ void __launch_bounds__(kTopThreads) select_top_kernel(const double *__restrict__ gscore, int ng, int pick,
                                                                  int G, int32_t *__restrict__ O)
{
    sqd::pdl_launch_dependents();
    sqd::pdl_wait();
    __shared__ unsigned int hist[256];
    __shared__ int scan_sm[64];
    __shared__ unsigned long long s_prefix;
    __shared__ int s_need;
    const int tid = threadIdx.x;
    const uint64_t *key = reinterpret_cast<const uint64_t *>(gscore);

    // 1. radix select, most significant byte first: the key T of the pick-th
    //    largest score, and how many keys equal to T are still to be taken.
    //    Each thread keeps its keys (i = tid + j * kTopThreads) in registers
    //    when they fit (ng <= kTopKeys * kTopThreads).
    uint64_t kreg[kTopKeys];
    const bool in_regs = ng <= kTopKeys * kTopThreads;
#pragma unroll
    for (int j = 0; j < kTopKeys; ++j) {
        const int i = tid + j * kTopThreads;
        kreg[j] = (in_regs && i < ng) ? __ldg(key + i) : 0ull;
    }
    uint64_t prefix = 0, pmask = 0;
    int need = pick;
    if (pick > 0) {
        for (int d = 7; d >= 0; --d) {
            for (int i = tid; i < 256; i += kTopThreads) hist[i] = 0u;
            __syncthreads();
            // Neighbouring scores share their high bytes, so many keys fall in
            // the same bin: lanes with equal bins add their count once.
            auto count = [&](uint64_t kv, bool valid) {
                const unsigned bin = (valid && (kv & pmask) == prefix) ? static_cast<unsigned>((kv >> (8 * d)) & 255u)
                                                                        : 256u;
                const unsigned same = __match_any_sync(0xFFFFFFFFu, bin);
                if (bin < 256u && (tid & 31) == __ffs(same) - 1) atomicAdd(&hist[bin], static_cast<unsigned>(__popc(same)));
            };
            if (in_regs) {
#pragma unroll
                for (int j = 0; j < kTopKeys; ++j) count(kreg[j], tid + j * kTopThreads < ng);
            } else {
                for (int i0 = 0; i0 < ng; i0 += kTopThreads) {
                    const int i = i0 + tid;
                    count(i < ng ? __ldg(key + i) : 0ull, i < ng);
                }
            }
            __syncthreads();
            if (tid < 32) {
                // Bins from the top: lane l holds bins 255-8l .. 248-8l.  The
                // first bin v (from 255 down) whose count from 255 to v
                // reaches `need` is the digit of T.
                int c[8], sum = 0;
#pragma unroll
                for (int b = 0; b < 8; ++b) {
                    c[b] = static_cast<int>(hist[255 - 8 * tid - b]);
                    sum += c[b];
                }
                int incl = sum;
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    const int y = __shfl_up_sync(0xFFFFFFFFu, incl, off);
                    if (tid >= off) incl += y;
                }
                const int excl = incl - sum;
                const unsigned hit = __ballot_sync(0xFFFFFFFFu, incl >= need);
                const int owner = hit ? __ffs(hit) - 1 : 31;
                if (tid == owner) {
                    int cum = excl, b = 0;
                    for (; b < 7; ++b) {
                        if (cum + c[b] >= need) break;
                        cum += c[b];
                    }
                    s_need = need - cum;
                    s_prefix = prefix | (static_cast<uint64_t>(255 - 8 * tid - b) << (8 * d));
                }
            }
            __syncthreads();
            need = s_need;
            prefix = s_prefix;
            pmask |= 0xFFull << (8 * d);
            __syncthreads();
        }
    }

    // 2. selected: key > T, or key == T among the first `need` such indices.
    //    Each thread owns a contiguous index range, so ranks follow index order.
    const int per = (ng + kTopThreads - 1) / kTopThreads;
    const int i0 = min(ng, tid * per), i1 = min(ng, i0 + per);
    int eq = 0;
    if (pick > 0)
        for (int i = i0; i < i1; ++i) eq += (__ldg(key + i) == prefix) ? 1 : 0;
    int tot;
    int eq_before = cta_exclusive_scan(eq, scan_sm, tot);
    auto chosen = [&](int i, int &eq_seen) -> bool {
        if (pick == 0) return false;
        const uint64_t kv = __ldg(key + i);
        if (kv > prefix) return true;
        if (kv == prefix) return eq_seen++ < need;
        return false;
    };
    int nsel = 0;
    {
        int seen = eq_before;
        for (int i = i0; i < i1; ++i) nsel += chosen(i, seen) ? 1 : 0;
    }
    const int pos0 = cta_exclusive_scan(nsel, scan_sm, tot);

    // 3. O: channels of the selected groups, ascending.
    int seen = eq_before, pos = pos0;
    for (int i = i0; i < i1; ++i) {
        if (chosen(i, seen)) {
            for (int c = 0; c < G; ++c) O[static_cast<int64_t>(pos) * G + c] = i * G + c;
            ++pos;
        }
    }
}

}  // namespace sqs
