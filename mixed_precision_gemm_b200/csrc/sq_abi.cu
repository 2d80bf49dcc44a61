// C ABI of the dual-path sparse-quantized linear layer (declared in include/sq.h).
//
// Host side only: argument validation, layout arithmetic, TMA tensor-map
// encoding and kernel launches.  Every kernel lives in the .cuh files included
// below so that the whole library is one translation unit (one device error
// word per device).
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <cstdarg>
#include <cstdio>
#include <mutex>
#include <type_traits>
#include <string>
#include <vector>

#include "../../include/sq.h"
#include "sq_device.cuh"
#include "sq_gemm_common.cuh"
#include "sq_gemm_pair.cuh"
#include "sq_gemm_skinny.cuh"
#include "sq_mxquant.cuh"
#include "sq_rowquant.cuh"
#include "sq_rowquant_stream.cuh"
#include "sq_select.cuh"
#include "sq_sqf.cuh"

namespace {

thread_local std::string g_detail;

sq_status fail(sq_status st, const char *fmt, ...)
{
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_detail = buf;
    return st;
}

sq_status cuda_fail(cudaError_t e, const char *what)
{
    return fail(SQ_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int64_t round_up(int64_t v, int64_t m) { return (v + m - 1) / m * m; }

constexpr int kMaxDevices = 64;

struct DevInfo {
    bool ready = false;
    bool sm100 = false;
    int sms = 0;
};

DevInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

sq_status device_info(DevInfo &out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices) return fail(SQ_ERR_UNSUPPORTED, "device index %d", dev);
    std::lock_guard<std::mutex> lk(g_dev_mu);
    DevInfo &d = g_dev[dev];
    if (!d.ready) {
        int major = 0, sms = 0;
        if ((e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess)
            return cuda_fail(e, "cudaDeviceGetAttribute");
        if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
            return cuda_fail(e, "cudaDeviceGetAttribute");
        d.sm100 = (major == 10);
        d.sms = sms;
        d.ready = true;
    }
    out = d;
    if (!out.sm100) return fail(SQ_ERR_UNSUPPORTED, "this library needs an sm_100 (B200-class) device");
    return SQ_OK;
}

// ---------------------------------------------------------------- current context
// Settings made on a device (a kernel's shared-memory opt-in, the address of
// a module variable) belong to the device's current context; a device reset
// (cudaDeviceReset) ends it and the next call runs in a new one.  The caches
// below are therefore keyed by the context handle, read from the driver.
typedef CUresult (*PFN_ctx_get_current)(CUcontext *);
PFN_ctx_get_current g_ctx_get = nullptr;
std::once_flag g_ctx_once;

sq_status current_context(CUcontext &ctx)
{
    std::call_once(g_ctx_once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 4000, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_ctx_get = reinterpret_cast<PFN_ctx_get_current>(p);
    });
    if (!g_ctx_get) return fail(SQ_ERR_CUDA, "cuCtxGetCurrent is not available from the driver");
    ctx = nullptr;
    if (g_ctx_get(&ctx) != CUDA_SUCCESS) return fail(SQ_ERR_CUDA, "cuCtxGetCurrent failed");
    return SQ_OK;   // NULL when the runtime has not made a context current on this thread yet
}

// ---------------------------------------------------------------- per-kernel launch set-up
// The dynamic shared-memory opt-in of each kernel (a per-function limit:
// only ever raised, to the largest size launched so far) and its occupancy
// per launch shape are set and queried once per device and context; later
// calls (including calls made while a stream is captured into a CUDA graph)
// only look them up.
struct KernelLimit {
    const void *fn;
    int dev;
    CUcontext ctx;
    size_t smem_max;
};
struct KernelSetup {
    const void *fn;
    int dev;
    size_t smem;
    int threads;
    int per_sm;
};
std::vector<KernelLimit> g_limits;
std::vector<KernelSetup> g_setups;
std::mutex g_setup_mu;

sq_status kernel_setup(const void *fn, int threads, size_t smem, int &per_sm, const char *what)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    CUcontext ctx;
    const sq_status cst = current_context(ctx);
    if (cst != SQ_OK) return cst;
    std::lock_guard<std::mutex> lk(g_setup_mu);
    KernelLimit *lim = nullptr;
    for (KernelLimit &l : g_limits)
        if (l.fn == fn && l.dev == dev) lim = &l;
    if (lim && ctx && lim->ctx != ctx) *lim = {fn, dev, ctx, 48 * 1024};   // a new context: the opt-in is gone
    if (!lim) {
        g_limits.push_back({fn, dev, ctx, 48 * 1024});
        lim = &g_limits.back();
    }
    if (smem > lim->smem_max) {
        if ((e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem))) !=
            cudaSuccess)
            return cuda_fail(e, what);
        lim->smem_max = smem;
    }
    for (const KernelSetup &k : g_setups)
        if (k.fn == fn && k.dev == dev && k.smem == smem && k.threads == threads) {
            per_sm = k.per_sm;
            return SQ_OK;
        }
    if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, threads, smem)) != cudaSuccess)
        return cuda_fail(e, what);
    if (per_sm < 1) return fail(SQ_ERR_UNSUPPORTED, "%s: kernel does not fit on an SM", what);
    g_setups.push_back({fn, dev, smem, threads, per_sm});
    return SQ_OK;
}

// ---------------------------------------------------------------- tensor maps
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

sq_status get_encode(PFN_cuTensorMapEncodeTiled_v12000 &fn)
{
    std::call_once(g_encode_once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    fn = g_encode;
    if (!fn) return fail(SQ_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
    return SQ_OK;
}

// 2-D row-major tensor: `inner` elements per row (contiguous), `outer` rows,
// rows `row_bytes` apart; box of box_inner x box_outer elements.
sq_status make_map(CUtensorMap &map, const void *base, CUtensorMapDataType dt, uint64_t inner,
                   uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
                   CUtensorMapSwizzle swz)
{
    PFN_cuTensorMapEncodeTiled_v12000 enc;
    sq_status st = get_encode(enc);
    if (st != SQ_OK) return st;
    cuuint64_t dims[2] = {inner, outer};
    cuuint64_t strides[1] = {row_bytes};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(&map, dt, 2, const_cast<void *>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(SQ_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
    return SQ_OK;
}

// ---------------------------------------------------------------- launches
// Every kernel goes out with programmatic stream serialization: it may start
// its set-up while the previous kernel in the stream finishes, and waits for
// it (griddepcontrol.wait) before touching memory that kernel may own.
// cluster_x > 0 also sets the cluster shape (cluster_x, 1, 1).
template <typename... KArgs, typename... Args>
cudaError_t launch_k(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                     unsigned cluster_x, Args &&...args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    unsigned n = 0;
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
    if (cluster_x > 0) {
        attr[n].id = cudaLaunchAttributeClusterDimension;
        attr[n].val.clusterDim.x = cluster_x;
        attr[n].val.clusterDim.y = 1;
        attr[n].val.clusterDim.z = 1;
        ++n;
    }
    cfg.attrs = attr;
    cfg.numAttrs = n;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// ---------------------------------------------------------------- row quantizer
template <int G, int CPT>
sq_status launch_rowquant_t(const DevInfo &di, const uint16_t *src, int64_t rows, int K, int64_t ld,
                            const uint32_t *tab, int nO, int kn_pad, int no_pad, uint8_t *dn, float *ds,
                            uint16_t *dout, cudaStream_t stream)
{
    auto kern = sqq::rowquant_kernel<G, CPT>;
    constexpr int T = 32 * G;
    // constant tables, outlier channel list, two alternating packed code rows
    const size_t smem = sizeof(sqq::QuantTables) + ((2u * static_cast<size_t>(no_pad) + 15u) & ~size_t(15)) +
                        2u * (static_cast<size_t>(kn_pad / 2) + 16u);
    int per_sm = 0;
    sq_status st = kernel_setup(reinterpret_cast<const void *>(kern), T, smem, per_sm, "rowquant set-up");
    if (st != SQ_OK) return st;
    const int64_t grid = std::min<int64_t>(rows, static_cast<int64_t>(per_sm) * di.sms);
    cudaError_t e = launch_k(kern, dim3(static_cast<unsigned>(grid)), dim3(T), smem, stream, 0u, src, rows, K, ld, tab,
                             nO, kn_pad, no_pad, dn, ds, dout);
    if (e != cudaSuccess) return cuda_fail(e, "rowquant launch");
    return SQ_OK;
}

template <int G>
sq_status launch_rowquant_g(const DevInfo &di, const uint16_t *src, int64_t rows, int K, int64_t ld,
                            const uint32_t *tab, int nO, int kn_pad, int no_pad, uint8_t *dn, float *ds,
                            uint16_t *dout, cudaStream_t stream)
{
    const int cpt = (K / 8 + 32 * G - 1) / (32 * G);  // chunks of 8 channels per thread
    if (cpt <= 1) return launch_rowquant_t<G, 1>(di, src, rows, K, ld, tab, nO, kn_pad, no_pad, dn, ds, dout, stream);
    if (cpt <= 2) return launch_rowquant_t<G, 2>(di, src, rows, K, ld, tab, nO, kn_pad, no_pad, dn, ds, dout, stream);
    if (cpt <= 4) return launch_rowquant_t<G, 4>(di, src, rows, K, ld, tab, nO, kn_pad, no_pad, dn, ds, dout, stream);
    if (cpt <= 8) return launch_rowquant_t<G, 8>(di, src, rows, K, ld, tab, nO, kn_pad, no_pad, dn, ds, dout, stream);
    return launch_rowquant_t<G, 16>(di, src, rows, K, ld, tab, nO, kn_pad, no_pad, dn, ds, dout, stream);
}

// Rows streamed through shared memory (K <= 16384): as many consumer groups
// of G warps as the shared memory holds (two row slots each), one CTA per SM.
template <int G, bool FP8>
sq_status launch_rowquant_stream(const DevInfo &di, const uint16_t *src, int64_t rows, int K, int64_t ld,
                                 const uint32_t *tab, int nO, int kn_pad, int no_pad, uint8_t *dn, float *ds,
                                 uint16_t *dout, cudaStream_t stream)
{
    constexpr int kSmemLimit = 232448 - 1024;
    // Two row slots per group (the next row in flight while one is read) and as
    // many groups as fit: more groups measured faster than deeper slots, the
    // kernel being bound by instruction issue rather than by memory latency.
    const int spg = 2;
    int ngrp = sqq::stream_max_groups(G);
    while (ngrp > 1 && sqq::StreamLayout(K, kn_pad, no_pad, ngrp, spg, FP8).bytes > kSmemLimit) --ngrp;
    const size_t smem = static_cast<size_t>(sqq::StreamLayout(K, kn_pad, no_pad, ngrp, spg, FP8).bytes);
    if (smem > static_cast<size_t>(kSmemLimit))
        return fail(SQ_ERR_UNSUPPORTED, "quantize-gather: K=%d, nO=%d do not fit in shared memory", K, nO);
    auto kern = sqq::rowquant_stream_kernel<G, FP8>;
    const int threads = 32 * (1 + ngrp * G);
    int per_sm = 0;
    sq_status st = kernel_setup(reinterpret_cast<const void *>(kern), threads, smem, per_sm, "rowquant stream set-up");
    if (st != SQ_OK) return st;
    const int64_t grid = std::min<int64_t>(rows, static_cast<int64_t>(per_sm) * di.sms);
    cudaError_t e = launch_k(kern, dim3(static_cast<unsigned>(grid)), dim3(threads), smem, stream, 0u, src, rows, K, ld,
                             tab, nO, kn_pad, no_pad, dn, ds, dout, ngrp, spg);
    if (e != cudaSuccess) return cuda_fail(e, "rowquant stream launch");
    return SQ_OK;
}

template <bool FP8>
sq_status launch_rowquant_streamed(const DevInfo &di, const uint16_t *src, int64_t rows, int k, int64_t ld,
                                   const uint32_t *tab, int no, int kn_pad, int no_pad, uint8_t *dn, float *ds,
                                   uint16_t *dout, cudaStream_t stream)
{
    // up to 2048 channels per warp (8 chunks of 8 per thread); narrow rows
    // take more warps per row, so that each SM runs more warps
    if (k <= 1024) return launch_rowquant_stream<1, FP8>(di, src, rows, k, ld, tab, no, kn_pad, no_pad, dn, ds, dout, stream);
    if (k <= 2048) return launch_rowquant_stream<2, FP8>(di, src, rows, k, ld, tab, no, kn_pad, no_pad, dn, ds, dout, stream);
    if (k <= 8192) return launch_rowquant_stream<4, FP8>(di, src, rows, k, ld, tab, no, kn_pad, no_pad, dn, ds, dout, stream);
    return launch_rowquant_stream<8, FP8>(di, src, rows, k, ld, tab, no, kn_pad, no_pad, dn, ds, dout, stream);
}

// fp8: E4M3 codes (the FP8 low path) instead of packed INT4 codes.
sq_status launch_rowquant(const uint16_t *src, int64_t rows, int64_t K, int64_t ld, const uint32_t *tab,
                          int64_t nO, uint8_t *dn, float *ds, uint16_t *dout, cudaStream_t stream, bool fp8 = false)
{
    if (rows == 0) return SQ_OK;
    DevInfo di;
    sq_status st = device_info(di);
    if (st != SQ_OK) return st;
    const int kn_pad = static_cast<int>(sq_kn_pad(K, nO));
    const int no_pad = static_cast<int>(sq_no_pad(nO));
    const int k = static_cast<int>(K), no = static_cast<int>(nO);
    if (fp8) {
        if (K > sqq::kStreamMaxK)
            return fail(SQ_ERR_UNSUPPORTED, "the FP8 low path supports K <= %d (K=%lld)", sqq::kStreamMaxK, (long long)K);
        return launch_rowquant_streamed<true>(di, src, rows, k, ld, tab, no, kn_pad, no_pad, dn, ds, dout, stream);
    }
    if (K <= sqq::kStreamMaxK)
        return launch_rowquant_streamed<false>(di, src, rows, k, ld, tab, no, kn_pad, no_pad, dn, ds, dout, stream);
    // Wider rows stay in registers: a group of 16 warps per row, 8 or 16
    // chunks of 8 channels per thread.
    return launch_rowquant_g<16>(di, src, rows, k, ld, tab, no, kn_pad, no_pad, dn, ds, dout, stream);
}

// ---------------------------------------------------------------- GEMM
// Raster band height (in M-tiles).  Tiles are handed out M-fastest within a
// band, so the CTAs at work together share a band of X rows and a few W
// tiles.  The band takes as many M-tiles as keep its X operands within about
// 48 MB of L2: when all of X fits, each W tile is fetched from HBM once.
int raster_group(int tiles_m, int tile_rows, int64_t kn_pad, int64_t no_pad)
{
    const int64_t band_bytes = static_cast<int64_t>(tile_rows) * (kn_pad / 2 + 2 * no_pad);
    int64_t g = band_bytes > 0 ? (48ll << 20) / band_bytes : tiles_m;
    if (g < 1) g = 1;
    if (g > tiles_m) g = tiles_m;
    return static_cast<int>(g);
}

// Pair (cta_group::2) kernel: 256 x 256 tiles over clusters of two CTAs.
// kLowFp8: E4M3 low path (kn_pad bytes per row, tiles loaded straight into
// the operand ring with the 128-byte swizzle).  kLowMx: packed E2M1 (kn_pad /
// 2 bytes per row, kn_pad = sq_kn_pad_mx, 128-byte boxes of 256 codes, also
// straight into the ring) plus the tiled E8M0 scales S_X / S_W (passed in
// place of s_x / s_w), read as rows of 128 bytes, 8 rows (two tiles) per box.
// kLowInt4: packed INT4 (kn_pad / 2 bytes per row, 64-byte staging boxes).
template <class C, int LOW>
sq_status launch_gemm_pair_t(const DevInfo &di, const void *X_N, const float *s_x, const void *X_O, const void *W_N,
                             const float *s_w, const void *W_O, int64_t M, int64_t N, int64_t K, int64_t nO, void *Y,
                             int64_t ldy, int32_t *dbg_i, float *dbg_f, cudaStream_t stream,
                             const float *addend = nullptr)
{
    constexpr bool FP8 = LOW == sqg::kLowFp8, MX = LOW == sqg::kLowMx;
    const int64_t kn_pad = MX ? sq_kn_pad_mx(K, nO) : sq_kn_pad(K, nO), no_pad = sq_no_pad(nO);
    CUtensorMap m_xo{}, m_wo{}, m_xn{}, m_wn{}, m_sx{}, m_sw{};
    sq_status st;
    if (kn_pad > 0) {
        const int64_t rb = FP8 ? kn_pad : kn_pad / 2;
        const uint32_t box = (FP8 || MX) ? 128u : static_cast<uint32_t>(sqg::PROWB);
        const CUtensorMapSwizzle swz = (FP8 || MX) ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE;
        if ((st = make_map(m_xn, X_N, CU_TENSOR_MAP_DATA_TYPE_UINT8, rb, M, rb, box, 128, swz)) != SQ_OK) return st;
        if ((st = make_map(m_wn, W_N, CU_TENSOR_MAP_DATA_TYPE_UINT8, rb, N, rb, box, 128, swz)) != SQ_OK) return st;
        if (MX) {
            const uint64_t sx_rows = static_cast<uint64_t>(sq_mx_scale_bytes(M, K, nO) / 128);
            const uint64_t sw_rows = static_cast<uint64_t>(sq_mx_scale_bytes(N, K, nO) / 128);
            if ((st = make_map(m_sx, s_x, CU_TENSOR_MAP_DATA_TYPE_UINT8, 128, sx_rows, 128, 128, 8,
                               CU_TENSOR_MAP_SWIZZLE_NONE)) != SQ_OK)
                return st;
            if ((st = make_map(m_sw, s_w, CU_TENSOR_MAP_DATA_TYPE_UINT8, 128, sw_rows, 128, 128, 8,
                               CU_TENSOR_MAP_SWIZZLE_NONE)) != SQ_OK)
                return st;
        }
    }
    if (no_pad > 0) {
        if ((st = make_map(m_xo, X_O, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, no_pad, M, no_pad * 2, sqg::KB_BF, 128,
                           CU_TENSOR_MAP_SWIZZLE_128B)) != SQ_OK)
            return st;
        if ((st = make_map(m_wo, W_O, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, no_pad, N, no_pad * 2, sqg::KB_BF, 128,
                           CU_TENSOR_MAP_SWIZZLE_128B)) != SQ_OK)
            return st;
    }
    sqg::GemmArgs a;
    a.s_x = s_x;
    a.s_w = s_w;
    a.Y = static_cast<uint16_t *>(Y);
    a.dbg_i = dbg_i;
    a.dbg_f = dbg_f;
    a.addend = addend;
    a.M = static_cast<int>(M);
    a.N = static_cast<int>(N);
    a.ldy = ldy;
    a.nkb_i = static_cast<int>(kn_pad / (MX ? sqg::KB_MX : sqg::KB_I8));
    a.nkb_o = static_cast<int>(no_pad / sqg::KB_BF);
    if (MX) a.s_x = a.s_w = nullptr;
    a.tiles_m = static_cast<int>((M + sqg::PAIR_BM - 1) / sqg::PAIR_BM);
    a.tiles_n = static_cast<int>((N + sqg::PAIR_BN - 1) / sqg::PAIR_BN);
    a.group_m = raster_group(a.tiles_m, sqg::PAIR_BM, kn_pad, no_pad);
    const int64_t ntiles = static_cast<int64_t>(a.tiles_m) * a.tiles_n;
    const int64_t clusters = std::min<int64_t>(ntiles, di.sms / 2);
    // Y by bulk tensor stores of 16-column x 32-row boxes (Y is 16-byte aligned and
    // ldy a multiple of 8, so its rows are 16-byte aligned).
    CUtensorMap m_y{};
    if (C::YB > 0 && aligned16(Y) && ldy % 8 == 0) {
        if ((st = make_map(m_y, Y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, static_cast<uint64_t>(N), static_cast<uint64_t>(M),
                           static_cast<uint64_t>(ldy) * 2, 16, 32, CU_TENSOR_MAP_SWIZZLE_NONE)) != SQ_OK)
            return st;
        a.y_tma = 1;
    }
    const bool dbg = dbg_i || dbg_f;
    auto kern = dbg ? sqg::dual_gemm_pair_kernel<C, true, LOW> : sqg::dual_gemm_pair_kernel<C, false, LOW>;
    int per_sm = 0;
    if ((st = kernel_setup(reinterpret_cast<const void *>(kern), sqg::PAIR_THREADS, C::SMEM_BYTES, per_sm, "gemm pair set-up")) != SQ_OK)
        return st;
    cudaError_t e;
    if ((e = launch_k(kern, dim3(static_cast<unsigned>(2 * clusters)), dim3(sqg::PAIR_THREADS), C::SMEM_BYTES, stream, 0u,
                      m_xo, m_wo, m_xn, m_wn, m_sx, m_sw, m_y, a)) != cudaSuccess)
        return cuda_fail(e, "gemm pair launch");
    return SQ_OK;
}

// Swapped-operand split-K kernel for M <= 128: tiles of 128 W rows x MP
// tokens; the K-blocks of each tile are spread over a cluster of S CTAs.
// kLowMx passes the tiled block scales S_X / S_W in place of s_x / s_w.
template <class C, int LOW>
sq_status launch_gemm_skinny_t(const DevInfo &di, const void *X_N, const float *s_x, const void *X_O,
                               const void *W_N, const float *s_w, const void *W_O, int64_t M, int64_t N, int64_t K,
                               int64_t nO, void *Y, int64_t ldy, int32_t *dbg_i, float *dbg_f, cudaStream_t stream,
                               const float *addend = nullptr)
{
    constexpr bool FP8 = LOW == sqg::kLowFp8, MX = LOW == sqg::kLowMx;
    const int64_t kn_pad = MX ? sq_kn_pad_mx(K, nO) : sq_kn_pad(K, nO), no_pad = sq_no_pad(nO);
    CUtensorMap m_xo{}, m_wo{}, m_xn{}, m_wn{}, m_sx{}, m_sw{};
    sq_status st;
    if (kn_pad > 0) {
        // 128-byte boxes (two INT4 K-blocks, one E4M3 K-block or one E2M1 K-block) with the 128-byte swizzle.
        const int64_t rb = FP8 ? kn_pad : kn_pad / 2;
        if ((st = make_map(m_xn, X_N, CU_TENSOR_MAP_DATA_TYPE_UINT8, rb, M, rb, 128, C::MP,
                           CU_TENSOR_MAP_SWIZZLE_128B)) != SQ_OK)
            return st;
        if ((st = make_map(m_wn, W_N, CU_TENSOR_MAP_DATA_TYPE_UINT8, rb, N, rb, 128, 128,
                           CU_TENSOR_MAP_SWIZZLE_128B)) != SQ_OK)
            return st;
        if (MX) {
            const uint64_t sx_rows = static_cast<uint64_t>(sq_mx_scale_bytes(M, K, nO) / 128);
            const uint64_t sw_rows = static_cast<uint64_t>(sq_mx_scale_bytes(N, K, nO) / 128);
            if ((st = make_map(m_sx, s_x, CU_TENSOR_MAP_DATA_TYPE_UINT8, 128, sx_rows, 128, 128, 8,
                               CU_TENSOR_MAP_SWIZZLE_NONE)) != SQ_OK)
                return st;
            if ((st = make_map(m_sw, s_w, CU_TENSOR_MAP_DATA_TYPE_UINT8, 128, sw_rows, 128, 128, 8,
                               CU_TENSOR_MAP_SWIZZLE_NONE)) != SQ_OK)
                return st;
        }
    }
    if (no_pad > 0) {
        if ((st = make_map(m_xo, X_O, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, no_pad, M, no_pad * 2, sqg::KB_BF, C::MP,
                           CU_TENSOR_MAP_SWIZZLE_128B)) != SQ_OK)
            return st;
        if ((st = make_map(m_wo, W_O, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, no_pad, N, no_pad * 2, sqg::KB_BF, 128,
                           CU_TENSOR_MAP_SWIZZLE_128B)) != SQ_OK)
            return st;
    }
    sqg::SkinnyArgs a;
    a.s_x = s_x;
    a.s_w = s_w;
    a.Y = static_cast<uint16_t *>(Y);
    a.dbg_i = dbg_i;
    a.dbg_f = dbg_f;
    a.addend = addend;
    a.M = static_cast<int>(M);
    a.N = static_cast<int>(N);
    a.ldy = ldy;
    a.nkb_i = static_cast<int>(kn_pad / (MX ? sqg::KB_MX : sqg::KB_I8));
    a.nkb_o = static_cast<int>(no_pad / sqg::KB_BF);
    if (MX) a.s_x = a.s_w = nullptr;
    const int64_t tiles_n = (N + 127) / 128;
    // As many K ranges per W tile as fill the SMs once, at most 8 (portable
    // cluster size) and at most half the tile's byte count in 64-byte units,
    // so that every range holds at least one K-block.
    const int cost = (MX ? 2 : 1) * a.nkb_i + 2 * a.nkb_o;
    int64_t S = tiles_n >= di.sms ? 1 : di.sms / tiles_n;
    S = std::min<int64_t>(S, sqg::SK_MAX_SPLITS);
    S = std::min<int64_t>(S, std::max(1, cost / 2));
    S = std::max<int64_t>(S, 1);
    a.splits = static_cast<int>(S);
    const bool dbg = dbg_i || dbg_f;
    auto kern = dbg ? sqg::dual_gemm_skinny_kernel<C, true, LOW> : sqg::dual_gemm_skinny_kernel<C, false, LOW>;
    int per_sm = 0;
    if ((st = kernel_setup(reinterpret_cast<const void *>(kern), sqg::SK_THREADS, C::SMEM_BYTES, per_sm, "gemm skinny set-up")) != SQ_OK)
        return st;
    cudaError_t e;
    if ((e = launch_k(kern, dim3(static_cast<unsigned>(tiles_n * S)), dim3(sqg::SK_THREADS), C::SMEM_BYTES, stream,
                      static_cast<unsigned>(S), m_xo, m_wo, m_xn, m_wn, m_sx, m_sw, a)) != cudaSuccess)
        return cuda_fail(e, "gemm skinny launch");
    return SQ_OK;
}

using CfgPair = sqg::CfgPair<4, 4, 2>;     // INT4: per-lane Y stores (bulk stores measured 1.5-3 % slower)
using CfgPairSqf = sqg::CfgPair<4, 4, 2, 0, 2>;  // SQ-format low part: Y by bulk tensor stores
using CfgPairF8 = sqg::CfgPair<6, 0, 2, 0, 2>;  // E4M3 tiles need no staging ring: a deeper operand ring instead
using CfgPairMx = sqg::CfgPair<6, 0, 2, sqg::MX_SF_BYTES, 1>;  // E2M1 tiles plus their block scales; one Y box per warp
// INT4 stages carry two K-blocks.  The W codes go to tensor memory; the
// operand ring (six slots: the expansion runs up to three stages ahead of the
// MMAs) holds only the token rows, which leaves room for deeper staging rings.
using CfgSk16 = sqg::CfgSkinny<16, 10, 6, 0, true>;
using CfgSk32 = sqg::CfgSkinny<32, 9, 6, 0, true>;
using CfgSk64 = sqg::CfgSkinny<64, 7, 6, 0, true>;
using CfgSk128 = sqg::CfgSkinny<128, 3, 6, 0, true>;
// E4M3 stages are read by the MMA in place: a deeper staging ring instead.
using CfgSk16F8 = sqg::CfgSkinny<16, 8, 3>;
using CfgSk32F8 = sqg::CfgSkinny<32, 7, 3>;
using CfgSk64F8 = sqg::CfgSkinny<64, 6, 2>;
using CfgSk128F8 = sqg::CfgSkinny<128, 4, 2>;
// MX: no operand ring (stages are read in place), a deeper staging ring with 2 KB of scales per stage.
using CfgSk16Mx = sqg::CfgSkinny<16, 10, 0, 2048>;
using CfgSk32Mx = sqg::CfgSkinny<32, 9, 0, 2048>;
using CfgSk64Mx = sqg::CfgSkinny<64, 8, 0, 2048>;
using CfgSk128Mx = sqg::CfgSkinny<128, 6, 0, 2048>;


template <bool FP8>
sq_status gemm_dispatch(const DevInfo &di, const void *X_N, const float *s_x, const void *X_O, const void *W_N,
                        const float *s_w, const void *W_O, int64_t M, int64_t N, int64_t K, int64_t nO, void *Y,
                        int64_t ldy, int32_t *dbg_i, float *dbg_f, cudaStream_t stream)
{
    using Pair = typename std::conditional<FP8, CfgPairF8, CfgPair>::type;
    if (M > 128)
        return launch_gemm_pair_t<Pair, FP8 ? sqg::kLowFp8 : sqg::kLowInt4>(di, X_N, s_x, X_O, W_N, s_w, W_O, M, N, K, nO, Y, ldy, dbg_i, dbg_f, stream);
    if (M <= 16)
        return launch_gemm_skinny_t<typename std::conditional<FP8, CfgSk16F8, CfgSk16>::type, FP8 ? sqg::kLowFp8 : sqg::kLowInt4>(di, X_N, s_x, X_O, W_N, s_w, W_O, M, N, K, nO, Y, ldy, dbg_i, dbg_f, stream);
    if (M <= 32)
        return launch_gemm_skinny_t<typename std::conditional<FP8, CfgSk32F8, CfgSk32>::type, FP8 ? sqg::kLowFp8 : sqg::kLowInt4>(di, X_N, s_x, X_O, W_N, s_w, W_O, M, N, K, nO, Y, ldy, dbg_i, dbg_f, stream);
    if (M <= 64)
        return launch_gemm_skinny_t<typename std::conditional<FP8, CfgSk64F8, CfgSk64>::type, FP8 ? sqg::kLowFp8 : sqg::kLowInt4>(di, X_N, s_x, X_O, W_N, s_w, W_O, M, N, K, nO, Y, ldy, dbg_i, dbg_f, stream);
    return launch_gemm_skinny_t<typename std::conditional<FP8, CfgSk128F8, CfgSk128>::type, FP8 ? sqg::kLowFp8 : sqg::kLowInt4>(di, X_N, s_x, X_O, W_N, s_w, W_O, M, N, K, nO, Y, ldy, dbg_i, dbg_f, stream);
}

sq_status gemm_impl(const void *X_N, const float *s_x, const void *X_O, const void *W_N, const float *s_w,
                    const void *W_O, int64_t M, int64_t N, int64_t K, int64_t nO, void *Y, int64_t ldy,
                    int32_t *dbg_i, float *dbg_f, cudaStream_t stream, bool fp8)
{
    if (M == 0 || N == 0) return SQ_OK;
    DevInfo di;
    sq_status st = device_info(di);
    if (st != SQ_OK) return st;
    return fp8 ? gemm_dispatch<true>(di, X_N, s_x, X_O, W_N, s_w, W_O, M, N, K, nO, Y, ldy, dbg_i, dbg_f, stream)
               : gemm_dispatch<false>(di, X_N, s_x, X_O, W_N, s_w, W_O, M, N, K, nO, Y, ldy, dbg_i, dbg_f, stream);
}

// ---------------------------------------------------------------- validation
sq_status check_K_nO(int64_t K, int64_t nO)
{
    if (K < 8 || K > SQ_MAX_K || K % 8 != 0)
        return fail(SQ_ERR_INVALID_ARG, "K=%lld must be a multiple of 8 in [8, %d]", (long long)K, SQ_MAX_K);
    if (nO < 0 || nO > K) return fail(SQ_ERR_INVALID_ARG, "nO=%lld must lie in [0, K]", (long long)nO);
    return SQ_OK;
}

sq_status check_ptr(const void *p, bool needed, const char *name)
{
    if (!needed) return SQ_OK;
    if (!p) return fail(SQ_ERR_INVALID_ARG, "%s is NULL", name);
    if (!aligned16(p)) return fail(SQ_ERR_MISALIGNED, "%s is not 16-byte aligned", name);
    return SQ_OK;
}

#define SQ_TRY(expr)                 \
    do {                             \
        sq_status st_ = (expr);      \
        if (st_ != SQ_OK) return st_; \
    } while (0)

sq_status quant_gather_impl(const void *X, int64_t M, int64_t K, int64_t ldx, const uint32_t *chan_tab, int64_t nO,
                            void *X_N, float *s_x, void *X_O, cudaStream_t stream, bool fp8 = false)
{
    SQ_TRY(check_K_nO(K, nO));
    if (M < 0) return fail(SQ_ERR_INVALID_ARG, "M < 0");
    if (ldx < K || ldx % 8 != 0) return fail(SQ_ERR_INVALID_ARG, "ldx must be >= K and a multiple of 8");
    if (M == 0) return SQ_OK;
    const int64_t kn_pad = sq_kn_pad(K, nO);
    SQ_TRY(check_ptr(X, true, "X"));
    SQ_TRY(check_ptr(chan_tab, true, "chan_tab"));
    SQ_TRY(check_ptr(X_N, kn_pad > 0, "X_N"));
    SQ_TRY(check_ptr(s_x, true, "s_x"));
    SQ_TRY(check_ptr(X_O, nO > 0, "X_O"));
    return launch_rowquant(static_cast<const uint16_t *>(X), M, K, ldx, chan_tab, nO, static_cast<uint8_t *>(X_N), s_x,
                           static_cast<uint16_t *>(X_O), stream, fp8);
}

sq_status gemm_checked(const void *X_N, const float *s_x, const void *X_O, const void *W_N, const float *s_w,
                       const void *W_O, int64_t M, int64_t N, int64_t K, int64_t nO, void *Y, int64_t ldy,
                       int32_t *dbg_i, float *dbg_f, cudaStream_t stream, bool fp8 = false)
{
    if (fp8 && K > sqq::kStreamMaxK)
        return fail(SQ_ERR_UNSUPPORTED, "the FP8 low path supports K <= %d (K=%lld)", sqq::kStreamMaxK, (long long)K);
    SQ_TRY(check_K_nO(K, nO));
    if (M < 0 || M > (1ll << 30)) return fail(SQ_ERR_INVALID_ARG, "M out of range");
    if (N < 0 || N % 8 != 0 || N > (1ll << 30)) return fail(SQ_ERR_INVALID_ARG, "N must be a non-negative multiple of 8");
    if (ldy < N || ldy % 8 != 0) return fail(SQ_ERR_INVALID_ARG, "ldy must be >= N and a multiple of 8");
    if (M == 0 || N == 0) return SQ_OK;
    const int64_t kn_pad = sq_kn_pad(K, nO);
    SQ_TRY(check_ptr(X_N, kn_pad > 0, "X_N"));
    SQ_TRY(check_ptr(W_N, kn_pad > 0, "W_N"));
    SQ_TRY(check_ptr(X_O, nO > 0, "X_O"));
    SQ_TRY(check_ptr(W_O, nO > 0, "W_O"));
    SQ_TRY(check_ptr(s_x, true, "s_x"));
    SQ_TRY(check_ptr(s_w, true, "s_w"));
    SQ_TRY(check_ptr(Y, true, "Y"));
    if (dbg_i && !aligned16(dbg_i)) return fail(SQ_ERR_MISALIGNED, "dbg_acc_i32 is not 16-byte aligned");
    if (dbg_f && !aligned16(dbg_f)) return fail(SQ_ERR_MISALIGNED, "dbg_acc_f32 is not 16-byte aligned");
    return gemm_impl(X_N, s_x, X_O, W_N, s_w, W_O, M, N, K, nO, Y, ldy, dbg_i, dbg_f, stream, fp8);
}

// Single-thread kernel that waits on a barrier nobody completes, with a
// bounded wait, then records the timeout and exits.
__global__ void watchdog_selftest_kernel(unsigned long long limit_ns)
{
    __shared__ __align__(8) uint64_t bar;
    const uint32_t b = sqd::smem_u32(&bar);
    sqd::mbar_init(b, 1);
    sqd::fence_barrier_init();
    const unsigned long long t0 = sqd::globaltimer();
    while (!sqd::mbar_try_wait(b, 0)) {
        if (sqd::globaltimer() - t0 > limit_ns) {
            atomicCAS(&g_sq_dev_error, 0u, 0x7E57u);
            return;
        }
    }
}

// Low-path code bytes per row: kn_pad / 2 (packed INT4) or kn_pad (E4M3).
int64_t code_row_bytes(int64_t K, int64_t nO, bool fp8) { return fp8 ? sq_kn_pad(K, nO) : sq_kn_pad(K, nO) / 2; }

size_t linear_ws_bytes(int64_t M, int64_t K, int64_t nO, bool fp8)
{
    if (M <= 0) return 0;
    const int64_t xn = round_up(M * code_row_bytes(K, nO, fp8), 256);
    const int64_t sx = round_up(M * 4, 256);
    const int64_t xo = round_up(M * sq_no_pad(nO) * 2, 256);
    return static_cast<size_t>(xn + sx + xo);
}

// O: host list, already validated.  Static channel table: one word per 8
// channels, (outliers below) << 8 | outlier bits; copied on stream s from a
// host vector that lives until the caller synchronizes.
sq_status upload_chan_table(const int32_t *O, int64_t nO, int64_t K, uint32_t *chan_tab, cudaStream_t s)
{
    static thread_local std::vector<uint32_t> tab;
    tab.assign(static_cast<size_t>(K / 8), 0u);
    for (int64_t j = 0; j < nO; ++j) tab[O[j] / 8] |= 1u << (O[j] % 8);
    uint32_t below = 0;
    for (int64_t c = 0; c < K / 8; ++c) {
        const uint32_t mask = tab[c];
        tab[c] = (below << 8) | mask;
        below += static_cast<uint32_t>(__builtin_popcount(mask));
    }
    cudaError_t e = cudaMemcpyAsync(chan_tab, tab.data(), tab.size() * sizeof(uint32_t), cudaMemcpyHostToDevice, s);
    if (e != cudaSuccess) return cuda_fail(e, "copy of the channel table");
    return SQ_OK;
}

sq_status check_outlier_list(const int32_t *O, int64_t nO, int64_t K)
{
    if (nO > 0 && !O) return fail(SQ_ERR_INVALID_ARG, "O is NULL");
    for (int64_t j = 0; j < nO; ++j) {
        if (O[j] < 0 || O[j] >= K) return fail(SQ_ERR_INVALID_ARG, "O[%lld]=%d outside [0, K)", (long long)j, O[j]);
        if (j > 0 && O[j] <= O[j - 1]) return fail(SQ_ERR_INVALID_ARG, "O must be strictly increasing (index %lld)", (long long)j);
    }
    return SQ_OK;
}

sq_status prepare_impl(const void *W, int64_t N, int64_t K, int64_t ldw, const int32_t *O, int64_t nO, void *W_N,
                       float *s_w, void *W_O, uint32_t *chan_tab, cudaStream_t s, bool fp8)
{
    SQ_TRY(check_K_nO(K, nO));
    if (fp8 && K > sqq::kStreamMaxK)
        return fail(SQ_ERR_UNSUPPORTED, "the FP8 low path supports K <= %d (K=%lld)", sqq::kStreamMaxK, (long long)K);
    if (N < 0) return fail(SQ_ERR_INVALID_ARG, "N < 0");
    if (ldw < K || ldw % 8 != 0) return fail(SQ_ERR_INVALID_ARG, "ldw must be >= K and a multiple of 8");
    SQ_TRY(check_outlier_list(O, nO, K));
    SQ_TRY(check_ptr(chan_tab, true, "chan_tab"));
    const int64_t kn_pad = sq_kn_pad(K, nO);
    if (N > 0) {
        SQ_TRY(check_ptr(W, true, "W"));
        SQ_TRY(check_ptr(W_N, kn_pad > 0, "W_N"));
        SQ_TRY(check_ptr(s_w, true, "s_w"));
        SQ_TRY(check_ptr(W_O, nO > 0, "W_O"));
    }
    DevInfo di;
    SQ_TRY(device_info(di));
    SQ_TRY(upload_chan_table(O, nO, K, chan_tab, s));
    cudaError_t e;
    SQ_TRY(launch_rowquant(static_cast<const uint16_t *>(W), N, K, ldw, chan_tab, nO, static_cast<uint8_t *>(W_N), s_w,
                           static_cast<uint16_t *>(W_O), s, fp8));
    if ((e = cudaStreamSynchronize(s)) != cudaSuccess) return cuda_fail(e, "sq_prepare_weights");
    return SQ_OK;
}

sq_status linear_impl(const void *X, int64_t M, int64_t K, int64_t ldx, const uint32_t *chan_tab, const void *W_N,
                      const float *s_w, const void *W_O, int64_t N, int64_t nO, void *Y, int64_t ldy, void *workspace,
                      size_t ws_bytes, cudaStream_t s, bool fp8)
{
    SQ_TRY(check_K_nO(K, nO));
    if (M < 0) return fail(SQ_ERR_INVALID_ARG, "M < 0");
    if (M == 0) return SQ_OK;
    const size_t need = linear_ws_bytes(M, K, nO, fp8);
    if (ws_bytes < need) return fail(SQ_ERR_INVALID_ARG, "workspace of %zu bytes, %zu needed", ws_bytes, need);
    SQ_TRY(check_ptr(workspace, true, "workspace"));
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    const int64_t kn_pad = sq_kn_pad(K, nO), no_pad = sq_no_pad(nO);
    const int64_t xn_bytes = round_up(M * code_row_bytes(K, nO, fp8), 256);
    uint8_t *X_N = ws;
    float *s_x = reinterpret_cast<float *>(ws + xn_bytes);
    uint16_t *X_O = reinterpret_cast<uint16_t *>(ws + xn_bytes + round_up(M * 4, 256));
    SQ_TRY(quant_gather_impl(X, M, K, ldx, chan_tab, nO, kn_pad > 0 ? X_N : nullptr, s_x, no_pad > 0 ? X_O : nullptr, s,
                             fp8));
    return gemm_checked(kn_pad > 0 ? X_N : nullptr, s_x, no_pad > 0 ? X_O : nullptr, W_N, s_w, W_O, M, N, K, nO, Y, ldy,
                        nullptr, nullptr, s, fp8);
}

// ---------------------------------------------------------------- MXFP4 low path
// Quantize-and-gather of `rows` rows into packed E2M1 codes (dn), tiled
// E8M0 block scales (ds, rows padded to 128) and the compact outlier part.
sq_status launch_mxquant(const uint16_t *src, int64_t rows, int64_t K, int64_t ld, const uint32_t *tab, int64_t nO,
                         uint8_t *dn, uint8_t *ds, uint16_t *dout, cudaStream_t stream)
{
    if (rows == 0) return SQ_OK;
    DevInfo di;
    SQ_TRY(device_info(di));
    const int64_t kn_pad = sq_kn_pad_mx(K, nO), no_pad = sq_no_pad(nO);
    const int64_t rows_pad = round_up(rows, 128);
    const size_t smem = static_cast<size_t>(2 * (kn_pad + no_pad));
    int per_sm = 0;
    SQ_TRY(kernel_setup(reinterpret_cast<const void *>(sqq::mx_quant_kernel), sqq::kMxThreads, smem, per_sm,
                        "MX quantize set-up"));
    const int64_t grid = std::min<int64_t>(rows_pad, static_cast<int64_t>(di.sms) * per_sm);
    cudaError_t e = launch_k(sqq::mx_quant_kernel, dim3(static_cast<unsigned>(grid)), dim3(sqq::kMxThreads), smem,
                             stream, 0u, src, static_cast<int>(rows), static_cast<int>(rows_pad), static_cast<int>(K),
                             ld, tab, static_cast<int>(nO), static_cast<int>(K - nO), static_cast<int>(kn_pad),
                             static_cast<int>(no_pad), dn, ds, dout);
    if (e != cudaSuccess) return cuda_fail(e, "MX quantize launch");
    return SQ_OK;
}

sq_status quant_gather_mx_impl(const void *X, int64_t M, int64_t K, int64_t ldx, const uint32_t *chan_tab, int64_t nO,
                               void *X_N4, void *S_X, void *X_O, cudaStream_t stream)
{
    SQ_TRY(check_K_nO(K, nO));
    if (M < 0 || M > (1ll << 30)) return fail(SQ_ERR_INVALID_ARG, "M out of range");
    if (ldx < K || ldx % 8 != 0) return fail(SQ_ERR_INVALID_ARG, "ldx must be >= K and a multiple of 8");
    if (M == 0) return SQ_OK;
    const int64_t kn_pad = sq_kn_pad_mx(K, nO);
    SQ_TRY(check_ptr(X, true, "X"));
    SQ_TRY(check_ptr(chan_tab, true, "chan_tab"));
    SQ_TRY(check_ptr(X_N4, kn_pad > 0, "X_N4"));
    SQ_TRY(check_ptr(S_X, kn_pad > 0, "S_X"));
    SQ_TRY(check_ptr(X_O, nO > 0, "X_O"));
    return launch_mxquant(static_cast<const uint16_t *>(X), M, K, ldx, chan_tab, nO, static_cast<uint8_t *>(X_N4),
                          static_cast<uint8_t *>(S_X), static_cast<uint16_t *>(X_O), stream);
}

sq_status gemm_mx_checked(const void *X_N4, const void *S_X, const void *X_O, const void *W_N4, const void *S_W,
                          const void *W_O, int64_t M, int64_t N, int64_t K, int64_t nO, void *Y, int64_t ldy,
                          float *dbg, cudaStream_t stream)
{
    SQ_TRY(check_K_nO(K, nO));
    if (M < 0 || M > (1ll << 30)) return fail(SQ_ERR_INVALID_ARG, "M out of range");
    if (N < 0 || N % 8 != 0 || N > (1ll << 30)) return fail(SQ_ERR_INVALID_ARG, "N must be a non-negative multiple of 8");
    if (ldy < N || ldy % 8 != 0) return fail(SQ_ERR_INVALID_ARG, "ldy must be >= N and a multiple of 8");
    if (M == 0 || N == 0) return SQ_OK;
    const int64_t kn_pad = sq_kn_pad_mx(K, nO);
    SQ_TRY(check_ptr(X_N4, kn_pad > 0, "X_N4"));
    SQ_TRY(check_ptr(W_N4, kn_pad > 0, "W_N4"));
    SQ_TRY(check_ptr(S_X, kn_pad > 0, "S_X"));
    SQ_TRY(check_ptr(S_W, kn_pad > 0, "S_W"));
    SQ_TRY(check_ptr(X_O, nO > 0, "X_O"));
    SQ_TRY(check_ptr(W_O, nO > 0, "W_O"));
    SQ_TRY(check_ptr(Y, true, "Y"));
    if (dbg && !aligned16(dbg)) return fail(SQ_ERR_MISALIGNED, "dbg_acc is not 16-byte aligned");
    DevInfo di;
    SQ_TRY(device_info(di));
    // The scale operands travel in place of the fp32 scale pointers.
    const float *sx = static_cast<const float *>(S_X), *sw = static_cast<const float *>(S_W);
    if (M > 128)
        return launch_gemm_pair_t<CfgPairMx, sqg::kLowMx>(di, X_N4, sx, X_O, W_N4, sw, W_O, M, N, K, nO, Y, ldy,
                                                          nullptr, dbg, stream);
    if (M <= 16)
        return launch_gemm_skinny_t<CfgSk16Mx, sqg::kLowMx>(di, X_N4, sx, X_O, W_N4, sw, W_O, M, N, K, nO, Y, ldy,
                                                            nullptr, dbg, stream);
    if (M <= 32)
        return launch_gemm_skinny_t<CfgSk32Mx, sqg::kLowMx>(di, X_N4, sx, X_O, W_N4, sw, W_O, M, N, K, nO, Y, ldy,
                                                            nullptr, dbg, stream);
    if (M <= 64)
        return launch_gemm_skinny_t<CfgSk64Mx, sqg::kLowMx>(di, X_N4, sx, X_O, W_N4, sw, W_O, M, N, K, nO, Y, ldy,
                                                            nullptr, dbg, stream);
    return launch_gemm_skinny_t<CfgSk128Mx, sqg::kLowMx>(di, X_N4, sx, X_O, W_N4, sw, W_O, M, N, K, nO, Y, ldy,
                                                         nullptr, dbg, stream);
}

size_t linear_ws_bytes_mx(int64_t M, int64_t K, int64_t nO)
{
    if (M <= 0) return 0;
    const int64_t xn = round_up(M * (sq_kn_pad_mx(K, nO) / 2), 256);
    const int64_t sx = round_up(static_cast<int64_t>(sq_mx_scale_bytes(M, K, nO)), 256);
    const int64_t xo = round_up(M * sq_no_pad(nO) * 2, 256);
    return static_cast<size_t>(xn + sx + xo);
}

sq_status prepare_mx_impl(const void *W, int64_t N, int64_t K, int64_t ldw, const int32_t *O, int64_t nO, void *W_N4,
                          void *S_W, void *W_O, uint32_t *chan_tab, cudaStream_t s)
{
    SQ_TRY(check_K_nO(K, nO));
    if (N < 0 || N > (1ll << 30)) return fail(SQ_ERR_INVALID_ARG, "N out of range");
    if (ldw < K || ldw % 8 != 0) return fail(SQ_ERR_INVALID_ARG, "ldw must be >= K and a multiple of 8");
    SQ_TRY(check_outlier_list(O, nO, K));
    SQ_TRY(check_ptr(chan_tab, true, "chan_tab"));
    const int64_t kn_pad = sq_kn_pad_mx(K, nO);
    if (N > 0) {
        SQ_TRY(check_ptr(W, true, "W"));
        SQ_TRY(check_ptr(W_N4, kn_pad > 0, "W_N4"));
        SQ_TRY(check_ptr(S_W, kn_pad > 0, "S_W"));
        SQ_TRY(check_ptr(W_O, nO > 0, "W_O"));
    }
    DevInfo di;
    SQ_TRY(device_info(di));
    SQ_TRY(upload_chan_table(O, nO, K, chan_tab, s));
    SQ_TRY(launch_mxquant(static_cast<const uint16_t *>(W), N, K, ldw, chan_tab, nO, static_cast<uint8_t *>(W_N4),
                          static_cast<uint8_t *>(S_W), static_cast<uint16_t *>(W_O), s));
    cudaError_t e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail(e, "sq_prepare_weights_mx");
    return SQ_OK;
}

sq_status linear_mx_impl(const void *X, int64_t M, int64_t K, int64_t ldx, const uint32_t *chan_tab, const void *W_N4,
                         const void *S_W, const void *W_O, int64_t N, int64_t nO, void *Y, int64_t ldy,
                         void *workspace, size_t ws_bytes, cudaStream_t s)
{
    SQ_TRY(check_K_nO(K, nO));
    if (M < 0) return fail(SQ_ERR_INVALID_ARG, "M < 0");
    if (M == 0) return SQ_OK;
    const size_t need = linear_ws_bytes_mx(M, K, nO);
    if (ws_bytes < need) return fail(SQ_ERR_INVALID_ARG, "workspace of %zu bytes, %zu needed", ws_bytes, need);
    SQ_TRY(check_ptr(workspace, true, "workspace"));
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    const int64_t kn_pad = sq_kn_pad_mx(K, nO), no_pad = sq_no_pad(nO);
    const int64_t xn_bytes = round_up(M * (kn_pad / 2), 256);
    const int64_t sx_bytes = round_up(static_cast<int64_t>(sq_mx_scale_bytes(M, K, nO)), 256);
    uint8_t *X_N4 = ws;
    uint8_t *S_X = ws + xn_bytes;
    uint16_t *X_O = reinterpret_cast<uint16_t *>(ws + xn_bytes + sx_bytes);
    SQ_TRY(quant_gather_mx_impl(X, M, K, ldx, chan_tab, nO, kn_pad > 0 ? X_N4 : nullptr, kn_pad > 0 ? S_X : nullptr,
                                no_pad > 0 ? X_O : nullptr, s));
    return gemm_mx_checked(kn_pad > 0 ? X_N4 : nullptr, kn_pad > 0 ? S_X : nullptr, no_pad > 0 ? X_O : nullptr, W_N4,
                           S_W, W_O, M, N, K, nO, Y, ldy, nullptr, s);
}

// ---------------------------------------------------------------- element-level SQ-format
using CfgHigh32 = sqf::CfgHigh<32, 6>;
using CfgHigh128 = sqf::CfgHigh<128, 4>;
using CfgHigh32x2 = sqf::CfgHigh<32, 6, 2>;     // K stages split over a cluster of two CTAs
using CfgHigh128x2 = sqf::CfgHigh<128, 4, 2>;
using CfgHighPair = sqf::CfgHighPair<4, 8>;

bool sqf_bank_ok(int bank, int h) { return (bank == 4 || bank == 8 || bank == 16) && (h == 1 || h == 2); }

sq_status check_sqf_K(int64_t K)
{
    if (K < 256 || K > sqq::kStreamMaxK || K % 256 != 0)
        return fail(SQ_ERR_INVALID_ARG, "the SQ-format path needs K a multiple of 256 in [256, %d] (K=%lld)",
                    sqq::kStreamMaxK, (long long)K);
    return SQ_OK;
}

size_t sqf_ws_bytes(int64_t M, int64_t N, int64_t K)
{
    if (M <= 0) return 0;
    return static_cast<size_t>(round_up(M * K / 2, 256) + round_up(M * 4, 256) + round_up(M * K, 256) +
                               round_up(M * 4, 256) + round_up(M * N * 4, 256));
}

sq_status prepare_sqf_impl(const void *W, int64_t N, int64_t K, int64_t ldw, int bank, int h, void *W_N, float *s_lo,
                           void *W_H, void *W_E, float *s_hi, uint32_t *chan_tab, cudaStream_t s)
{
    SQ_TRY(check_sqf_K(K));
    if (!sqf_bank_ok(bank, h)) return fail(SQ_ERR_INVALID_ARG, "bank must be 4, 8 or 16 and h 1 or 2 (bank=%d h=%d)", bank, h);
    if (N < 0 || N > (1ll << 30)) return fail(SQ_ERR_INVALID_ARG, "N out of range");
    if (ldw < K || ldw % 8 != 0) return fail(SQ_ERR_INVALID_ARG, "ldw must be >= K and a multiple of 8");
    SQ_TRY(check_ptr(chan_tab, true, "chan_tab"));
    if (N > 0) {
        SQ_TRY(check_ptr(W, true, "W"));
        SQ_TRY(check_ptr(W_N, true, "W_N"));
        SQ_TRY(check_ptr(s_lo, true, "s_lo"));
        SQ_TRY(check_ptr(W_H, true, "W_H"));
        SQ_TRY(check_ptr(W_E, true, "W_E"));
        SQ_TRY(check_ptr(s_hi, true, "s_hi"));
    }
    DevInfo di;
    SQ_TRY(device_info(di));
    // no outlier channels: the channel table is all zeros
    cudaError_t e = cudaMemsetAsync(chan_tab, 0, static_cast<size_t>(K / 8) * 4, s);
    if (e != cudaSuccess) return cuda_fail(e, "channel table");
    if (N > 0) {
        const int64_t grid = std::min<int64_t>((N + 7) / 8, static_cast<int64_t>(di.sms) * 8);
        if ((e = launch_k(sqf::sqf_prep_kernel, dim3(static_cast<unsigned>(grid)), dim3(sqf::kPrepThreads), 0, s, 0u,
                          static_cast<const uint16_t *>(W), static_cast<int>(N), static_cast<int>(K), ldw, bank, h,
                          static_cast<uint8_t *>(W_N), s_lo, static_cast<uint8_t *>(W_H), static_cast<uint8_t *>(W_E),
                          s_hi)) != cudaSuccess)
            return cuda_fail(e, "SQ-format weight preparation");
    }
    if ((e = cudaStreamSynchronize(s)) != cudaSuccess) return cuda_fail(e, "sq_prepare_weights_sqf");
    return SQ_OK;
}

sq_status quant_sqf_impl(const void *X, int64_t M, int64_t K, int64_t ldx, const uint32_t *chan_tab, void *X_N,
                         float *s_x4, void *X_8, float *s_x8, cudaStream_t s)
{
    SQ_TRY(check_sqf_K(K));
    if (M < 0 || M > (1ll << 30)) return fail(SQ_ERR_INVALID_ARG, "M out of range");
    if (ldx < K || ldx % 8 != 0) return fail(SQ_ERR_INVALID_ARG, "ldx must be >= K and a multiple of 8");
    if (M == 0) return SQ_OK;
    SQ_TRY(check_ptr(X, true, "X"));
    SQ_TRY(check_ptr(chan_tab, true, "chan_tab"));
    SQ_TRY(check_ptr(X_N, true, "X_N"));
    SQ_TRY(check_ptr(s_x4, true, "s_x4"));
    SQ_TRY(check_ptr(X_8, true, "X_8"));
    SQ_TRY(check_ptr(s_x8, true, "s_x8"));
    const uint16_t *x = static_cast<const uint16_t *>(X);
    SQ_TRY(launch_rowquant(x, M, K, ldx, chan_tab, 0, static_cast<uint8_t *>(X_N), s_x4, nullptr, s, false));
    return launch_rowquant(x, M, K, ldx, chan_tab, 0, static_cast<uint8_t *>(X_8), s_x8, nullptr, s, true);
}

sq_status gemm_sqf_impl(const void *X_N, const float *s_x4, const void *X_8, const float *s_x8, const void *W_N,
                        const float *s_lo, const void *W_H, const void *W_E, const float *s_hi, int64_t M, int64_t N,
                        int64_t K, void *Y, int64_t ldy, float *P, int32_t *dbg_lo, cudaStream_t s)
{
    SQ_TRY(check_sqf_K(K));
    if (M < 0 || M > (1ll << 30)) return fail(SQ_ERR_INVALID_ARG, "M out of range");
    if (N < 0 || N % 8 != 0 || N > (1ll << 30)) return fail(SQ_ERR_INVALID_ARG, "N must be a non-negative multiple of 8");
    if (ldy < N || ldy % 8 != 0) return fail(SQ_ERR_INVALID_ARG, "ldy must be >= N and a multiple of 8");
    if (M == 0 || N == 0) return SQ_OK;
    SQ_TRY(check_ptr(X_N, true, "X_N"));
    SQ_TRY(check_ptr(s_x4, true, "s_x4"));
    SQ_TRY(check_ptr(X_8, true, "X_8"));
    SQ_TRY(check_ptr(s_x8, true, "s_x8"));
    SQ_TRY(check_ptr(W_N, true, "W_N"));
    SQ_TRY(check_ptr(s_lo, true, "s_lo"));
    SQ_TRY(check_ptr(W_H, true, "W_H"));
    SQ_TRY(check_ptr(W_E, true, "W_E"));
    SQ_TRY(check_ptr(s_hi, true, "s_hi"));
    SQ_TRY(check_ptr(Y, true, "Y"));
    SQ_TRY(check_ptr(P, true, "P"));
    if (dbg_lo && !aligned16(dbg_lo)) return fail(SQ_ERR_MISALIGNED, "dbg_acc_lo is not 16-byte aligned");
    DevInfo di;
    SQ_TRY(device_info(di));
    // 1. high part on the sparse tensor cores: P = s_x8 s_hi (e(X) . e(W_hi)^T); CTA pairs of
    //    256 W rows x 256 tokens for M > 128, single CTAs of 128 W rows x 32 or 128 tokens otherwise
    CUtensorMap m_wh{}, m_we{}, m_x8{};
    const bool pair = M > 128;
    const bool small = M <= 32;
    const int mt = small ? CfgHigh32::MT : CfgHigh128::MT;   // token rows per TMA box (128 for the pair kernel)
    SQ_TRY(make_map(m_wh, W_H, CU_TENSOR_MAP_DATA_TYPE_UINT8, K / 2, N, K / 2, 128, 128, CU_TENSOR_MAP_SWIZZLE_128B));
    SQ_TRY(make_map(m_we, W_E, CU_TENSOR_MAP_DATA_TYPE_UINT8, K / 8, N, K / 8, 16, 128, CU_TENSOR_MAP_SWIZZLE_NONE));
    SQ_TRY(make_map(m_x8, X_8, CU_TENSOR_MAP_DATA_TYPE_UINT8, K, M, K, 128, static_cast<uint32_t>(mt),
                    CU_TENSOR_MAP_SWIZZLE_128B));
    sqf::HighArgs ha;
    ha.s_x8 = s_x8;
    ha.s_hi = s_hi;
    ha.P = P;
    ha.M = static_cast<int>(M);
    ha.N = static_cast<int>(N);
    ha.K = static_cast<int>(K);
    // bands of M-tiles whose E4M3 token rows (K bytes each) stay in L2 while the W tiles stream
    ha.group_m = raster_group(static_cast<int>((M + 255) / 256), 256, 2 * K, 0);
    cudaError_t e;
    if (pair) {
        // persistent: one cluster per SM pair, tiles handed out in the band order
        auto kern = sqf::sqf_high_pair_kernel<CfgHighPair>;
        const int64_t tiles = ((N + 255) / 256) * ((M + 255) / 256);
        const int64_t clusters = std::min<int64_t>(tiles, di.sms / 2);
        int per_sm = 0;
        SQ_TRY(kernel_setup(reinterpret_cast<const void *>(kern), CfgHighPair::THREADS, CfgHighPair::SMEM_BYTES,
                            per_sm, "SQ-format high part set-up"));
        e = launch_k(kern, dim3(static_cast<unsigned>(2 * clusters)), dim3(CfgHighPair::THREADS),
                     CfgHighPair::SMEM_BYTES, s, 0u, m_wh, m_we, m_x8, ha);
    } else {
        // One CTA per 128 W rows x mt tokens; when that fills at most half of the SMs and there
        // are two or more K stages, a cluster of two CTAs splits each tile's K stages.
        const int64_t tiles = ((N + 127) / 128) * ((M + mt - 1) / mt);
        const bool split = K / 256 >= 2 && 2 * tiles <= di.sms;
        const dim3 grid(static_cast<unsigned>((N + 127) / 128 * (split ? 2 : 1)), static_cast<unsigned>((M + mt - 1) / mt));
        auto kern = split ? (small ? sqf::sqf_high_kernel<CfgHigh32x2> : sqf::sqf_high_kernel<CfgHigh128x2>)
                          : (small ? sqf::sqf_high_kernel<CfgHigh32> : sqf::sqf_high_kernel<CfgHigh128>);
        const size_t smem = small ? CfgHigh32::SMEM_BYTES : CfgHigh128::SMEM_BYTES;
        int per_sm = 0;
        SQ_TRY(kernel_setup(reinterpret_cast<const void *>(kern), sqf::kHiThreads, smem, per_sm,
                            "SQ-format high part set-up"));
        e = launch_k(kern, grid, dim3(sqf::kHiThreads), smem, s, split ? 2u : 0u, m_wh, m_we, m_x8, ha);
    }
    if (e != cudaSuccess) return cuda_fail(e, "SQ-format high part launch");
    // 2. low part (INT4, mask code cleared) with P added before the bf16 rounding
    const float *sx = s_x4, *sw = s_lo;
    if (pair)
        return launch_gemm_pair_t<CfgPairSqf, sqg::kLowSqf>(di, X_N, sx, nullptr, W_N, sw, nullptr, M, N, K, 0, Y, ldy,
                                                         dbg_lo, nullptr, s, P);
    if (M <= 16)
        return launch_gemm_skinny_t<CfgSk16, sqg::kLowSqf>(di, X_N, sx, nullptr, W_N, sw, nullptr, M, N, K, 0, Y, ldy,
                                                           dbg_lo, nullptr, s, P);
    if (M <= 32)
        return launch_gemm_skinny_t<CfgSk32, sqg::kLowSqf>(di, X_N, sx, nullptr, W_N, sw, nullptr, M, N, K, 0, Y, ldy,
                                                           dbg_lo, nullptr, s, P);
    if (M <= 64)
        return launch_gemm_skinny_t<CfgSk64, sqg::kLowSqf>(di, X_N, sx, nullptr, W_N, sw, nullptr, M, N, K, 0, Y, ldy,
                                                           dbg_lo, nullptr, s, P);
    return launch_gemm_skinny_t<CfgSk128, sqg::kLowSqf>(di, X_N, sx, nullptr, W_N, sw, nullptr, M, N, K, 0, Y, ldy,
                                                        dbg_lo, nullptr, s, P);
}

sq_status linear_sqf_impl(const void *X, int64_t M, int64_t K, int64_t ldx, const uint32_t *chan_tab, const void *W_N,
                          const float *s_lo, const void *W_H, const void *W_E, const float *s_hi, int64_t N, void *Y,
                          int64_t ldy, void *workspace, size_t ws_bytes, cudaStream_t s)
{
    SQ_TRY(check_sqf_K(K));
    if (M < 0 || N < 0) return fail(SQ_ERR_INVALID_ARG, "M and N must be non-negative");
    if (M == 0 || N == 0) return SQ_OK;
    const size_t need = sqf_ws_bytes(M, N, K);
    if (ws_bytes < need) return fail(SQ_ERR_INVALID_ARG, "workspace of %zu bytes, %zu needed", ws_bytes, need);
    SQ_TRY(check_ptr(workspace, true, "workspace"));
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    uint8_t *X_N = ws;
    float *s_x4 = reinterpret_cast<float *>(ws + round_up(M * K / 2, 256));
    uint8_t *X_8 = reinterpret_cast<uint8_t *>(s_x4) + round_up(M * 4, 256);
    float *s_x8 = reinterpret_cast<float *>(X_8 + round_up(M * K, 256));
    float *P = reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(s_x8) + round_up(M * 4, 256));
    SQ_TRY(quant_sqf_impl(X, M, K, ldx, chan_tab, X_N, s_x4, X_8, s_x8, s));
    return gemm_sqf_impl(X_N, s_x4, X_8, s_x8, W_N, s_lo, W_H, W_E, s_hi, M, N, K, Y, ldy, P, nullptr, s);
}

// ---------------------------------------------------------------- static outlier selection
struct SelectLayout {
    int64_t nbx, nbw, off_px, off_pw, off_score, off_gs, bytes;
    SelectLayout(int64_t Mc, int64_t N, int64_t K, int64_t group)
    {
        nbx = (Mc + sqs::kSelBlock - 1) / sqs::kSelBlock;
        nbw = (N + sqs::kSelBlock - 1) / sqs::kSelBlock;
        off_px = 0;
        off_pw = round_up(nbx * K * 8, 256);
        off_score = off_pw + round_up(nbw * K * 8, 256);
        off_gs = off_score + round_up(K * 8, 256);
        bytes = off_gs + round_up((group > 0 ? K / group : K) * 8, 256);
    }
};

sq_status select_impl(const void *Xc, int64_t Mc, int64_t K, int64_t ldx, const void *W, int64_t N, int64_t ldw,
                      int64_t nO, int64_t group, int32_t *O, double *scores, void *workspace, size_t ws_bytes,
                      cudaStream_t s)
{
    if (K < 1 || K > SQ_MAX_K) return fail(SQ_ERR_INVALID_ARG, "K=%lld outside [1, %d]", (long long)K, SQ_MAX_K);
    if (Mc < 1 || N < 1) return fail(SQ_ERR_INVALID_ARG, "Mc and N must be positive");
    if ((Mc + sqs::kSelBlock - 1) / sqs::kSelBlock > 65535 || (N + sqs::kSelBlock - 1) / sqs::kSelBlock > 65535)
        return fail(SQ_ERR_UNSUPPORTED, "more than 65535 blocks of %d rows", sqs::kSelBlock);
    if (ldx < K || ldw < K) return fail(SQ_ERR_INVALID_ARG, "ldx and ldw must be >= K");
    if (group < 1 || K % group != 0) return fail(SQ_ERR_INVALID_ARG, "group must divide K");
    if (nO < 0 || nO > K || nO % group != 0) return fail(SQ_ERR_INVALID_ARG, "nO must lie in [0, K] and divide by group");
    if (!Xc || !W) return fail(SQ_ERR_INVALID_ARG, "Xc or W is NULL");
    if (nO > 0 && !O) return fail(SQ_ERR_INVALID_ARG, "O is NULL");
    SQ_TRY(check_ptr(workspace, true, "workspace"));
    if (scores && (reinterpret_cast<uintptr_t>(scores) & 7u)) return fail(SQ_ERR_MISALIGNED, "scores is not 8-byte aligned");
    const SelectLayout L(Mc, N, K, group);
    if (ws_bytes < static_cast<size_t>(L.bytes))
        return fail(SQ_ERR_INVALID_ARG, "workspace of %zu bytes, %lld needed", ws_bytes, (long long)L.bytes);
    DevInfo di;
    SQ_TRY(device_info(di));
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    double *px = reinterpret_cast<double *>(ws + L.off_px);
    double *pw = reinterpret_cast<double *>(ws + L.off_pw);
    double *sc = scores ? scores : reinterpret_cast<double *>(ws + L.off_score);
    double *gs = reinterpret_cast<double *>(ws + L.off_gs);
    const int k = static_cast<int>(K), ng = static_cast<int>(K / group);
    const unsigned gk = static_cast<unsigned>((K + sqs::kColThreads - 1) / sqs::kColThreads);
    cudaError_t e;
    auto colsums = [&](const void *A, int64_t rows, int64_t ld, int square, double *part, int64_t nb) {
        const bool pair = K % 2 == 0 && ld % 2 == 0 && (reinterpret_cast<uintptr_t>(A) & 3u) == 0;
        const unsigned g = static_cast<unsigned>((K / (pair ? 2 : 1) + sqs::kColThreads - 1) / sqs::kColThreads);
        const dim3 grid(g, static_cast<unsigned>(nb));
        return pair ? launch_k(sqs::colsum_blocks_kernel<true>, grid, dim3(sqs::kColThreads), 0, s, 0u,
                               static_cast<const uint16_t *>(A), rows, k, ld, square, part)
                    : launch_k(sqs::colsum_blocks_kernel<false>, grid, dim3(sqs::kColThreads), 0, s, 0u,
                               static_cast<const uint16_t *>(A), rows, k, ld, square, part);
    };
    if ((e = colsums(Xc, Mc, ldx, 0, px, L.nbx)) != cudaSuccess) return cuda_fail(e, "selection column sums (X)");
    if ((e = colsums(W, N, ldw, 1, pw, L.nbw)) != cudaSuccess) return cuda_fail(e, "selection column sums (W)");
    if ((e = launch_k(sqs::score_kernel, dim3(gk), dim3(sqs::kColThreads), 0, s, 0u, static_cast<const double *>(px),
                      static_cast<int>(L.nbx), Mc, static_cast<const double *>(pw), static_cast<int>(L.nbw), k, sc)) !=
        cudaSuccess)
        return cuda_fail(e, "selection scores");
    if ((e = launch_k(sqs::group_score_kernel, dim3(static_cast<unsigned>((ng + sqs::kColThreads - 1) / sqs::kColThreads)),
                      dim3(sqs::kColThreads), 0, s, 0u, static_cast<const double *>(sc), ng, static_cast<int>(group),
                      gs)) != cudaSuccess)
        return cuda_fail(e, "selection group scores");
    if ((e = launch_k(sqs::select_top_kernel, dim3(1), dim3(sqs::kTopThreads), 0, s, 0u, static_cast<const double *>(gs),
                      ng, static_cast<int>(nO / group), static_cast<int>(group), O)) != cudaSuccess)
        return cuda_fail(e, "selection top-k");
    return SQ_OK;
}

}  // namespace

// ================================================================ C ABI
extern "C" {

const char *sq_status_string(sq_status s)
{
    switch (s) {
    case SQ_OK: return "SQ_OK";
    case SQ_ERR_INVALID_ARG: return "SQ_ERR_INVALID_ARG";
    case SQ_ERR_UNSUPPORTED: return "SQ_ERR_UNSUPPORTED";
    case SQ_ERR_MISALIGNED: return "SQ_ERR_MISALIGNED";
    case SQ_ERR_CUDA: return "SQ_ERR_CUDA";
    case SQ_ERR_TIMEOUT: return "SQ_ERR_TIMEOUT";
    }
    return "SQ_ERR_UNKNOWN";
}

const char *sq_last_error_detail(void) { return g_detail.c_str(); }

int64_t sq_kn_pad(int64_t K, int64_t nO) { return round_up(K - nO, 128); }

int64_t sq_no_pad(int64_t nO) { return round_up(nO, 64); }

int64_t sq_chan_table_words(int64_t K) { return K / 8; }

size_t sq_linear_workspace_bytes(int64_t M, int64_t K, int64_t nO) { return linear_ws_bytes(M, K, nO, false); }

size_t sq_linear_workspace_bytes_fp8(int64_t M, int64_t K, int64_t nO) { return linear_ws_bytes(M, K, nO, true); }

int64_t sq_kn_pad_mx(int64_t K, int64_t nO) { return round_up(K - nO, 256); }

size_t sq_linear_workspace_bytes_sqf(int64_t M, int64_t N, int64_t K) { return sqf_ws_bytes(M, N, K); }

sq_status sq_prepare_weights_sqf(const void *W, int64_t N, int64_t K, int64_t ldw, int bank, int h, void *W_N,
                                 float *s_lo, void *W_H, void *W_E, float *s_hi, uint32_t *chan_tab,
                                 sq_stream_t stream)
{
    g_detail.clear();
    return prepare_sqf_impl(W, N, K, ldw, bank, h, W_N, s_lo, W_H, W_E, s_hi, chan_tab,
                            reinterpret_cast<cudaStream_t>(stream));
}

sq_status sq_quant_gather_sqf(const void *X, int64_t M, int64_t K, int64_t ldx, const uint32_t *chan_tab, void *X_N,
                              float *s_x4, void *X_8, float *s_x8, sq_stream_t stream)
{
    g_detail.clear();
    return quant_sqf_impl(X, M, K, ldx, chan_tab, X_N, s_x4, X_8, s_x8, reinterpret_cast<cudaStream_t>(stream));
}

sq_status sq_gemm_sqf(const void *X_N, const float *s_x4, const void *X_8, const float *s_x8, const void *W_N,
                      const float *s_lo, const void *W_H, const void *W_E, const float *s_hi, int64_t M, int64_t N,
                      int64_t K, void *Y, int64_t ldy, float *P, int32_t *dbg_acc_lo, sq_stream_t stream)
{
    g_detail.clear();
    return gemm_sqf_impl(X_N, s_x4, X_8, s_x8, W_N, s_lo, W_H, W_E, s_hi, M, N, K, Y, ldy, P, dbg_acc_lo,
                         reinterpret_cast<cudaStream_t>(stream));
}

sq_status sq_linear_sqf(const void *X, int64_t M, int64_t K, int64_t ldx, const uint32_t *chan_tab, const void *W_N,
                        const float *s_lo, const void *W_H, const void *W_E, const float *s_hi, int64_t N, void *Y,
                        int64_t ldy, void *workspace, size_t ws_bytes, sq_stream_t stream)
{
    g_detail.clear();
    return linear_sqf_impl(X, M, K, ldx, chan_tab, W_N, s_lo, W_H, W_E, s_hi, N, Y, ldy, workspace, ws_bytes,
                           reinterpret_cast<cudaStream_t>(stream));
}

size_t sq_mx_scale_bytes(int64_t rows, int64_t K, int64_t nO)
{
    if (rows <= 0) return 0;
    return static_cast<size_t>(round_up(rows, 128) * (sq_kn_pad_mx(K, nO) / 32));
}

size_t sq_linear_workspace_bytes_mx(int64_t M, int64_t K, int64_t nO) { return linear_ws_bytes_mx(M, K, nO); }

sq_status sq_prepare_weights_mx(const void *W, int64_t N, int64_t K, int64_t ldw, const int32_t *O, int64_t nO,
                                void *W_N4, void *S_W, void *W_O, uint32_t *chan_tab, sq_stream_t stream)
{
    g_detail.clear();
    return prepare_mx_impl(W, N, K, ldw, O, nO, W_N4, S_W, W_O, chan_tab, reinterpret_cast<cudaStream_t>(stream));
}

sq_status sq_quant_gather_mx(const void *X, int64_t M, int64_t K, int64_t ldx, const uint32_t *chan_tab, int64_t nO,
                             void *X_N4, void *S_X, void *X_O, sq_stream_t stream)
{
    g_detail.clear();
    return quant_gather_mx_impl(X, M, K, ldx, chan_tab, nO, X_N4, S_X, X_O, reinterpret_cast<cudaStream_t>(stream));
}

sq_status sq_gemm_mx(const void *X_N4, const void *S_X, const void *X_O, const void *W_N4, const void *S_W,
                     const void *W_O, int64_t M, int64_t N, int64_t K, int64_t nO, void *Y, int64_t ldy,
                     float *dbg_acc, sq_stream_t stream)
{
    g_detail.clear();
    return gemm_mx_checked(X_N4, S_X, X_O, W_N4, S_W, W_O, M, N, K, nO, Y, ldy, dbg_acc,
                           reinterpret_cast<cudaStream_t>(stream));
}

sq_status sq_linear_mx(const void *X, int64_t M, int64_t K, int64_t ldx, const uint32_t *chan_tab, const void *W_N4,
                       const void *S_W, const void *W_O, int64_t N, int64_t nO, void *Y, int64_t ldy, void *workspace,
                       size_t ws_bytes, sq_stream_t stream)
{
    g_detail.clear();
    return linear_mx_impl(X, M, K, ldx, chan_tab, W_N4, S_W, W_O, N, nO, Y, ldy, workspace, ws_bytes,
                          reinterpret_cast<cudaStream_t>(stream));
}

sq_status sq_prepare_weights(const void *W, int64_t N, int64_t K, int64_t ldw, const int32_t *O, int64_t nO,
                             void *W_N, float *s_w, void *W_O, uint32_t *chan_tab, sq_stream_t stream)
{
    g_detail.clear();
    return prepare_impl(W, N, K, ldw, O, nO, W_N, s_w, W_O, chan_tab, reinterpret_cast<cudaStream_t>(stream), false);
}

sq_status sq_prepare_weights_fp8(const void *W, int64_t N, int64_t K, int64_t ldw, const int32_t *O, int64_t nO,
                                 void *W_N8, float *s_w, void *W_O, uint32_t *chan_tab, sq_stream_t stream)
{
    g_detail.clear();
    return prepare_impl(W, N, K, ldw, O, nO, W_N8, s_w, W_O, chan_tab, reinterpret_cast<cudaStream_t>(stream), true);
}

sq_status sq_quant_gather(const void *X, int64_t M, int64_t K, int64_t ldx, const uint32_t *chan_tab, int64_t nO,
                          void *X_N, float *s_x, void *X_O, sq_stream_t stream)
{
    g_detail.clear();
    return quant_gather_impl(X, M, K, ldx, chan_tab, nO, X_N, s_x, X_O, reinterpret_cast<cudaStream_t>(stream));
}

sq_status sq_quant_gather_fp8(const void *X, int64_t M, int64_t K, int64_t ldx, const uint32_t *chan_tab, int64_t nO,
                              void *X_N8, float *s_x, void *X_O, sq_stream_t stream)
{
    g_detail.clear();
    return quant_gather_impl(X, M, K, ldx, chan_tab, nO, X_N8, s_x, X_O, reinterpret_cast<cudaStream_t>(stream), true);
}

sq_status sq_gemm(const void *X_N, const float *s_x, const void *X_O, const void *W_N, const float *s_w,
                  const void *W_O, int64_t M, int64_t N, int64_t K, int64_t nO, void *Y, int64_t ldy,
                  int32_t *dbg_acc_i32, float *dbg_acc_f32, sq_stream_t stream)
{
    g_detail.clear();
    return gemm_checked(X_N, s_x, X_O, W_N, s_w, W_O, M, N, K, nO, Y, ldy, dbg_acc_i32, dbg_acc_f32,
                        reinterpret_cast<cudaStream_t>(stream));
}

sq_status sq_gemm_fp8(const void *X_N8, const float *s_x, const void *X_O, const void *W_N8, const float *s_w,
                      const void *W_O, int64_t M, int64_t N, int64_t K, int64_t nO, void *Y, int64_t ldy,
                      float *dbg_acc_8, float *dbg_acc_f32, sq_stream_t stream)
{
    g_detail.clear();
    return gemm_checked(X_N8, s_x, X_O, W_N8, s_w, W_O, M, N, K, nO, Y, ldy, reinterpret_cast<int32_t *>(dbg_acc_8),
                        dbg_acc_f32, reinterpret_cast<cudaStream_t>(stream), true);
}

sq_status sq_linear(const void *X, int64_t M, int64_t K, int64_t ldx, const uint32_t *chan_tab, const void *W_N,
                    const float *s_w, const void *W_O, int64_t N, int64_t nO, void *Y, int64_t ldy, void *workspace,
                    size_t ws_bytes, sq_stream_t stream)
{
    g_detail.clear();
    return linear_impl(X, M, K, ldx, chan_tab, W_N, s_w, W_O, N, nO, Y, ldy, workspace, ws_bytes,
                       reinterpret_cast<cudaStream_t>(stream), false);
}

sq_status sq_linear_fp8(const void *X, int64_t M, int64_t K, int64_t ldx, const uint32_t *chan_tab, const void *W_N8,
                        const float *s_w, const void *W_O, int64_t N, int64_t nO, void *Y, int64_t ldy, void *workspace,
                        size_t ws_bytes, sq_stream_t stream)
{
    g_detail.clear();
    return linear_impl(X, M, K, ldx, chan_tab, W_N8, s_w, W_O, N, nO, Y, ldy, workspace, ws_bytes,
                       reinterpret_cast<cudaStream_t>(stream), true);
}

size_t sq_select_outliers_workspace_bytes(int64_t Mc, int64_t N, int64_t K, int64_t group)
{
    if (Mc < 1 || N < 1 || K < 1 || group < 1) return 0;
    return static_cast<size_t>(SelectLayout(Mc, N, K, group).bytes);
}

sq_status sq_select_outliers(const void *Xc, int64_t Mc, int64_t K, int64_t ldx, const void *W, int64_t N, int64_t ldw,
                             int64_t nO, int64_t group, int32_t *O, double *scores, void *workspace, size_t ws_bytes,
                             sq_stream_t stream)
{
    g_detail.clear();
    return select_impl(Xc, Mc, K, ldx, W, N, ldw, nO, group, O, scores, workspace, ws_bytes,
                       reinterpret_cast<cudaStream_t>(stream));
}

sq_status sq_check(sq_stream_t stream)
{
    g_detail.clear();
    cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "sq_check");
    unsigned int word = 0;
    if ((e = cudaMemcpyFromSymbol(&word, g_sq_dev_error, sizeof word)) != cudaSuccess)
        return cuda_fail(e, "reading the device error word");
    if (word != 0) {
        const unsigned int zero = 0;
        if ((e = cudaMemcpyToSymbol(g_sq_dev_error, &zero, sizeof zero)) != cudaSuccess)
            return cuda_fail(e, "clearing the device error word");
        return fail(SQ_ERR_TIMEOUT, "a bounded wait ran out (site 0x%x)", word);
    }
    return SQ_OK;
}

sq_status sq_selftest_watchdog(int timeout_ms, sq_stream_t stream)
{
    g_detail.clear();
    if (timeout_ms < 1 || timeout_ms > 10000) return fail(SQ_ERR_INVALID_ARG, "timeout_ms must lie in [1, 10000]");
    DevInfo di;
    SQ_TRY(device_info(di));
    watchdog_selftest_kernel<<<1, 1, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        static_cast<unsigned long long>(timeout_ms) * 1000000ull);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "watchdog self-test launch");
    return SQ_OK;
}

}  // extern "C"

// ================================================================ workspace-free sq_linear
// Scratch for sq_linear_noalloc: a fixed array in the library, one per device
// that loads it.  Host code must not hand this symbol to a kernel directly
// (on the host it names a stand-in, not device memory); the device address is
// looked up once per device below.
static __device__ __align__(256) uint8_t g_sq_noalloc_ws[SQ_NOALLOC_WS_BYTES];

namespace {

void *g_noalloc_addr[kMaxDevices];
CUcontext g_noalloc_ctx[kMaxDevices];
std::mutex g_noalloc_mu;

// Device address of the scratch array on the current device, looked up on the
// first call for each device (with that device current) and again only if
// the device's context has changed since (after a device reset the module,
// and with it the array, is loaded anew).
sq_status noalloc_scratch(void **out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices) return fail(SQ_ERR_UNSUPPORTED, "device index %d", dev);
    CUcontext ctx;
    SQ_TRY(current_context(ctx));
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    if (!g_noalloc_addr[dev] || (ctx && g_noalloc_ctx[dev] != ctx)) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_sq_noalloc_ws);   // makes the device's context current if needed
        if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(scratch)");
        SQ_TRY(current_context(ctx));
        g_noalloc_addr[dev] = p;
        g_noalloc_ctx[dev] = ctx;
    }
    *out = g_noalloc_addr[dev];
    return SQ_OK;
}

}  // namespace

extern "C" sq_status sq_linear_noalloc(const void *X, int64_t M, int64_t K, int64_t ldx, const uint32_t *chan_tab,
                                       const void *W_N, const float *s_w, const void *W_O, int64_t N, int64_t nO,
                                       void *Y, int64_t ldy, sq_stream_t stream)
{
    g_detail.clear();
    SQ_TRY(check_K_nO(K, nO));
    if (M < 0) return fail(SQ_ERR_INVALID_ARG, "M < 0");
    if (M == 0) return SQ_OK;
    const size_t need = sq_linear_workspace_bytes(M, K, nO);
    if (need > SQ_NOALLOC_WS_BYTES)
        return fail(SQ_ERR_UNSUPPORTED,
                    "sq_linear_noalloc: M=%lld, K=%lld, nO=%lld need %zu scratch bytes but the built-in scratch "
                    "holds %u; split the tokens into smaller calls or use sq_linear with a workspace",
                    (long long)M, (long long)K, (long long)nO, need, SQ_NOALLOC_WS_BYTES);
    void *ws = nullptr;
    SQ_TRY(noalloc_scratch(&ws));
    return sq_linear(X, M, K, ldx, chan_tab, W_N, s_w, W_O, N, nO, Y, ldy, ws, SQ_NOALLOC_WS_BYTES, stream);
}
