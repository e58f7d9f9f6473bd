// convrot.cu -- the C ABI declared in include/convrot.h: argument validation,
// TMA descriptor encoding and kernel launches.  One translation unit holds the
// whole library so that the device status word has a single definition.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdarg>
#include <cstdio>
#include <mutex>
#include <string>
#include <utility>

#include "../../include/convrot.h"
#include "device_utils.cuh"
#include "gemm_tcgen05.cuh"
#include "gemv.cuh"
#include "rotate_quant.cuh"

namespace {

constexpr int kVersion = 100;  // 0.1.0
thread_local std::string g_last_error;

convrot_status_t fail(convrot_status_t st, const char *fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return st;
}

convrot_status_t ok() { return CONVROT_OK; }

#define CR_REQUIRE(cond, status, ...)                  \
    do {                                               \
        if (!(cond)) return fail(status, __VA_ARGS__); \
    } while (0)

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }
bool is_pow2(int64_t v) { return v > 0 && (v & (v - 1)) == 0; }
int ilog2(int64_t v) {
    int l = 0;
    while ((int64_t(1) << l) < v) ++l;
    return l;
}
size_t round256(size_t v) { return (v + 255) & ~size_t(255); }

// ---------------------------------------------------------------- device info

struct DeviceInfo {
    int major = 0, minor = 0, sms = 0;
    bool attrs_set = false;
};
constexpr int kMaxDevices = 64;
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mutex;

convrot_status_t current_device(int *dev, DeviceInfo **info) {
    cudaError_t e = cudaGetDevice(dev);
    CR_REQUIRE(e == cudaSuccess, CONVROT_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    CR_REQUIRE(*dev >= 0 && *dev < kMaxDevices, CONVROT_ERR_UNSUPPORTED, "device ordinal %d out of range", *dev);
    std::lock_guard<std::mutex> lock(g_dev_mutex);
    DeviceInfo &d = g_dev[*dev];
    if (d.sms == 0) {
        cudaDeviceGetAttribute(&d.major, cudaDevAttrComputeCapabilityMajor, *dev);
        cudaDeviceGetAttribute(&d.minor, cudaDevAttrComputeCapabilityMinor, *dev);
        e = cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, *dev);
        CR_REQUIRE(e == cudaSuccess, CONVROT_ERR_CUDA, "cudaDeviceGetAttribute: %s", cudaGetErrorString(e));
    }
    *info = &d;
    CR_REQUIRE(d.major == 10 && d.minor == 0, CONVROT_ERR_UNSUPPORTED,
               "this library is built for sm_100a (B200); device %d is sm_%d%d", *dev, d.major, d.minor);
    return ok();
}

convrot_status_t launch_status(const char *what) {
    cudaError_t e = cudaGetLastError();
    CR_REQUIRE(e == cudaSuccess, CONVROT_ERR_CUDA, "%s launch: %s", what, cudaGetErrorString(e));
    return ok();
}

// ---------------------------------------------------------------- TMA descriptors

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// A row-major matrix (rows x cols elements of `dtype`, `elem_bytes` each) read
// or written in boxes of box_rows x box_cols elements.
convrot_status_t make_map(CUtensorMap *map, const void *base, CUtensorMapDataType dtype, int elem_bytes, int64_t rows,
                          int64_t cols, int box_rows, int box_cols, CUtensorMapSwizzle swizzle) {
    EncodeTiledFn fn = encode_fn();
    CR_REQUIRE(fn != nullptr, CONVROT_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols * elem_bytes)};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(box_cols), static_cast<cuuint32_t>(box_rows)};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, dtype, 2, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    CR_REQUIRE(r == CUDA_SUCCESS, CONVROT_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
    return ok();
}

// ---------------------------------------------------------------- shared checks

convrot_status_t check_shape(int64_t rows, int64_t K, int block, const char *rows_name) {
    CR_REQUIRE(rows >= 0 && rows < (int64_t(1) << 31), CONVROT_ERR_INVALID_ARG, "%s = %lld out of [0, 2^31)",
               rows_name, static_cast<long long>(rows));
    CR_REQUIRE(K >= 128 && K <= 32768 && K % 128 == 0, CONVROT_ERR_INVALID_ARG,
               "K = %lld must be a multiple of 128 in [128, 32768]", static_cast<long long>(K));
    CR_REQUIRE(block >= 1 && block <= 256 && is_pow2(block) && K % block == 0, CONVROT_ERR_INVALID_ARG,
               "block = %d must be a power of two in [1, 256] dividing K", block);
    return ok();
}

convrot_status_t check_bits(int bits) {
    CR_REQUIRE(bits == 8 || bits == 4, CONVROT_ERR_INVALID_ARG, "bits = %d must be 8 or 4", bits);
    return ok();
}

#define CR_TRY(expr)                          \
    do {                                      \
        convrot_status_t st_ = (expr);        \
        if (st_ != CONVROT_OK) return st_;    \
    } while (0)

// Rows per CTA and threads per CTA of the rotation kernels (K/32 threads per
// row, at least 256 threads per CTA where K allows).
void rotate_geometry(int64_t K, int *rows, int *threads) {
    const int L = static_cast<int>(K / convrot::kElemsPerThread);
    int R = L >= 256 ? 1 : 256 / L;
    if (R > convrot::kMaxRowsPerCta) R = convrot::kMaxRowsPerCta;
    *rows = R;
    *threads = ((R * L + 31) / 32) * 32;
}

// For the activation kernel: the rows per CTA that minimise (waves x rows per
// CTA) given the kernel's real occupancy, so that a problem that fits in one
// wave is launched as exactly one wave (a partial second wave would repeat the
// whole load-compute-store latency).  Candidates are CTAs of whole warps with
// no padding threads and at least two warps, ties going to more rows; only if
// none exists are padded CTAs of at least 256 threads taken.  (Measured on
// B200, CUDA-graph-timed, rows per CTA: 16384 x 4096 1 row 51.1 us against 2
// rows 53.6; 5184 x 4096 20.1 against 20.4; 8192 x 1536 2 rows 13.96 against 5
// rows 14.2 and 1 padded row 14.8; 5184 x 1024 1 row of 32 threads 7.1 against
// 2 rows 6.5.)
template <typename Kern>
void act_geometry(Kern kernel, int sms, int64_t M, int64_t K, int *rows, int *threads, int *resident) {
    const int L = static_cast<int>(K / convrot::kElemsPerThread);
    int R0, T0;
    rotate_geometry(K, &R0, &T0);
    int best_R = R0, best_T = T0, best_cap = 0;
    int64_t best_cost = -1;
    const int rmax_threads = 1024 / L;
    const int r_hi = rmax_threads < convrot::kMaxRowsPerCta ? rmax_threads : convrot::kMaxRowsPerCta;
    for (int pass = 0; pass < 2 && best_cost < 0; ++pass) {
        for (int R = pass == 0 ? 1 : R0; R <= r_hi; ++R) {
            if (pass == 0 && ((R * L) % 32 != 0 || R * L < 64)) continue;
            const int T = ((R * L + 31) / 32) * 32;
            int per_sm = 0;
            if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, T, convrot::act_smem_bytes(T)) !=
                    cudaSuccess ||
                per_sm <= 0) {
                cudaGetLastError();
                continue;
            }
            const int64_t ctas = (M + R - 1) / R;
            const int64_t cap = static_cast<int64_t>(per_sm) * sms;
            const int64_t waves = (ctas + cap - 1) / cap;
            const int64_t cost = waves * R;
            if (best_cost < 0 || cost < best_cost || (pass == 0 && cost == best_cost)) {
                best_cost = cost;
                best_R = R;
                best_T = T;
                best_cap = static_cast<int>(cap);
            }
        }
    }
    *rows = best_R;
    *threads = best_T;
    *resident = best_cap;  // CTAs of this geometry the GPU holds at once (0: unknown)
}

// Launches with programmatic stream serialization: the kernel may begin while
// the previous kernel in the stream finishes; it waits (griddepcontrol.wait)
// before touching memory that kernel may use.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// As launch_pdl, with clusters of `cluster_x` CTAs along x.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl_cluster(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                               unsigned cluster_x, Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = cluster_x;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Extra grid-stride work of the activation launch: zeroing the workspace's
// counters, and widening the W4A4 linear's packed weights to int8 codes.
struct ActExtras {
    uint4 *zero16 = nullptr;
    int64_t n_zero16 = 0;
    const uint4 *w_packed = nullptr;
    uint4 *w_wide = nullptr;
    int64_t n_w16 = 0;
};

template <int LOG2B, int BITS, bool PACKED>
void launch_act(const void *X, int64_t M, int64_t K, void *Xq, float *xs, cudaStream_t st, int sms, int dev,
                const ActExtras &ex) {
    auto kern = convrot::act_rotate_quant_kernel<LOG2B, BITS, PACKED>;
    {
        static bool configured[kMaxDevices];
        static std::mutex mu;
        std::lock_guard<std::mutex> lock(mu);
        if (!configured[dev]) {
            cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, convrot::act_smem_bytes(1024));
            // the largest shared-memory carve-out, so occupancy is limited by registers only
            cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
            configured[dev] = true;
        }
    }
    int R, T, resident;
    act_geometry(kern, sms, M, K, &R, &T, &resident);
    const int64_t grid = (M + R - 1) / R;
    // a grid of more than one wave prefetches one wave ahead
    const int pf_ahead = (resident > 0 && grid > resident) ? resident : 0;
    launch_pdl(kern, dim3(static_cast<unsigned>(grid)), dim3(T), static_cast<size_t>(convrot::act_smem_bytes(T)), st,
               static_cast<const __half *>(X), M, static_cast<int>(K), R, Xq, xs, ex.zero16, ex.n_zero16, ex.w_packed,
               ex.w_wide, ex.n_w16, pf_ahead);
}

template <int BITS, bool PACKED>
void dispatch_act(int log2b, const void *X, int64_t M, int64_t K, void *Xq, float *xs, cudaStream_t st, int sms,
                  int dev, const ActExtras &ex) {
    switch (log2b) {
        case 0: launch_act<0, BITS, PACKED>(X, M, K, Xq, xs, st, sms, dev, ex); break;
        case 1: launch_act<1, BITS, PACKED>(X, M, K, Xq, xs, st, sms, dev, ex); break;
        case 2: launch_act<2, BITS, PACKED>(X, M, K, Xq, xs, st, sms, dev, ex); break;
        case 3: launch_act<3, BITS, PACKED>(X, M, K, Xq, xs, st, sms, dev, ex); break;
        case 4: launch_act<4, BITS, PACKED>(X, M, K, Xq, xs, st, sms, dev, ex); break;
        case 5: launch_act<5, BITS, PACKED>(X, M, K, Xq, xs, st, sms, dev, ex); break;
        case 6: launch_act<6, BITS, PACKED>(X, M, K, Xq, xs, st, sms, dev, ex); break;
        case 7: launch_act<7, BITS, PACKED>(X, M, K, Xq, xs, st, sms, dev, ex); break;
        default: launch_act<8, BITS, PACKED>(X, M, K, Xq, xs, st, sms, dev, ex); break;
    }
}

// Tensor-wise passes: see weight_rotate_quant_kernel (all null = row-wise).
struct WeightPass {
    const float *given_amax = nullptr;
    const int *given_alpha = nullptr;
    float *row_amax_out = nullptr;
    double *row_err_out = nullptr;
};

template <int LOG2B>
void launch_weight(const void *W, int dtype, int64_t N, int64_t K, int bits, int clip, void *Wq, float *ws,
                   cudaStream_t st, const WeightPass &ps) {
    int R, T;
    rotate_geometry(K, &R, &T);
    const int64_t grid = (N + R - 1) / R;
    convrot::weight_rotate_quant_kernel<LOG2B><<<static_cast<unsigned>(grid), T, 0, st>>>(
        W, dtype, N, static_cast<int>(K), R, bits, clip, Wq, ws, ps.given_amax, ps.given_alpha, ps.row_amax_out,
        ps.row_err_out);
}

void dispatch_weight(int log2b, const void *W, int dtype, int64_t N, int64_t K, int bits, int clip, void *Wq,
                     float *ws, cudaStream_t st, const WeightPass &ps = WeightPass()) {
    switch (log2b) {
        case 0: launch_weight<0>(W, dtype, N, K, bits, clip, Wq, ws, st, ps); break;
        case 1: launch_weight<1>(W, dtype, N, K, bits, clip, Wq, ws, st, ps); break;
        case 2: launch_weight<2>(W, dtype, N, K, bits, clip, Wq, ws, st, ps); break;
        case 3: launch_weight<3>(W, dtype, N, K, bits, clip, Wq, ws, st, ps); break;
        case 4: launch_weight<4>(W, dtype, N, K, bits, clip, Wq, ws, st, ps); break;
        case 5: launch_weight<5>(W, dtype, N, K, bits, clip, Wq, ws, st, ps); break;
        case 6: launch_weight<6>(W, dtype, N, K, bits, clip, Wq, ws, st, ps); break;
        case 7: launch_weight<7>(W, dtype, N, K, bits, clip, Wq, ws, st, ps); break;
        default: launch_weight<8>(W, dtype, N, K, bits, clip, Wq, ws, st, ps); break;
    }
}

// packed: int4 codes two per byte (bits = 4 only); otherwise one byte per code.
convrot_status_t rotate_quant_act_impl(const void *X, int64_t M, int64_t K, int block, int bits, bool packed,
                                       void *Xq, float *x_scale, cudaStream_t st, int sms, int dev,
                                       const ActExtras &ex = ActExtras()) {
    const int log2b = ilog2(block);
    if (bits == 8) dispatch_act<8, false>(log2b, X, M, K, Xq, x_scale, st, sms, dev, ex);
    else if (packed) dispatch_act<4, true>(log2b, X, M, K, Xq, x_scale, st, sms, dev, ex);
    else dispatch_act<4, false>(log2b, X, M, K, Xq, x_scale, st, sms, dev, ex);
    return launch_status("act_rotate_quant");
}

// ---------------------------------------------------------------- GEMM launch

// GEMM launch plan: operand order, tile width and K split.
struct GemmPlan {
    bool swap = false;  // feature-major (weights on the MMA's 128-row side)
    bool pair = false;  // token-major 256 x 256 tiles on CTA pairs (cta_group::2)
    bool gemv = false;  // at most 16 tokens with int8 activation codes: weight-streaming kernel
    int bn = 256;       // MMA N: output features (token-major) or tokens (feature-major)
    int splits = 1;
    int64_t tiles = 0;
    int streamk = 0;    // token-major stream-K: CTAs sharing the K steps of all tiles (0: off)
};

constexpr int kCounterWords = 512;               // stream-K / fused-panel counters in a linear's workspace
constexpr size_t kCounterBytes = kCounterWords * 4;
static_assert(kCounterBytes == convrot::kFuseMaxPanels * 4, "the fused linear's panel counters fill the counter area");
constexpr int64_t kSwapMaxTokens = 128;          // feature-major up to this many tokens
// K steps of 128 in a feature-major split-K slice (B200, CUDA-graph-timed: at
// K = 1024 splitting in two is 0.2-0.6 us slower than whole tiles, at K = 2048
// two slices beat four and eight, at K = 4096 four and eight tie)
constexpr int kMinSliceSteps = 8;
// Stream-K: the cost of the shared tiles (148 partial tiles of 128 KB stored and
// read back, ~5 us on B200), in 128-deep steps of a 256-wide tile: int8 weights
// / widened int4 weights (whose steps are slower).  Measured, CUDA-graph-timed,
// against the whole-tile plan: ViT-L widths at K = 1024 +5 us (int8 and int4),
// K = 4096 N = 1024 +1.1 us (int8) and -4.2 us (int4).
constexpr double kStreamKOverheadSteps8 = 16.0;
constexpr double kStreamKOverheadSteps4 = 9.0;

// Few tokens: feature-major tiles of 128 features x all the tokens (32, 64 or
// 128 columns), so that every weight byte is read once.  Where the tiles alone
// leave SMs idle, K is split over a cluster of 2, 4 or 8 CTAs (each slice at
// least kMinSliceSteps steps of 128), whose partial accumulators are added
// after shared-memory bulk copies between the cluster's CTAs.  Otherwise
// token-major 128 x 256 tiles,
// narrowed when narrower tiles finish in fewer rounds.  (Measured on B200 with
// CUDA-graph launches: feature-major wins up to 128 tokens, token-major from 192.)
GemmPlan plan_gemm(int sms, int64_t M, int64_t N, int64_t K, bool allow_split, bool w4 = false) {
    GemmPlan p;
    if (M <= kSwapMaxTokens) {
        p.swap = true;
        p.bn = M <= 32 ? 32 : (M <= 64 ? 64 : 128);
        p.tiles = (N + 127) / 128;
        // for the fewest tokens the weight-streaming kernel runs instead (int8
        // activation codes; the feature-major tiles stay for packed ones).
        // Measured on B200 (K = N = 4096, CUDA graphs): faster up to 4 tokens
        // with int8 weights (4.9 against 8.2 us at M = 1), up to 8 with int4
        p.gemv = M <= (w4 ? 8 : 4);
        if (!p.gemv) {
            int s = 8;
            while (s > 1 && (p.tiles * s > sms || K / 128 < static_cast<int64_t>(s) * kMinSliceSteps)) s /= 2;
            p.splits = s;
        }
        return p;
    }
    // tile width: fewest rounds of tiles weighted by a tile's measured relative
    // cost (B200, CUDA-graph-timed: a 192-wide tile takes 0.83 of a 256-wide
    // one's time with int8 weights, 0.80 with widened int4; a 128-wide one
    // 0.78 / 0.63), ties to the wider tile
    const int64_t tiles_m = (M + 127) / 128;
    const int widths[3] = {256, 192, 128};
    const double cost8[3] = {1.0, 0.83, 0.78}, cost4[3] = {1.0, 0.80, 0.63};
    double best = -1.0;
    for (int i = 0; i < 3; ++i) {
        const int bn = widths[i];
        if (bn > 128 && N < bn) continue;
        const int64_t tiles = tiles_m * ((N + bn - 1) / bn);
        const double c = static_cast<double>((tiles + sms - 1) / sms) * (w4 ? cost4[i] : cost8[i]);
        if (best < 0.0 || c < best - 1e-9) {
            best = c;
            p.bn = bn;
            p.tiles = tiles;
        }
    }
    // CTA pairs halve each SM's operand traffic, which pays where the main loop
    // dominates: deep K and at least two rounds of 256 x 256 tiles (int8
    // weights; with widened int4 weights pairs measured slower)
    const int64_t pair_tiles = ((M + 255) / 256) * ((N + 255) / 256);
    p.pair = p.bn == 256 && !w4 && K >= 1536 && pair_tiles >= sms;
    // Stream-K (needs the workspace's partial-tile slots): every SM takes an
    // equal share of the K steps of all 256-wide tiles, so a partly filled last
    // round of tiles costs nothing; each boundary between two SMs' shares
    // costs one partial tile stored and read back.  Used where it beats the
    // rounds of whole tiles (in 128-deep steps of a 256-wide tile) by 5 %,
    // which takes deep K (int4 weights from K = 4096, int8 from ~8192).
    const int64_t t256 = tiles_m * ((N + 255) / 256), nkb = K / 128;
    if (allow_split && !p.pair && N >= 256 && sms < convrot::kStreamKFlags && t256 >= sms && t256 % sms != 0 &&
        t256 * nkb < (int64_t(1) << 31)) {
        const double sk = static_cast<double>(t256) * static_cast<double>(nkb) / sms +
                          (w4 ? kStreamKOverheadSteps4 : kStreamKOverheadSteps8);
        if (sk < 0.95 * best * static_cast<double>(nkb)) {
            p.bn = 256;
            p.tiles = t256;
            p.streamk = sms;
        }
    }
    return p;
}

// The partial-tile slots of a stream-K GEMM (one 128 x BN int32 tile per
// boundary between CTAs; a feature-major split-K GEMM needs no global state).
size_t split_buffer_bytes(const GemmPlan &p, int64_t M, int64_t N) {
    (void)M;
    (void)N;
    return p.streamk > 0 ? static_cast<size_t>(p.streamk + 1) * 128 * p.bn * 4 : 0;
}

// The fused linear's activation input: the fp16 X, its block size and the
// panel counters in the workspace (the codes and scales go to the GEMM's Xc / sx).
struct FusePrologue {
    const void *X = nullptr;
    int log2b = 0;
    unsigned int *panels = nullptr;
};

// Block sizes the fused linear is built for (others take two launches).
constexpr bool fuse_block_supported(int log2b) { return log2b == 7; }

// The W4A4 linear over more than 128 tokens (token-major tiles) widens its
// packed weights once per call to int8 codes in the workspace, in its
// activation launch, and runs the int8-weight GEMM on them: every M tile would
// otherwise widen the same weight tiles again in shared memory.  The products
// are the same integers either way.
bool w4_prewidens(int64_t M) { return M > kSwapMaxTokens; }

// Offset of the widened weights: after the codes, scales, counters and the
// split buffer of the int8-weight plan.
size_t w4_wide_offset(int sms, int64_t M, int64_t K, int64_t N) {
    return round256(static_cast<size_t>(M) * K) + round256(static_cast<size_t>(M) * 4) + kCounterBytes +
           split_buffer_bytes(plan_gemm(sms, M, N, K, true, false), M, N);
}

// Xc: activation codes (M x K), Wc: weight codes (N x K); A4 / B4 of Cfg refer
// to the MMA's operands (token-major: A = activations; feature-major: A = weights).
// FL >= 0: fused prologue with block 2^FL and FB-wide activation codes (Xc and
// sx are then written by the kernel).
template <class Cfg, int FL = -1, int FB = 8>
convrot_status_t launch_gemm_cfg(DeviceInfo *info, int dev, const void *Xc, const void *Wc, int64_t M, int64_t N,
                                 int64_t K, const float *sx, const float *sw, const void *bias, void *Y,
                                 int32_t *acc_out, cudaStream_t st, int splits, int32_t *acc_buf,
                                 unsigned int *counters, int streamk = 0, const FusePrologue *fuse = nullptr,
                                 bool w_early = true) {
    const auto kern = convrot::gemm_i8_tcgen05_kernel<Cfg, FL, FB>;
    const __half *fx = fuse ? static_cast<const __half *>(fuse->X) : nullptr;
    int8_t *fq = fuse ? static_cast<int8_t *>(const_cast<void *>(Xc)) : nullptr;
    float *fs = fuse ? const_cast<float *>(sx) : nullptr;
    unsigned int *ff = fuse ? fuse->panels : nullptr;
    {
        static std::mutex mu;
        static bool done[kMaxDevices] = {};
        std::lock_guard<std::mutex> lock(mu);
        if (!done[dev]) {
            cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM_BYTES);
            CR_REQUIRE(e == cudaSuccess, CONVROT_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
            done[dev] = true;
        }
    }
    CUtensorMap ta, tb, ty;
    // int8 operands: 128-byte boxes with the 128B swizzle the MMA reads; packed
    // int4 operands: 64-byte boxes of dense rows for the converters
    const auto op_map = [&](CUtensorMap *m, const void *base, int64_t rows, int box_rows, bool packed) {
        return make_map(m, base, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, rows, packed ? K / 2 : K, box_rows,
                        packed ? Cfg::BK / 2 : Cfg::BK,
                        packed ? CU_TENSOR_MAP_SWIZZLE_NONE : CU_TENSOR_MAP_SWIZZLE_128B);
    };
    const int64_t rows_a = Cfg::SWAP ? N : M, rows_b = Cfg::SWAP ? M : N;
    CR_TRY(op_map(&ta, Cfg::SWAP ? Wc : Xc, rows_a, Cfg::BM, Cfg::A4));
    CR_TRY(op_map(&tb, Cfg::SWAP ? Xc : Wc, rows_b, Cfg::B_ROWS, Cfg::B4));
    if (Cfg::SWAP) ty = ta;  // stores go straight to Y
    else CR_TRY(make_map(&ty, Y, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, M, N, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B));
    const int64_t tiles = ((rows_a + Cfg::TILE_M - 1) / Cfg::TILE_M) * ((rows_b + Cfg::BN - 1) / Cfg::BN);
    if (Cfg::SWAP && splits > 1) {
        // the clusters of all tiles must be co-resident (one CTA per SM): fewer
        // K slices where the GPCs cannot place that many clusters of this size
        static std::mutex mu;
        static int max_clusters[kMaxDevices][4] = {};  // by log2 of the cluster size
        std::lock_guard<std::mutex> lock(mu);
        while (splits > 1) {
            const int lg = splits == 2 ? 1 : (splits == 4 ? 2 : 3);
            int &mc = max_clusters[dev][lg];
            if (mc == 0) {
                cudaLaunchConfig_t occ = {};
                occ.gridDim = dim3(static_cast<unsigned>(splits * (info->sms / splits)));
                occ.blockDim = dim3(Cfg::NUM_THREADS);
                occ.dynamicSmemBytes = Cfg::SMEM_BYTES;
                cudaLaunchAttribute attr[1];
                attr[0].id = cudaLaunchAttributeClusterDimension;
                attr[0].val.clusterDim.x = static_cast<unsigned>(splits);
                attr[0].val.clusterDim.y = 1;
                attr[0].val.clusterDim.z = 1;
                occ.attrs = attr;
                occ.numAttrs = 1;
                int n = 0;
                cudaError_t e = cudaOccupancyMaxActiveClusters(&n, kern, &occ);
                if (e != cudaSuccess) cudaGetLastError();
                mc = (e == cudaSuccess && n > 0) ? n : -1;
            }
            if (mc > 0 && tiles <= mc) break;
            splits /= 2;
        }
    }
    const int64_t units = tiles * splits;
    if (Cfg::PAIR) {
        // persistent: one cluster of two CTAs per co-resident pair of SMs
        static int max_clusters[kMaxDevices] = {};
        {
            static std::mutex mu;
            std::lock_guard<std::mutex> lock(mu);
            if (max_clusters[dev] == 0) {
                cudaLaunchConfig_t occ = {};
                occ.gridDim = dim3(2 * (info->sms / 2));
                occ.blockDim = dim3(Cfg::NUM_THREADS);
                occ.dynamicSmemBytes = Cfg::SMEM_BYTES;
                cudaLaunchAttribute attr[1];
                attr[0].id = cudaLaunchAttributeClusterDimension;
                attr[0].val.clusterDim.x = 2;
                attr[0].val.clusterDim.y = 1;
                attr[0].val.clusterDim.z = 1;
                occ.attrs = attr;
                occ.numAttrs = 1;
                int n = 0;
                cudaError_t e = cudaOccupancyMaxActiveClusters(&n, kern, &occ);
                CR_REQUIRE(e == cudaSuccess && n > 0, CONVROT_ERR_CUDA, "cudaOccupancyMaxActiveClusters: %s (%d)",
                           cudaGetErrorString(e), n);
                max_clusters[dev] = n;
            }
        }
        const int64_t clusters = units < max_clusters[dev] ? units : max_clusters[dev];
        launch_pdl_cluster(kern, dim3(static_cast<unsigned>(2 * clusters)), dim3(Cfg::NUM_THREADS), Cfg::SMEM_BYTES, st,
                           2u, ta, tb, ty, static_cast<int>(rows_a), static_cast<int>(rows_b), static_cast<int>(K), sx,
                           sw, static_cast<const __half *>(bias), static_cast<__half *>(Y), acc_out, splits, acc_buf,
                           counters, 0, fx, fq, fs, ff, w_early ? 1 : 0);
        return launch_status("gemm_i8_tcgen05 (CTA pairs)");
    }
    if (Cfg::SWAP && splits > 1) {
        // split K: one CTA per (tile, K slice), the slices of a tile in one cluster
        launch_pdl_cluster(kern, dim3(static_cast<unsigned>(units)), dim3(Cfg::NUM_THREADS), Cfg::SMEM_BYTES, st,
                           static_cast<unsigned>(splits), ta, tb, ty, static_cast<int>(rows_a),
                           static_cast<int>(rows_b), static_cast<int>(K), sx, sw, static_cast<const __half *>(bias),
                           static_cast<__half *>(Y), acc_out, splits, acc_buf, counters, 0, fx, fq, fs, ff,
                           w_early ? 1 : 0);
        return launch_status("gemm_i8_tcgen05 (split-K clusters)");
    }
    // persistent: one CTA per SM (stream-K: exactly the planned number of shares)
    const int grid = streamk > 0 ? streamk : static_cast<int>(units < info->sms ? units : info->sms);
    launch_pdl(kern, dim3(grid), dim3(Cfg::NUM_THREADS), Cfg::SMEM_BYTES, st, ta, tb, ty, static_cast<int>(rows_a),
               static_cast<int>(rows_b), static_cast<int>(K), sx, sw, static_cast<const __half *>(bias),
               static_cast<__half *>(Y), acc_out, splits, acc_buf, counters, streamk, fx, fq, fs, ff, w_early ? 1 : 0);
    return launch_status("gemm_i8_tcgen05");
}

// Weight-streaming GEMM for the fewest tokens (int8 activation codes; W4 =
// packed int4 weights): blocks of R output features, at most `max_warps`
// warps splitting K in 512-code chunks.
template <bool W4, int MT, int R>
convrot_status_t launch_gemv_mt(const void *Xc, const void *Wc, int64_t M, int64_t N, int64_t K, const float *sx,
                                const float *sw, const void *bias, void *Y, int32_t *acc_out, cudaStream_t st,
                                int64_t max_warps) {
    int64_t nw = K / convrot::kGemvChunk;
    nw = nw < 1 ? 1 : (nw > max_warps ? max_warps : nw);
    const int64_t grid = (N + R - 1) / R;
    launch_pdl(convrot::gemv_i8_kernel<W4, MT, R>, dim3(static_cast<unsigned>(grid)),
               dim3(static_cast<unsigned>(32 * nw)), 0, st, static_cast<const int8_t *>(Xc), sx,
               static_cast<const uint8_t *>(Wc), sw, static_cast<const __half *>(bias), static_cast<__half *>(Y),
               acc_out, static_cast<int>(M), static_cast<int>(N), static_cast<int>(K));
    return launch_status("gemv_i8");
}

// Features per block and warps per block (B200, CUDA graphs, weights beyond
// L2, the linear / its GEMM alone, us):
//  * int8 weights, 1-2 tokens: 4 features and at most 4 warps where the grid
//    is wide and K moderate (K = N = 4096: 1 token 6.37 / 4.40 -> 5.84 /
//    4.35, 2 tokens 6.77 -> 6.42 linear; 1 x 1024 -> 3072 3.50 -> 3.44),
//    and 2 features for one token from K = 4096 (K = N = 4096: 6.00 / 4.33
//    -> 5.83 / 4.10; 1 x 8192 -> 4096 GEMM alone 7.5 -> 6.8; at K = 1024
//    slower, 3.49 -> 3.78);
//  * the other 1-2 token cases (int4 weights among them): at most 8 warps
//    (1 x 16384 -> 4096 GEMM alone 12.2 against 14.5 with 4; int4 K = N =
//    4096 5.33 against 5.98) and 8 features, halved down to 2 while the grid
//    would hold fewer than 48 K threads, since the weight loads' latency is
//    covered by threads, not by bytes per thread (int8 1 x 4096 -> 1024
//    3.93 -> 3.77 with 4, 1 x 2048 -> 1024 3.48 -> 3.41 with 2; int4 1 x
//    4096 -> 1024 4.26 -> 3.88 and 1 x 1024 -> 3072 3.70 -> 3.48 with 4;
//    int4 K = N = 4096 stays at 8: 5.28, 6.38 with 4);
//  * 3-8 tokens: at most 4 warps (int8 3 / 4 tokens 8.11 / 8.62 -> 7.37 /
//    7.88, int4 4 / 8 tokens 8.05 / 13.1 -> 7.17 / 11.45 against 8 warps),
//    2 features up to 4 tokens (1 feature: 4 x 4096 -> 4096 7.99 -> 9.92);
//    5-8 tokens 4 features from N = 4096, else 2 (int4 8 x 1024 -> 3072
//    6.19 -> 5.82, 6 x 4096 -> 1024 8.51 -> 7.50; 8 x 4096 -> 4096 11.46
//    with 4, 14.2 with 2).
template <bool W4>
convrot_status_t launch_gemv(const void *Xc, const void *Wc, int64_t M, int64_t N, int64_t K, const float *sx,
                             const float *sw, const void *bias, void *Y, int32_t *acc_out, cudaStream_t st) {
    if (M <= 2) {
        if (!W4 && N >= 2048 && K <= 8192) {
            if (M <= 1 && K >= 4096)
                return launch_gemv_mt<W4, 1, 2>(Xc, Wc, M, N, K, sx, sw, bias, Y, acc_out, st, 4);
            if (M <= 1) return launch_gemv_mt<W4, 1, 4>(Xc, Wc, M, N, K, sx, sw, bias, Y, acc_out, st, 4);
            return launch_gemv_mt<W4, 2, 4>(Xc, Wc, M, N, K, sx, sw, bias, Y, acc_out, st, 4);
        }
        int64_t nw = K / convrot::kGemvChunk;
        nw = nw < 1 ? 1 : (nw > 8 ? 8 : nw);
        int r = 8;
        while (r > 2 && (N + r - 1) / r * nw * 32 < 48 * 1024) r /= 2;
        if (M <= 1) {
            if (r == 8) return launch_gemv_mt<W4, 1, 8>(Xc, Wc, M, N, K, sx, sw, bias, Y, acc_out, st, 8);
            if (r == 4) return launch_gemv_mt<W4, 1, 4>(Xc, Wc, M, N, K, sx, sw, bias, Y, acc_out, st, 8);
            return launch_gemv_mt<W4, 1, 2>(Xc, Wc, M, N, K, sx, sw, bias, Y, acc_out, st, 8);
        }
        if (r == 8) return launch_gemv_mt<W4, 2, 8>(Xc, Wc, M, N, K, sx, sw, bias, Y, acc_out, st, 8);
        if (r == 4) return launch_gemv_mt<W4, 2, 4>(Xc, Wc, M, N, K, sx, sw, bias, Y, acc_out, st, 8);
        return launch_gemv_mt<W4, 2, 2>(Xc, Wc, M, N, K, sx, sw, bias, Y, acc_out, st, 8);
    }
    if (M <= 4) return launch_gemv_mt<W4, 4, 2>(Xc, Wc, M, N, K, sx, sw, bias, Y, acc_out, st, 4);
    if (M <= 8 && N >= 4096) return launch_gemv_mt<W4, 8, 4>(Xc, Wc, M, N, K, sx, sw, bias, Y, acc_out, st, 4);
    if (M <= 8) return launch_gemv_mt<W4, 8, 2>(Xc, Wc, M, N, K, sx, sw, bias, Y, acc_out, st, 4);
    return CONVROT_ERR_UNSUPPORTED;  // the planner hands at most 8 tokens to this kernel
}

// X4 / W4: activation / weight codes packed int4.
// The fused W8A8 linear (token-major, whole tiles, block 2^7): the plan's tile
// width and pair choice, launched as one kernel whose activation warps rotate
// and quantize X beside the main loop.
convrot_status_t launch_gemm_fused(DeviceInfo *info, int dev, const void *Xc, const void *Wc, int64_t M, int64_t N,
                                   int64_t K, const float *sx, const float *sw, const void *bias, void *Y,
                                   cudaStream_t st, const GemmPlan &p, const FusePrologue &fz) {
    using convrot::GemmCfg;
    if (p.bn == 192)
        return launch_gemm_cfg<GemmCfg<192, false, false, false, false, false, true>, 7, 8>(
            info, dev, Xc, Wc, M, N, K, sx, sw, bias, Y, nullptr, st, 1, nullptr, nullptr, 0, &fz);
    if (p.bn == 256) {
        if (p.pair)
            return launch_gemm_cfg<GemmCfg<256, false, false, false, true, false, true>, 7, 8>(
                info, dev, Xc, Wc, M, N, K, sx, sw, bias, Y, nullptr, st, 1, nullptr, nullptr, 0, &fz);
        return launch_gemm_cfg<GemmCfg<256, false, false, false, false, false, true>, 7, 8>(
            info, dev, Xc, Wc, M, N, K, sx, sw, bias, Y, nullptr, st, 1, nullptr, nullptr, 0, &fz);
    }
    return launch_gemm_cfg<GemmCfg<128, false, false, false, false, false, true>, 7, 8>(
        info, dev, Xc, Wc, M, N, K, sx, sw, bias, Y, nullptr, st, 1, nullptr, nullptr, 0, &fz);
}

// K limit of the fused linear (one row fits its activation warps once).
// K limit of the fused linear.  One row fits its activation warps once up to
// 8192 features, but beyond 2048 a unit holds fewer than 4 rows and the eight
// activation warps would take longer than the main loop they run beside.
constexpr int64_t kFuseMaxK = 2048;
static_assert(kFuseMaxK <= convrot::GemmCfg<256, false, false, false, false, false, true>::ACT_MAX_K,
              "a row fits the activation warps");

template <bool X4, bool W4>
convrot_status_t launch_gemm(DeviceInfo *info, int dev, const void *Xc, const void *Wc, int64_t M, int64_t N,
                             int64_t K, const float *sx, const float *sw, const void *bias, void *Y,
                             int32_t *acc_out, cudaStream_t st, const GemmPlan &p, int32_t *acc_buf = nullptr,
                             unsigned int *counters = nullptr, bool w_early = true) {
    using convrot::GemmCfg;
    if constexpr (!X4) {
        if (p.gemv) return launch_gemv<W4>(Xc, Wc, M, N, K, sx, sw, bias, Y, acc_out, st);
    }
    if (p.swap) {
        if (p.bn == 32)
            return launch_gemm_cfg<GemmCfg<32, W4, X4, true>>(info, dev, Xc, Wc, M, N, K, sx, sw, bias, Y, acc_out, st,
                                                              p.splits, nullptr, nullptr, 0, nullptr, w_early);
        if (p.bn == 64)
            return launch_gemm_cfg<GemmCfg<64, W4, X4, true>>(info, dev, Xc, Wc, M, N, K, sx, sw, bias, Y, acc_out, st,
                                                              p.splits, nullptr, nullptr, 0, nullptr, w_early);
        return launch_gemm_cfg<GemmCfg<128, W4, X4, true>>(info, dev, Xc, Wc, M, N, K, sx, sw, bias, Y, acc_out, st,
                                                           p.splits, nullptr, nullptr, 0, nullptr, w_early);
    }
    if constexpr (!X4) {  // (stream-K needs a linear's workspace, whose activation codes are bytes)
        if (p.streamk > 0)  // token-major, single CTAs, 256-wide tiles
            return launch_gemm_cfg<GemmCfg<256, false, W4, false, false, true>>(
                info, dev, Xc, Wc, M, N, K, sx, sw, bias, Y, acc_out, st, 1, acc_buf, counters, p.streamk, nullptr,
                w_early);
    }
    if (p.bn == 192)
        return launch_gemm_cfg<GemmCfg<192, X4, W4>>(info, dev, Xc, Wc, M, N, K, sx, sw, bias, Y, acc_out, st, 1,
                                                     nullptr, nullptr, 0, nullptr, w_early);
    if (p.bn == 256) {
        if constexpr (!X4 && !W4) {
            if (p.pair)
                return launch_gemm_cfg<GemmCfg<256, false, false, false, true>>(info, dev, Xc, Wc, M, N, K, sx, sw,
                                                                                bias, Y, acc_out, st, 1, nullptr,
                                                                                nullptr, 0, nullptr, w_early);
        }
        return launch_gemm_cfg<GemmCfg<256, X4, W4>>(info, dev, Xc, Wc, M, N, K, sx, sw, bias, Y, acc_out, st, 1,
                                                     nullptr, nullptr, 0, nullptr, w_early);
    }
    return launch_gemm_cfg<GemmCfg<128, X4, W4>>(info, dev, Xc, Wc, M, N, K, sx, sw, bias, Y, acc_out, st, 1, nullptr,
                                                 nullptr, 0, nullptr, w_early);
}

convrot_status_t check_gemm_args(const void *Xq, const float *xs, int64_t M, const void *Wq, const float *ws,
                                 int64_t N, int64_t K, const void *bias, const void *Y) {
    CR_TRY(check_shape(M, K, 1, "M"));
    CR_REQUIRE(N >= 0 && N < (int64_t(1) << 31), CONVROT_ERR_INVALID_ARG, "N = %lld out of [0, 2^31)",
               static_cast<long long>(N));
    CR_REQUIRE(N % 8 == 0, CONVROT_ERR_INVALID_ARG, "N = %lld must be a multiple of 8", static_cast<long long>(N));
    if (M == 0 || N == 0) return ok();
    CR_REQUIRE(Xq && xs && Wq && ws && Y, CONVROT_ERR_INVALID_ARG, "null pointer argument");
    CR_REQUIRE(aligned(Xq, 16) && aligned(Wq, 16) && aligned(Y, 16), CONVROT_ERR_ALIGNMENT,
               "codes and Y must be 16-byte aligned");
    CR_REQUIRE(aligned(xs, 4), CONVROT_ERR_ALIGNMENT, "x_scale must be 4-byte aligned");
    CR_REQUIRE(aligned(ws, 16), CONVROT_ERR_ALIGNMENT, "w_scale must be 16-byte aligned");
    CR_REQUIRE(bias == nullptr || aligned(bias, 16), CONVROT_ERR_ALIGNMENT, "bias must be 16-byte aligned");
    return ok();
}

}  // namespace

// =============================================================================
// C ABI
// =============================================================================

extern "C" {

const char *convrot_status_string(convrot_status_t s) {
    switch (s) {
        case CONVROT_OK: return "ok";
        case CONVROT_ERR_INVALID_ARG: return "invalid argument";
        case CONVROT_ERR_UNSUPPORTED: return "unsupported";
        case CONVROT_ERR_ALIGNMENT: return "misaligned pointer";
        case CONVROT_ERR_CUDA: return "CUDA error";
        case CONVROT_ERR_TIMEOUT: return "device wait timed out";
        case CONVROT_ERR_WORKSPACE: return "workspace missing or too small";
    }
    return "unknown status";
}

const char *convrot_last_error(void) { return g_last_error.c_str(); }

int convrot_version(void) { return kVersion; }

size_t convrot_workspace_bytes(int64_t M, int64_t K, int bits) {
    if (M < 0 || K <= 0 || (bits != 8 && bits != 4)) return 0;
    // the linears keep one byte per activation code (int4 codes are widened
    // once here instead of in every GEMM tile that reads them)
    const size_t codes = static_cast<size_t>(M) * static_cast<size_t>(K);
    return round256(codes) + round256(static_cast<size_t>(M) * 4);
}

size_t convrot_linear_workspace_bytes(int64_t M, int64_t K, int64_t N, int bits) {
    const size_t base = convrot_workspace_bytes(M, K, bits);
    if (base == 0 || N < 0) return 0;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) {
        int v = 0;
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && v > 0) sms = v;
    } else {
        cudaGetLastError();
    }
    if (M == 0 || N == 0 || K % 128 != 0 || K < 128) return base + kCounterBytes;
    if (bits == 4 && w4_prewidens(M)) return w4_wide_offset(sms, M, K, N) + round256(static_cast<size_t>(N) * K);
    return base + kCounterBytes + split_buffer_bytes(plan_gemm(sms, M, N, K, true, bits == 4), M, N);
}

convrot_status_t convrot_quantize_weight(const void *W, int w_dtype, int64_t N, int64_t K, int block, int bits,
                                         int clip_mode, void *Wq, float *w_scale, void *stream) {
    g_last_error.clear();
    CR_TRY(check_shape(N, K, block, "N"));
    CR_TRY(check_bits(bits));
    CR_REQUIRE(w_dtype >= CONVROT_DTYPE_F16 && w_dtype <= CONVROT_DTYPE_F32, CONVROT_ERR_INVALID_ARG,
               "w_dtype = %d is not one of fp16 / bf16 / fp32", w_dtype);
    CR_REQUIRE(clip_mode == CONVROT_CLIP_ABSMAX || clip_mode == CONVROT_CLIP_MSE, CONVROT_ERR_INVALID_ARG,
               "clip_mode = %d", clip_mode);
    if (N == 0) return ok();
    CR_REQUIRE(W && Wq && w_scale, CONVROT_ERR_INVALID_ARG, "null pointer argument");
    CR_REQUIRE(aligned(W, 16) && aligned(Wq, 16), CONVROT_ERR_ALIGNMENT, "W and Wq must be 16-byte aligned");
    CR_REQUIRE(aligned(w_scale, 4), CONVROT_ERR_ALIGNMENT, "w_scale must be 4-byte aligned");
    int dev;
    DeviceInfo *info;
    CR_TRY(current_device(&dev, &info));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    dispatch_weight(ilog2(block), W, w_dtype, N, K, bits, clip_mode, Wq, w_scale, st);
    return launch_status("weight_rotate_quant");
}

size_t convrot_tensorwise_workspace_bytes(int64_t N, int clip_mode) {
    if (N < 0 || (clip_mode != CONVROT_CLIP_ABSMAX && clip_mode != CONVROT_CLIP_MSE)) return 0;
    size_t b = round256(static_cast<size_t>(N) * 4) + 256;  // row absmax, then the tensor's absmax and clip index
    if (clip_mode == CONVROT_CLIP_MSE) b += round256(static_cast<size_t>(N) * convrot::kMseGrid * 8);
    return b;
}

convrot_status_t convrot_quantize_weight_tensorwise(const void *W, int w_dtype, int64_t N, int64_t K, int block,
                                                    int bits, int clip_mode, void *Wq, float *w_scale,
                                                    void *workspace, size_t workspace_bytes, void *stream) {
    g_last_error.clear();
    CR_TRY(check_shape(N, K, block, "N"));
    CR_TRY(check_bits(bits));
    CR_REQUIRE(w_dtype >= CONVROT_DTYPE_F16 && w_dtype <= CONVROT_DTYPE_F32, CONVROT_ERR_INVALID_ARG,
               "w_dtype = %d is not one of fp16 / bf16 / fp32", w_dtype);
    CR_REQUIRE(clip_mode == CONVROT_CLIP_ABSMAX || clip_mode == CONVROT_CLIP_MSE, CONVROT_ERR_INVALID_ARG,
               "clip_mode = %d", clip_mode);
    if (N == 0) return ok();
    CR_REQUIRE(W && Wq && w_scale, CONVROT_ERR_INVALID_ARG, "null pointer argument");
    CR_REQUIRE(aligned(W, 16) && aligned(Wq, 16), CONVROT_ERR_ALIGNMENT, "W and Wq must be 16-byte aligned");
    CR_REQUIRE(aligned(w_scale, 4), CONVROT_ERR_ALIGNMENT, "w_scale must be 4-byte aligned");
    const size_t need = convrot_tensorwise_workspace_bytes(N, clip_mode);
    CR_REQUIRE(workspace != nullptr && workspace_bytes >= need, CONVROT_ERR_WORKSPACE,
               "workspace of %zu bytes given, %zu needed", workspace_bytes, need);
    CR_REQUIRE(aligned(workspace, 16), CONVROT_ERR_ALIGNMENT, "workspace must be 16-byte aligned");
    int dev;
    DeviceInfo *info;
    CR_TRY(current_device(&dev, &info));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint8_t *wsp = static_cast<uint8_t *>(workspace);
    float *row_amax = reinterpret_cast<float *>(wsp);
    float *g_amax = reinterpret_cast<float *>(wsp + round256(static_cast<size_t>(N) * 4));
    int *g_alpha = reinterpret_cast<int *>(g_amax + 4);
    double *row_err = reinterpret_cast<double *>(wsp + round256(static_cast<size_t>(N) * 4) + 256);
    const int log2b = ilog2(block);
    WeightPass stats;
    stats.row_amax_out = row_amax;
    dispatch_weight(log2b, W, w_dtype, N, K, bits, clip_mode, Wq, w_scale, st, stats);
    convrot::amax_reduce_kernel<<<1, 1024, 0, st>>>(row_amax, N, g_amax);
    WeightPass quant;
    quant.given_amax = g_amax;
    if (clip_mode == CONVROT_CLIP_MSE) {
        WeightPass errs;
        errs.given_amax = g_amax;
        errs.row_err_out = row_err;
        dispatch_weight(log2b, W, w_dtype, N, K, bits, clip_mode, Wq, w_scale, st, errs);
        convrot::err_argmin_kernel<<<1, 64, 0, st>>>(row_err, N, g_alpha);
        quant.given_alpha = g_alpha;
    }
    dispatch_weight(log2b, W, w_dtype, N, K, bits, clip_mode, Wq, w_scale, st, quant);
    return launch_status("weight_rotate_quant (tensor-wise)");
}

convrot_status_t convrot_rotate_quant_act(const void *X, int64_t M, int64_t K, int block, int bits, void *Xq,
                                          float *x_scale, void *stream) {
    g_last_error.clear();
    CR_TRY(check_shape(M, K, block, "M"));
    CR_TRY(check_bits(bits));
    if (M == 0) return ok();
    CR_REQUIRE(X && Xq && x_scale, CONVROT_ERR_INVALID_ARG, "null pointer argument");
    CR_REQUIRE(aligned(X, 16) && aligned(Xq, 16), CONVROT_ERR_ALIGNMENT, "X and Xq must be 16-byte aligned");
    CR_REQUIRE(aligned(x_scale, 4), CONVROT_ERR_ALIGNMENT, "x_scale must be 4-byte aligned");
    int dev;
    DeviceInfo *info;
    CR_TRY(current_device(&dev, &info));
    return rotate_quant_act_impl(X, M, K, block, bits, bits == 4, Xq, x_scale, static_cast<cudaStream_t>(stream),
                                 info->sms, dev);
}

// Workspace layout of the linears: activation codes (one byte each); at the
// next 256-byte boundary the per-token scales; then (when the workspace is
// large enough) kCounterWords counters and the stream-K partial-tile slots.
static void workspace_parts(void *workspace, int64_t M, int64_t K, void **xq, float **xs,
                            unsigned int **counters = nullptr, int32_t **acc_buf = nullptr) {
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    *xq = ws;
    *xs = reinterpret_cast<float *>(ws + round256(static_cast<size_t>(M) * K));
    uint8_t *extra = ws + round256(static_cast<size_t>(M) * K) + round256(static_cast<size_t>(M) * 4);
    if (counters) *counters = reinterpret_cast<unsigned int *>(extra);
    if (acc_buf) *acc_buf = reinterpret_cast<int32_t *>(extra + kCounterBytes);
}

static convrot_status_t check_linear_shape(int64_t M, int64_t K, int block, int bits, int64_t N) {
    CR_TRY(check_shape(M, K, block, "M"));
    CR_TRY(check_bits(bits));
    CR_REQUIRE(N >= 0 && N < (int64_t(1) << 31) && N % 8 == 0, CONVROT_ERR_INVALID_ARG,
               "N = %lld must be a multiple of 8 in [0, 2^31)", static_cast<long long>(N));
    return ok();
}

static convrot_status_t check_workspace(const void *workspace, size_t workspace_bytes, int64_t M, int64_t K,
                                        int bits) {
    const size_t need = convrot_workspace_bytes(M, K, bits);
    CR_REQUIRE(workspace != nullptr && workspace_bytes >= need, CONVROT_ERR_WORKSPACE,
               "workspace of %zu bytes given, %zu needed", workspace_bytes, need);
    CR_REQUIRE(aligned(workspace, 16), CONVROT_ERR_ALIGNMENT, "workspace must be 16-byte aligned");
    return ok();
}

// n_features: the GEMM half's N where known (needed to widen weights).
// wide: the packed int4 weights (N x K/2) to widen into the workspace (see
// w4_prewidens), or null.
static convrot_status_t linear_act_impl(const void *X, int64_t M, int64_t K, int block, int bits, void *workspace,
                                        size_t workspace_bytes, cudaStream_t st, int64_t n_features = -1,
                                        const void *wide = nullptr) {
    CR_REQUIRE(X != nullptr, CONVROT_ERR_INVALID_ARG, "null pointer argument");
    CR_REQUIRE(aligned(X, 16), CONVROT_ERR_ALIGNMENT, "X must be 16-byte aligned");
    CR_TRY(check_workspace(workspace, workspace_bytes, M, K, bits));
    int dev;
    DeviceInfo *info;
    CR_TRY(current_device(&dev, &info));
    void *xq;
    float *xs;
    unsigned int *counters;
    workspace_parts(workspace, M, K, &xq, &xs, &counters);
    // the counters that follow the codes and scales are zeroed here for the
    // GEMM half (stream-K's partial slots are written before they are read)
    const size_t base = convrot_workspace_bytes(M, K, bits);
    size_t zero_bytes = 0;
    if (workspace_bytes > base)
        zero_bytes = (workspace_bytes - base < kCounterBytes ? workspace_bytes - base : kCounterBytes) & ~size_t(15);
    ActExtras ex;
    ex.zero16 = zero_bytes ? reinterpret_cast<uint4 *>(counters) : nullptr;
    ex.n_zero16 = static_cast<int64_t>(zero_bytes / 16);
    if (wide != nullptr) {
        ex.w_packed = static_cast<const uint4 *>(wide);
        ex.w_wide = reinterpret_cast<uint4 *>(static_cast<uint8_t *>(workspace) +
                                              w4_wide_offset(info->sms, M, K, n_features));
        ex.n_w16 = n_features * K / 32;  // 16 packed bytes (32 codes) per unit
    }
    return rotate_quant_act_impl(X, M, K, block, bits, false, xq, xs, st, info->sms, dev, ex);
}

// The GEMM plan of a linear's second launch: stream-K only when the workspace
// holds the counters (which the activation half zeroed) and the partial slots.
static GemmPlan two_launch_plan(int sms, int64_t M, int64_t N, int64_t K, int bits, size_t workspace_bytes) {
    GemmPlan p = plan_gemm(sms, M, N, K, true, bits == 4);
    const size_t base = convrot_workspace_bytes(M, K, bits) + kCounterBytes;
    if (p.streamk > 0 && workspace_bytes < base + split_buffer_bytes(p, M, N))
        p = plan_gemm(sms, M, N, K, false, bits == 4);
    return p;
}

// Whether a linear runs as one fused launch (token-major tiles for more than
// 128 tokens, a block size the prologue is built for, K within its consumer
// warps' reach and a workspace with room for the per-CTA flag words, which
// live in the split-K counter area that this plan does not use), and its plan.
static bool fused_plan(int sms, int64_t M, int64_t K, int64_t N, int bits, int block, size_t workspace_bytes,
                       GemmPlan *plan) {
    if (M <= kSwapMaxTokens || !fuse_block_supported(ilog2(block)) || K > kFuseMaxK) return false;
    if (bits != 8) return false;
    if ((M + 127) / 128 > convrot::kFuseMaxPanels) return false;
    if (workspace_bytes < convrot_workspace_bytes(M, K, bits) + kCounterBytes) return false;
    const GemmPlan p = plan_gemm(sms, M, N, K, false, bits == 4);  // whole tiles: no split state
    if (p.swap || p.gemv) return false;
    *plan = p;
    return true;
}

static convrot_status_t linear_gemm_impl(const void *workspace, size_t workspace_bytes, int64_t M, int64_t K,
                                         int bits, const void *Wq, const float *w_scale, int64_t N,
                                         const void *bias, void *Y, cudaStream_t st, bool w_early = true) {
    CR_TRY(check_workspace(workspace, workspace_bytes, M, K, bits));
    void *xq;
    float *xs;
    unsigned int *counters;
    int32_t *acc_buf;
    workspace_parts(const_cast<void *>(workspace), M, K, &xq, &xs, &counters, &acc_buf);
    CR_TRY(check_gemm_args(xq, xs, M, Wq, w_scale, N, K, bias, Y));
    int dev;
    DeviceInfo *info;
    CR_TRY(current_device(&dev, &info));
    const GemmPlan p = two_launch_plan(info->sms, M, N, K, bits, workspace_bytes);
    if (bits == 8)
        return launch_gemm<false, false>(info, dev, xq, Wq, M, N, K, xs, w_scale, bias, Y, nullptr, st, p, acc_buf,
                                         counters, w_early);
    return launch_gemm<false, true>(info, dev, xq, Wq, M, N, K, xs, w_scale, bias, Y, nullptr, st, p, acc_buf,
                                    counters, w_early);
}

static convrot_status_t linear_impl(int bits, const void *X, int64_t M, int64_t K, const void *Wq,
                                    const float *w_scale, int64_t N, const void *bias, int block, void *Y,
                                    void *workspace, size_t workspace_bytes, void *stream) {
    g_last_error.clear();
    CR_TRY(check_linear_shape(M, K, block, bits, N));
    if (M == 0 || N == 0) return ok();
    CR_REQUIRE(X && Wq && w_scale && Y, CONVROT_ERR_INVALID_ARG, "null pointer argument");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (bits == 4 && w4_prewidens(M) && workspace != nullptr) {
        CR_REQUIRE(aligned(Wq, 16), CONVROT_ERR_ALIGNMENT, "Wq must be 16-byte aligned");
        int dev;
        DeviceInfo *info;
        CR_TRY(current_device(&dev, &info));
        const size_t off = w4_wide_offset(info->sms, M, K, N);
        if (workspace_bytes >= off + round256(static_cast<size_t>(N) * K)) {
            // the activation launch also widens the weights; the int8-weight GEMM follows
            CR_TRY(linear_act_impl(X, M, K, block, 4, workspace, workspace_bytes, st, N, Wq));
            const int8_t *wide = static_cast<const int8_t *>(workspace) + off;
            // (the widened weights come from the activation launch: no early prefetch)
            return linear_gemm_impl(workspace, workspace_bytes, M, K, 8, wide, w_scale, N, bias, Y, st, false);
        }
    }
    CR_TRY(linear_act_impl(X, M, K, block, bits, workspace, workspace_bytes, st, N));
    return linear_gemm_impl(workspace, workspace_bytes, M, K, bits, Wq, w_scale, N, bias, Y, st);
}

convrot_status_t convrot_linear_quant_act(const void *X, int64_t M, int64_t K, int block, int bits, void *workspace,
                                          size_t workspace_bytes, void *stream) {
    g_last_error.clear();
    CR_TRY(check_shape(M, K, block, "M"));
    CR_TRY(check_bits(bits));
    if (M == 0) return ok();
    return linear_act_impl(X, M, K, block, bits, workspace, workspace_bytes, static_cast<cudaStream_t>(stream));
}

convrot_status_t convrot_linear_gemm(const void *workspace, size_t workspace_bytes, int64_t M, int64_t K, int bits,
                                     const void *Wq, const float *w_scale, int64_t N, const void *bias, void *Y,
                                     void *stream) {
    g_last_error.clear();
    CR_TRY(check_linear_shape(M, K, 1, bits, N));
    if (M == 0 || N == 0) return ok();
    return linear_gemm_impl(workspace, workspace_bytes, M, K, bits, Wq, w_scale, N, bias, Y,
                            static_cast<cudaStream_t>(stream));
}

convrot_status_t convrot_linear_w8a8(const void *X, int64_t M, int64_t K, const int8_t *Wq, const float *w_scale,
                                     int64_t N, const void *bias, int block, void *Y, void *workspace,
                                     size_t workspace_bytes, void *stream) {
    return linear_impl(8, X, M, K, Wq, w_scale, N, bias, block, Y, workspace, workspace_bytes, stream);
}

convrot_status_t convrot_linear_w4a4(const void *X, int64_t M, int64_t K, const uint8_t *Wq, const float *w_scale,
                                     int64_t N, const void *bias, int block, void *Y, void *workspace,
                                     size_t workspace_bytes, void *stream) {
    return linear_impl(4, X, M, K, Wq, w_scale, N, bias, block, Y, workspace, workspace_bytes, stream);
}

convrot_status_t convrot_linear_w8a8_fused(const void *X, int64_t M, int64_t K, const int8_t *Wq,
                                           const float *w_scale, int64_t N, const void *bias, int block, void *Y,
                                           void *workspace, size_t workspace_bytes, void *stream) {
    g_last_error.clear();
    CR_TRY(check_linear_shape(M, K, block, 8, N));
    if (M == 0 || N == 0) return ok();
    CR_REQUIRE(X && Wq && w_scale && Y, CONVROT_ERR_INVALID_ARG, "null pointer argument");
    const size_t need = convrot_workspace_bytes(M, K, 8) + kCounterBytes;
    CR_REQUIRE(workspace != nullptr && workspace_bytes >= need, CONVROT_ERR_WORKSPACE,
               "workspace of %zu bytes given, %zu needed (codes, scales and the panel counters)", workspace_bytes,
               need);
    CR_REQUIRE(aligned(workspace, 16), CONVROT_ERR_ALIGNMENT, "workspace must be 16-byte aligned");
    CR_REQUIRE(aligned(X, 16), CONVROT_ERR_ALIGNMENT, "X must be 16-byte aligned");
    CR_REQUIRE(M > kSwapMaxTokens && block == 128 && K <= kFuseMaxK && (M + 127) / 128 <= convrot::kFuseMaxPanels,
               CONVROT_ERR_UNSUPPORTED,
               "the fused linear takes more than %lld tokens, block 128, K <= %lld and at most %d panels "
               "(M = %lld, K = %lld, block = %d)",
               static_cast<long long>(kSwapMaxTokens), static_cast<long long>(kFuseMaxK), convrot::kFuseMaxPanels,
               static_cast<long long>(M), static_cast<long long>(K), block);
    int dev;
    DeviceInfo *info;
    CR_TRY(current_device(&dev, &info));
    GemmPlan p;
    CR_REQUIRE(fused_plan(info->sms, M, K, N, 8, block, workspace_bytes, &p), CONVROT_ERR_UNSUPPORTED,
               "no fused plan for M = %lld, N = %lld, K = %lld", static_cast<long long>(M), static_cast<long long>(N),
               static_cast<long long>(K));
    void *xq;
    float *xs;
    unsigned int *counters;
    workspace_parts(workspace, M, K, &xq, &xs, &counters);
    CR_TRY(check_gemm_args(xq, xs, M, Wq, w_scale, N, K, bias, Y));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // zero the panel counters (programmatic launch: overlaps the previous kernel's tail)
    const int panels = static_cast<int>((M + 127) / 128);
    launch_pdl(convrot::fuse_zero_kernel, dim3(1), dim3(256), 0, st, counters, panels);
    CR_TRY(launch_status("fuse_zero"));
    FusePrologue fz;
    fz.X = X;
    fz.log2b = ilog2(block);
    fz.panels = counters;
    return launch_gemm_fused(info, dev, xq, Wq, M, N, K, xs, w_scale, bias, Y, st, p, fz);
}

static convrot_status_t gemm_impl(bool w4, const void *Xq, const float *x_scale, int64_t M, const void *Wq,
                                  const float *w_scale, int64_t N, int64_t K, const void *bias, void *Y,
                                  int32_t *acc_out, void *stream) {
    g_last_error.clear();
    CR_TRY(check_gemm_args(Xq, x_scale, M, Wq, w_scale, N, K, bias, Y));
    if (M == 0 || N == 0) return ok();
    CR_REQUIRE(acc_out == nullptr || aligned(acc_out, 16), CONVROT_ERR_ALIGNMENT, "acc_out must be 16-byte aligned");
    int dev;
    DeviceInfo *info;
    CR_TRY(current_device(&dev, &info));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const GemmPlan p = plan_gemm(info->sms, M, N, K, false, w4);  // no workspace: no split-K
    if (w4) return launch_gemm<true, true>(info, dev, Xq, Wq, M, N, K, x_scale, w_scale, bias, Y, acc_out, st, p);
    return launch_gemm<false, false>(info, dev, Xq, Wq, M, N, K, x_scale, w_scale, bias, Y, acc_out, st, p);
}

convrot_status_t convrot_gemm_w8a8(const int8_t *Xq, const float *x_scale, int64_t M, const int8_t *Wq,
                                   const float *w_scale, int64_t N, int64_t K, const void *bias, void *Y,
                                   int32_t *acc_out, void *stream) {
    return gemm_impl(false, Xq, x_scale, M, Wq, w_scale, N, K, bias, Y, acc_out, stream);
}

convrot_status_t convrot_gemm_w4a4(const uint8_t *Xq, const float *x_scale, int64_t M, const uint8_t *Wq,
                                   const float *w_scale, int64_t N, int64_t K, const void *bias, void *Y,
                                   int32_t *acc_out, void *stream) {
    return gemm_impl(true, Xq, x_scale, M, Wq, w_scale, N, K, bias, Y, acc_out, stream);
}

// ---------------------------------------------------------------------------
// Allocation-free W8A8 linear.  Some callers cannot allocate device memory at
// all -- a plugin inside a host framework that owns every byte of the GPU and
// hands out no allocator, or a latency-critical path where an allocation (and
// the device synchronization it can imply) is not allowed.  For them this entry
// point keeps the activation codes and per-token scales in one fixed array
// compiled into the library instead of a caller workspace.
// ---------------------------------------------------------------------------

static constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;  // 16 MiB on every device that loads the library
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];
static void *g_noalloc_ptr[kMaxDevices];
static std::mutex g_noalloc_mutex;

convrot_status_t convrot_linear_w8a8_noalloc(const void *X, int64_t M, int64_t K, const int8_t *Wq,
                                             const float *w_scale, int64_t N, const void *bias, int block, void *Y,
                                             void *stream) {
    g_last_error.clear();
    CR_TRY(check_shape(M, K, block, "M"));
    CR_REQUIRE(N >= 0 && N < (int64_t(1) << 31) && N % 8 == 0, CONVROT_ERR_INVALID_ARG,
               "N = %lld must be a multiple of 8 in [0, 2^31)", static_cast<long long>(N));
    if (M == 0 || N == 0) return ok();
    const size_t need = convrot_workspace_bytes(M, K, 8);
    CR_REQUIRE(need <= kNoAllocScratchBytes, CONVROT_ERR_WORKSPACE,
               "M = %lld, K = %lld needs %zu bytes of scratch; the built-in array holds %zu "
               "(use convrot_linear_w8a8 with a workspace)",
               static_cast<long long>(M), static_cast<long long>(K), need, kNoAllocScratchBytes);
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    CR_REQUIRE(e == cudaSuccess, CONVROT_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    CR_REQUIRE(dev >= 0 && dev < kMaxDevices, CONVROT_ERR_UNSUPPORTED, "device ordinal %d out of range", dev);
    void *scratch = nullptr;
    {
        // The array's name is only a host-side stand-in: its device address is
        // looked up once per device, with that device current.
        std::lock_guard<std::mutex> lock(g_noalloc_mutex);
        if (g_noalloc_ptr[dev] == nullptr) {
            void *p = nullptr;
            e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
            CR_REQUIRE(e == cudaSuccess && p != nullptr, CONVROT_ERR_CUDA, "cudaGetSymbolAddress: %s",
                       cudaGetErrorString(e));
            g_noalloc_ptr[dev] = p;
        }
        scratch = g_noalloc_ptr[dev];
    }
    return linear_impl(8, X, M, K, Wq, w_scale, N, bias, block, Y, scratch, kNoAllocScratchBytes, stream);
}

convrot_status_t convrot_linear_plan(int64_t M, int64_t K, int64_t N, int bits, int block, size_t workspace_bytes,
                                     convrot_linear_plan_t *plan) {
    g_last_error.clear();
    CR_TRY(check_linear_shape(M, K, block, bits, N));
    CR_REQUIRE(plan != nullptr, CONVROT_ERR_INVALID_ARG, "null pointer argument");
    *plan = convrot_linear_plan_t();
    if (M == 0 || N == 0) return ok();
    CR_REQUIRE(workspace_bytes >= convrot_workspace_bytes(M, K, bits), CONVROT_ERR_WORKSPACE,
               "workspace of %zu bytes given, %zu needed", workspace_bytes, convrot_workspace_bytes(M, K, bits));
    int dev;
    DeviceInfo *info;
    CR_TRY(current_device(&dev, &info));
    const bool widened = bits == 4 && w4_prewidens(M) &&
                         workspace_bytes >= w4_wide_offset(info->sms, M, K, N) + round256(static_cast<size_t>(N) * K);
    const GemmPlan p = two_launch_plan(info->sms, M, N, K, widened ? 8 : bits, workspace_bytes);
    GemmPlan pf;
    plan->launches = 2;  // the activation kernel, then the GEMM
    plan->weights_widened = widened ? 1 : 0;
    plan->fused_available = (bits == 8 && fused_plan(info->sms, M, K, N, bits, block, workspace_bytes, &pf)) ? 1 : 0;
    plan->gemm_kind = p.gemv ? 2 : (p.swap ? 1 : 0);
    plan->tile_n = p.gemv ? 0 : p.bn;
    plan->cta_pair = p.pair ? 1 : 0;
    plan->stream_k = p.streamk > 0 ? 1 : 0;
    plan->k_splits = p.splits;
    return ok();
}

convrot_status_t convrot_test_abandoned_wait(int kind, uint64_t limit_ns, int32_t *result, void *stream) {
    g_last_error.clear();
    CR_REQUIRE(kind == 0 || kind == 1, CONVROT_ERR_INVALID_ARG, "kind = %d must be 0 or 1", kind);
    CR_REQUIRE(limit_ns >= 1000 && limit_ns <= 1000000000ull, CONVROT_ERR_INVALID_ARG,
               "limit_ns = %llu must be in [1 us, 1 s]", static_cast<unsigned long long>(limit_ns));
    CR_REQUIRE(result != nullptr && aligned(result, 16), CONVROT_ERR_ALIGNMENT, "result must be 16-byte aligned");
    int dev;
    DeviceInfo *info;
    CR_TRY(current_device(&dev, &info));
    convrot::abandoned_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(kind, limit_ns, result);
    return launch_status("abandoned_wait");
}

convrot_status_t convrot_device_status(void *stream) {
    g_last_error.clear();
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    CR_REQUIRE(e == cudaSuccess, CONVROT_ERR_CUDA, "stream: %s", cudaGetErrorString(e));
    unsigned int word = 0;
    e = cudaMemcpyFromSymbol(&word, convrot::g_device_status, sizeof(word));
    CR_REQUIRE(e == cudaSuccess, CONVROT_ERR_CUDA, "status read: %s", cudaGetErrorString(e));
    if (word != 0) {
        const unsigned int zero = 0;
        cudaMemcpyToSymbol(convrot::g_device_status, &zero, sizeof(zero));
        if (word & convrot::kStatusTimeout)
            return fail(CONVROT_ERR_TIMEOUT, "a kernel abandoned a device-side wait (status 0x%x)", word);
    }
    return ok();
}

}  // extern "C"
