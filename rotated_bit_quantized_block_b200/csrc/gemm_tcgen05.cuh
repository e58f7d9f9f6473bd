// gemm_tcgen05.cuh -- integer GEMM with the dequantizing epilogue of the
// ConvRot linear, on sm_100a 5th-generation tensor cores.
//
//   acc[m,n] = sum_k qx[m,k] * qw[n,k]                      (tcgen05.mma kind::i8, int32 in TMEM)
//   Y[m,n]   = fp16( fma( fp32(float(acc) * s_x[m]), s_w[n], bias[n] ) )   (fused epilogue)
//
// Method: civarchive.com "SAM 3.1 Multiplex ConvRot" release, "Quantization
// recipe" (W8A8 / W4A4 operations, per-row scales; INT4 multiplication falls
// back to INT8 multiplication where the hardware has no INT4 path -- sm_100
// tcgen05 has no integer-4 kind, so int4 tiles are widened to int8 in shared
// memory before the int8 MMA).
//
// Structure: persistent, warp-specialized CTAs (one per SM), accumulator tile
// 128 x BN, K step 128 bytes.
//   warp 0      TMA producer (one elected lane): A and B tiles -> smem ring
//   warp 1      TMEM allocator + MMA issuer (one lane): 4 x tcgen05.mma per K step
//   epilogue    16 warps (token-major, int8 weights, 128- or 256-wide tiles)
//               or 8: tcgen05.ld of the accumulator, scale, fp16, store
//   converters  int4 operands only, 12 warps: nibble ->
//               byte widening between a packed ring and the MMA ring
// Two TMEM accumulators (2 x BN columns) let the epilogue of one tile overlap
// the main loop of the next.  No TMA multicast is used anywhere.
//
// Two operand orders:
//   * token-major (SWAP = false): A = activation codes (128 tokens per tile),
//     B = weight codes (BN output features); the epilogue stages 32 x 32 fp16
//     boxes in shared memory and writes them with TMA stores.
//   * feature-major (SWAP = true, few tokens): A = weight codes (128 output
//     features per tile), B = activation codes (BN = 32, 64 or 128 tokens:
//     all of them, so every weight byte is read once), so the tensor core is
//     not spent on empty token rows and the weights stream through a deep
//     ring.  Each epilogue thread owns one output feature and writes token
//     columns with coalesced stores.  The K loop may be split over a cluster
//     of 2, 4 or 8 CTAs (one K slice each): the partial accumulators are added
//     through distributed shared memory, each CTA summing and storing the
//     pieces of some of its epilogue warps -- no global partials, counters or
//     zeroing.
//
// Fused linear (Cfg::FUSE, token-major): the kernel also rotates and
// quantizes the activations.  ACT_WARPS extra warps per CTA (register-fed, no
// shared memory) work through "units" of rows -- unit u (RPR = 32*ACT_WARPS /
// (K/32) rows) belongs to CTA u mod grid, so the first units of every CTA
// cover the first 128-token panels -- writing codes and per-token scales into
// the workspace (left in L2) and counting each finished unit into the counter
// of every panel it touches.  The producer loads a panel's A tiles only once
// its counter shows all of the panel's units (acquire, bounded wait), and
// issues the stage's weight tile first so that it is in flight meanwhile; the
// epilogue re-acquires the counter before it reads the panel's scales.  The
// rotation thus runs beside the main loop instead of in a launch of its own,
// and every panel is rotated exactly once.  The counters are zeroed by a small
// kernel launched just before (programmatic dependency).  The grid is at most
// one CTA (or CTA pair) per SM, all co-resident.
#pragma once

#include "device_utils.cuh"
#include "rotate_quant.cuh"

namespace convrot {

// Stream-K ready flags live in the counters array from this index on (the
// arrival counts below it): at most kStreamKFlags CTAs per stream-K grid.
constexpr int kStreamKFlags = 256;

// A4 / B4: the MMA's A / B operand arrives as packed int4 (two codes per byte)
// and is widened in shared memory; otherwise it is int8 loaded by TMA straight
// into the MMA ring.  Widened bytes hold 16 * code, so the accumulator carries
// a factor 16 per widened operand (ACC_SHIFT undoes it).
// PAIR: a cluster of two CTAs shares each 256 x BN tile through one
// cta_group::2 MMA (each CTA loads and keeps 128 rows of A and BN/2 rows of B).
// SK: token-major stream-K (equal shares of all tiles' K steps per CTA).
// FUSE: token-major linear with ACT_WARPS activation warps (see the header).
template <int BN_, bool A4_, bool B4_, bool SWAP_ = false, bool PAIR_ = false, bool SK_ = false, bool FUSE_ = false>
struct GemmCfg {
    static constexpr int BM = 128;   // rows of A per CTA
    static constexpr int BN = BN_;   // accumulator columns
    static constexpr int BK = 128;  // K elements per stage (= bytes of one int8 row segment)
    static constexpr bool A4 = A4_;
    static constexpr bool B4 = B4_;
    static constexpr bool SWAP = SWAP_;
    static constexpr bool PAIR = PAIR_;
    static constexpr bool SK = SK_;
    static constexpr bool FUSE = FUSE_;
    static constexpr int CTAS = PAIR ? 2 : 1;      // CTAs per tile
    static constexpr int TILE_M = BM * CTAS;       // accumulator rows per tile
    static constexpr int B_ROWS = BN / CTAS;       // rows of B held by one CTA
    static constexpr bool W4 = A4 || B4;          // some operand is widened by converter warps
    static constexpr bool TMA_RING = !(A4 && B4);  // some operand goes straight into the MMA ring
    static constexpr int ACC_SHIFT = (A4 ? 4 : 0) + (B4 ? 4 : 0);
    static constexpr int A_BYTES = BM * BK;
    static constexpr int B_BYTES = B_ROWS * BK;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr int PA_BYTES = A4 ? A_BYTES / 2 : 0;
    static constexpr int PB_BYTES = B4 ? B_BYTES / 2 : 0;
    static constexpr int PSTAGE_BYTES = PA_BYTES + PB_BYTES;
    static constexpr int PSTAGES = !W4 ? 0 : (!SWAP && BN == 256 ? 3 : 4);
    static constexpr int CONV_ROWS = (A4 ? BM : 0) + (B4 ? B_ROWS : 0);  // rows widened per stage
    // converter warps widening int4: 12, so that widening keeps pace with the MMA
    // (feature-major, measured on B200: 4 -> 12 warps took the W4A4 linear at 16
    // tokens, K = N = 4096, from 11.7 to 10.4 us, at 128 tokens from 16.8 to 15.5)
    static constexpr int CONV_WARPS = !W4 ? 0 : 12;
    static constexpr int CONV_THREADS = 32 * CONV_WARPS;
    // arrivals completing an MMA stage: the producer (TMA bytes) and/or one per converter warp
    static constexpr int FULL_COUNT = (TMA_RING ? 1 : 0) + CONV_WARPS;
    // two accumulators; the allocation is a power of two of at least 32 columns
    static constexpr int TMEM_COLS = 2 * BN <= 64 ? 64 : (2 * BN <= 128 ? 128 : (2 * BN <= 256 ? 256 : 512));
    // epilogue warps: per TMEM lane quarter, EPI_WARPS / 4 warps split the columns
    // (token-major: four, so that enough warps hide the dequant's latencies)
    static constexpr int EPI_WARPS = (SWAP || W4 || FUSE || BN % 128 != 0) ? 8 : 16;
    static constexpr int EPI_COLS = BN / (EPI_WARPS / 4);  // accumulator columns per epilogue warp
    // token-major: 32-column chunks (one TMEM load, one 32 x 32 fp16 output box);
    // feature-major: 16- or 32-column TMEM loads, stored directly
    static constexpr int CHUNK = !SWAP ? 32 : (EPI_COLS < 32 ? EPI_COLS : 32);
    static constexpr int OUT_BOX_BYTES = 32 * 32 * 2;  // 32 rows x 32 fp16, 64-byte rows
    static constexpr int OUT_BYTES = SWAP ? 0 : EPI_WARPS * OUT_BOX_BYTES;
    static constexpr int SCALE_BYTES = BN * 4 + BN * 2;  // the tile's column scale (fp32) and bias (fp16)
    static constexpr int FIRST_CONV_WARP = 2 + EPI_WARPS;
    // fused linear: activation warps after the converters
    static constexpr int ACT_WARPS = FUSE ? 8 : 0;
    static constexpr int ACT_THREADS = 32 * ACT_WARPS;
    static constexpr int FIRST_ACT_WARP = FIRST_CONV_WARP + CONV_WARPS;
    static constexpr int ACT_MAX_K = ACT_THREADS * kElemsPerThread;  // a row fits the activation warps once
    static constexpr int ACT_SMEM_BYTES = FUSE ? 2 * (ACT_THREADS / 4) * 4 : 0;  // row-segment maxima, 2 units
    static constexpr int NUM_THREADS = 32 * (FIRST_ACT_WARP + ACT_WARPS);
    static constexpr int FIXED_BARRIERS = 2 * PSTAGES + 4 + 1 + 2 + 2 + 1;
    // feature-major split K: an epilogue warp's piece of the accumulator (32
    // TMEM lanes x EPI_COLS int32), staged in the idle MMA ring; the peers'
    // shares of this CTA's columns arrive in a receive area of their own (at
    // most 7/8 of all pieces, for a cluster of 8), which no main loop uses
    static constexpr int PIECE_BYTES = 32 * EPI_COLS * 4;
    static constexpr int RECV_BYTES = SWAP ? EPI_WARPS * PIECE_BYTES / 8 * 7 : 0;
    // MMA ring depth: as many stages as fit in the shared-memory budget (at most 12)
    static constexpr int SMEM_LIMIT = 232448;
    static constexpr int STAGES_FIT = (SMEM_LIMIT - 1024 - PSTAGES * PSTAGE_BYTES - OUT_BYTES - RECV_BYTES -
                                       SCALE_BYTES - ACT_SMEM_BYTES - FIXED_BARRIERS * 8 - 16) /
                                      (STAGE_BYTES + 16);
    static constexpr int STAGES = STAGES_FIT < 12 ? STAGES_FIT : 12;
    static constexpr int NUM_BARRIERS = 2 * STAGES + FIXED_BARRIERS;
    static constexpr int SMEM_BYTES = 1024 /* alignment slack */ + STAGES * STAGE_BYTES + PSTAGES * PSTAGE_BYTES +
                                      OUT_BYTES + RECV_BYTES + SCALE_BYTES + ACT_SMEM_BYTES + NUM_BARRIERS * 8 + 16;
    static constexpr uint32_t IDESC = idesc_i8(TILE_M, BN);
    static_assert(STAGES >= 2, "pipeline depth");
    static_assert(!FUSE || (!SWAP && !A4 && !SK), "fused linear: token-major, int8 activation codes, whole tiles");
    static_assert(!PAIR || (!SWAP && !A4 && !B4 && BN == 256), "CTA pairs: token-major W8A8, 256-wide tiles");
    static_assert(!SK || (!SWAP && !PAIR), "stream-K: token-major, single CTAs");
    static_assert(SMEM_BYTES <= SMEM_LIMIT, "shared memory budget");
    static_assert(SWAP ? (BN == 32 || BN == 64 || BN == 128 || BN == 256) : (BN % 64 == 0 && BN >= 64 && BN <= 256),
                  "tile width");
    static_assert(TMEM_COLS >= 2 * BN, "accumulators fit the allocation");
    static_assert(EPI_COLS % CHUNK == 0 && CHUNK % 4 == 0, "epilogue chunking");
    static_assert(!SWAP || EPI_WARPS * PIECE_BYTES <= STAGES * STAGE_BYTES, "split-K pieces fit the ring");
};

// Sign-extends 16 packed int4 codes (8 bytes, low nibble = even element) to 16
// bytes holding 16 * code: shifting each nibble into the high half of its byte
// keeps the sign; the products are rescaled by 1/256 in the epilogue.
__device__ __forceinline__ uint4 widen_int4x16(uint2 p) {
    const uint32_t lo0 = (p.x << 4) & 0xf0f0f0f0u, hi0 = p.x & 0xf0f0f0f0u;
    const uint32_t lo1 = (p.y << 4) & 0xf0f0f0f0u, hi1 = p.y & 0xf0f0f0f0u;
    return make_uint4(__byte_perm(lo0, hi0, 0x5140), __byte_perm(lo0, hi0, 0x7362), __byte_perm(lo1, hi1, 0x5140),
                      __byte_perm(lo1, hi1, 0x7362));
}

// Dequantizes one accumulator: fp16(fma(fp32(float(acc) * sx), sw, bias)) (the
// final multiply-add is one explicit fused operation, so it rounds once).
__device__ __forceinline__ __half dequant1(int32_t a, float sxm, float swn, float bn) {
    return __float2half_rn(__fmaf_rn(__fmul_rn(__int2float_rn(a), sxm), swn, bn));
}

// Dequantizes 8 accumulators of one row (token-major order).  sw_s / b_s
// point at the tile's scale (fp32) and bias (fp16) staged in shared memory.
template <int SHIFT>
__device__ __forceinline__ uint4 dequant8(const uint32_t *r, float sxm, const float *sw_s, const __half *b_s) {
    const float4 w0 = *reinterpret_cast<const float4 *>(sw_s);
    const float4 w1 = *reinterpret_cast<const float4 *>(sw_s + 4);
    const float2 wv[4] = {make_float2(w0.x, w0.y), make_float2(w0.z, w0.w), make_float2(w1.x, w1.y),
                          make_float2(w1.z, w1.w)};
    const uint4 braw = *reinterpret_cast<const uint4 *>(b_s);
    const uint32_t bw[4] = {braw.x, braw.y, braw.z, braw.w};
    uint32_t out[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int32_t a0 = static_cast<int32_t>(r[2 * i]) >> SHIFT;
        const int32_t a1 = static_cast<int32_t>(r[2 * i + 1]) >> SHIFT;
        float2 t = make_float2(__int2float_rn(a0), __int2float_rn(a1));
        t = __fmul2_rn(t, make_float2(sxm, sxm));
        t = __ffma2_rn(t, wv[i], __half22float2(*reinterpret_cast<const __half2 *>(&bw[i])));
        const __half2 h = __floats2half2_rn(t.x, t.y);
        out[i] = *reinterpret_cast<const uint32_t *>(&h);
    }
    return make_uint4(out[0], out[1], out[2], out[3]);
}

// Loads CHUNK (2 to 32) accumulator columns of this warp's 32 TMEM lanes.
template <int CHUNK>
__device__ __forceinline__ void tmem_ld_chunk(uint32_t taddr, uint32_t (&r)[CHUNK]) {
    static_assert(CHUNK == 32 || CHUNK == 16 || CHUNK == 8 || CHUNK == 4 || CHUNK == 2, "TMEM load width");
    if constexpr (CHUNK == 32) tmem_ld_32x32(taddr, r);
    else if constexpr (CHUNK == 16) tmem_ld_32x16(taddr, r);
    else if constexpr (CHUNK == 8) tmem_ld_32x8(taddr, r);
    else if constexpr (CHUNK == 4) tmem_ld_32x4(taddr, r);
    else tmem_ld_32x2(taddr, r);
}

// ---------------------------------------------------------------- fused linear: panel counters
//
// One 32-bit counter per 128-token panel, in the workspace's counter area:
// the number of finished activation units that touch the panel.  A small
// kernel launched just before the fused kernel zeroes them (the fused kernel
// waits for it through its programmatic-launch dependency), so every launch,
// CUDA-graph replays included, counts from zero whatever the area held before.
constexpr int kFuseMaxPanels = 512;  // counters in the 2 KB area

// Zeroes the n panel counters of the next fused launch (one block).
__global__ void __launch_bounds__(256) fuse_zero_kernel(unsigned int *counters, int n) {
    pdl_wait();  // the previous launch on this workspace may still count into them
    for (int i = threadIdx.x; i < n; i += blockDim.x) counters[i] = 0u;
    pdl_launch_dependents();
}

// Number of units (RPR rows each) that touch panel p (rows [128 p, min(128 p + 128, M))).
__device__ __forceinline__ uint32_t fuse_panel_units(int64_t M, int rpr, int64_t p) {
    const int64_t r0 = 128 * p;
    const int64_t r1 = (r0 + 128 < M ? r0 + 128 : M) - 1;
    return static_cast<uint32_t>(r1 / rpr - r0 / rpr + 1);
}

// Rows per activation unit of `nt` threads (L = K/32 threads per row).
__host__ __device__ __forceinline__ int fuse_unit_rows(int nt, int K) { return nt / (K / kElemsPerThread); }

// Waits (acquire, bounded) until panel p's counter shows all of its units.
__device__ __forceinline__ bool fuse_panel_wait(const unsigned int *counters, int64_t M, int rpr, int64_t p,
                                                volatile int *abort, uint64_t limit_ns = kWaitLimitNs) {
    const unsigned int want = fuse_panel_units(M, rpr, p);
    const uint64_t t0 = globaltimer_ns();
    while (true) {
        unsigned int v;
        asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(counters + p) : "memory");
        if (v == want) return true;
        if (*abort) return false;
        if (globaltimer_ns() - t0 > limit_ns) {
            atomicOr(&g_device_status, kStatusTimeout);
            *abort = 1;
            return false;
        }
    }
}

// The activation warps of one CTA (thread at = 0 .. NT-1): rotate and quantize
// units blockIdx.x, blockIdx.x + gridDim.x, ... into Xq / x_scale (codes one
// byte each, range of BITS), loading the next unit while the current one is
// worked on, and count each finished unit into the counters of the panels it
// touches (release: the consumers acquire the counter, then fence the async
// proxy before their TMA loads).  Rows spanning several warps meet in s_part
// behind named barrier bar_id (all NT threads join it the same number of times).
// (Counting per warp instead, with one release reduction per warp and panel and
// no CTA-wide step, measured slower: 33.5 against 27.8 us for ViT-L qkv.)
template <int LOG2B, int BITS, int NT>
__device__ __forceinline__ void fuse_act_worker(int at, const __half *__restrict__ X, int64_t M, int K,
                                                int8_t *Xq, float *x_scale, unsigned int *counters,
                                                float *s_part, int bar_id) {
    const int lane = at & 31;
    const int L = K / kElemsPerThread;
    const int rpr = NT / L;
    const int r = at / L, l = at - r * L;
    const int g = l >> 2, p = l & 3;
    const int elem0 = 128 * g + 8 * p;
    const int G = reduce_width(L);
    const int segs = L / G;
    const int64_t units = (M + rpr - 1) / rpr;
    auto load = [&](int64_t u, uint4 (&dst)[4]) {
        const int64_t row = u * rpr + r;
        if (r < rpr && row < M) {
            const __half *src = X + row * K + elem0;
#pragma unroll
            for (int j = 0; j < 4; ++j) dst[j] = ld_stream_v4(src + 32 * j);
        } else {
#pragma unroll
            for (int j = 0; j < 4; ++j) dst[j] = make_uint4(0, 0, 0, 0);
        }
    };
    uint4 raw[4];
    int64_t u = blockIdx.x;
    if (u < units) load(u, raw);
    for (int it = 0; u < units; u += gridDim.x, ++it) {
        uint4 nxt[4];
        if (u + gridDim.x < units) load(u + gridDim.x, nxt);
        float2 v[2][8];
        raw_to_v(raw, v);
        fwht_act_order<LOG2B>(v, lane);
        float amax = 0.0f;
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int e = 0; e < 8; ++e) amax = absmax3(amax, v[h][e].x, v[h][e].y);
        for (int mm = 1; mm < G; mm <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, mm));
        if (G < L) {
            float *part = s_part + (it & 1) * (NT / 4);
            if (r < rpr && (l & (G - 1)) == 0) part[r * segs + l / G] = amax;
            named_bar_sync(bar_id, NT);
            if (r < rpr) {
                amax = part[r * segs];
                for (int sg = 1; sg < segs; ++sg) amax = fmaxf(amax, part[r * segs + sg]);
            }
        }
        const int64_t row = u * rpr + r;
        if (r < rpr && row < M) {
            float fac1;
            const float sc = act_row_scale<LOG2B, BITS>(amax, &fac1);
            if (l == 0) x_scale[row] = sc;
            const float2 fac = f2(fac1);
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
                for (int e = 0; e < 8; ++e) v[h][e] = __ffma2_rn(v[h][e], fac, f2(kRoundMagic));
            store_codes<8>(Xq + row * K, elem0, v);
        }
        named_bar_sync(bar_id, NT);  // every code and scale of the unit is written
        if (at == 0) {
            __threadfence();
            const int64_t r0 = u * rpr, r1 = (r0 + rpr < M ? r0 + rpr : M) - 1;
            for (int64_t pn = r0 / 128; pn <= r1 / 128; ++pn) atomicAdd(counters + pn, 1u);
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) raw[j] = nxt[j];
    }
}

// Diagnostics: one bounded wait whose target never completes, through the
// same routines the GEMM uses (kind 0: an mbarrier phase nobody completes;
// kind 1: a fused linear's panel counter nobody counts into).  result[0] = 1
// if the wait succeeded (it must not), result[1] = the abort flag it left; the
// panel counter is result[2], cleared here first.
__global__ void abandoned_wait_kernel(int kind, uint64_t limit_ns, int32_t *result) {
    __shared__ uint64_t bar;
    __shared__ int abort;
    unsigned int *word = reinterpret_cast<unsigned int *>(result + 2);
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort = 0;
        *word = 0;
        fence_mbarrier_init();
        __threadfence();
    }
    __syncthreads();
    if (threadIdx.x != 0) return;
    bool ok;
    if (kind == 0) ok = mbar_wait(&bar, 0, &abort, limit_ns);
    else ok = fuse_panel_wait(word, 128, 1, 0, &abort, limit_ns);
    result[0] = ok ? 1 : 0;
    result[1] = abort;
}

// Weight boxes a feature-major CTA prefetches into L2 before its grid-dependency wait.
constexpr int kMaxEarlyBoxes = 64;

// Where a feature-major epilogue thread stores: its output feature f (a row of
// the accumulator) at the tokens tok_base + column, with the token scales of
// those columns in col_s.
struct SplitOut {
    __half *Y;
    int32_t *acc_out;
    const float *col_s;
    int M, N, f, tok_base;
    float swf, bf;
    bool row_ok;
};

// Split K over a cluster of S CTAs, receiving side.  Every CTA's epilogue
// warp w holds a piece of its slice's partial accumulator (32 rows x EC
// columns); the CTA of rank r sums columns [r * EC / S, (r + 1) * EC / S) of
// every piece.  The other S - 1 CTAs have copied those columns of their piece w
// into recv (slot = sender rank, less one above r; then piece; then
// [column pair][lane][2] int32); this CTA's own partial is read straight from
// TMEM (taddr: the piece's first column).  Batches of up to 8 columns keep the
// registers few; every operand is local.
template <int S, int EC, int EPI_WARPS, int SHIFT>
__device__ __forceinline__ void split_sum_store(const uint8_t *recv, uint32_t rank, int ew, int lane, uint32_t taddr,
                                                const SplitOut &o) {
    constexpr int NP = EC / S / 2;  // column pairs of this CTA's share
    constexpr int G = NP < 4 ? NP : 4;
    static_assert(NP >= 1 && EC % (2 * S) == 0 && NP % G == 0, "share of whole column pairs");
    const int p0 = static_cast<int>(rank) * NP;
#pragma unroll 1
    for (int g0 = 0; g0 < NP; g0 += G) {
        uint32_t acc[2 * G];
        __syncwarp();
        tmem_ld_chunk<2 * G>(taddr + static_cast<uint32_t>(2 * (p0 + g0)), acc);
        tmem_ld_wait();
#pragma unroll
        for (int sl = 0; sl < S - 1; ++sl) {
            const uint8_t *src = recv + ((sl * EPI_WARPS + ew) * NP + g0) * 256 + lane * 8;
#pragma unroll
            for (int j = 0; j < G; ++j) {
                const uint2 v = *reinterpret_cast<const uint2 *>(src + j * 256);
                acc[2 * j] += v.x;
                acc[2 * j + 1] += v.y;
            }
        }
        if (!o.row_ok) continue;
#pragma unroll
        for (int c = 0; c < 2 * G; ++c) {
            const int col = 2 * (p0 + g0) + c;
            const int tok = o.tok_base + col;
            if (tok >= o.N) break;
            const int64_t idx = static_cast<int64_t>(tok) * o.M + o.f;
            const int32_t a = static_cast<int32_t>(acc[c]) >> SHIFT;
            o.Y[idx] = dequant1(a, o.col_s[col], o.swf, o.bf);
            if (o.acc_out != nullptr) o.acc_out[idx] = a;
        }
    }
}

// Kernel arguments, in the MMA's terms: the accumulator is M x N (rows of A x
// rows of B).  Token-major: M = tokens, N = output features.  Feature-major:
// M = output features, N = tokens.  sx is always the per-token scale, sw the
// per-feature scale, bias per feature; Y and acc_out are tokens x features.
// splits > 1 (feature-major): the K slices of a tile, one CTA each, launched
// as a cluster of `splits` CTAs.  acc_buf / counters (stream-K, Cfg::SK): the
// partial-tile slots (TILE_M x BN int32 per CTA boundary), per-boundary
// arrival counts (counters[b]) and ready flags (counters[kStreamKFlags + b]).
// Fused linear (Cfg::FUSE; block 2^FLOG2B, activation codes one byte each in
// the range of FBITS): X is the fp16 input, qx_out / sx_out the workspace that
// tmA and sx cover, panels the zeroed panel counters (see above).
// w_early != 0: the weight codes are not written by the previous kernel in the
// stream, so their first tiles may be prefetched before the dependency wait.
template <class Cfg, int FLOG2B = -1, int FBITS = 8>
__global__ void __launch_bounds__(Cfg::NUM_THREADS, 1)
    gemm_i8_tcgen05_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                           const __grid_constant__ CUtensorMap tmY, int M, int N, int K, const float *sx,
                           const float *__restrict__ sw, const __half *__restrict__ bias, __half *__restrict__ Y,
                           int32_t *__restrict__ acc_out, int splits, int32_t *__restrict__ acc_buf,
                           unsigned int *__restrict__ counters, int streamk, const __half *__restrict__ X,
                           int8_t *qx_out, float *sx_out, unsigned int *panels, int w_early) {
    constexpr bool FUSED = Cfg::FUSE;
    static_assert(FUSED == (FLOG2B >= 0), "the activation warps need the block size");
    constexpr int BM = Cfg::BM, BN = Cfg::BN, STAGES = Cfg::STAGES, PSTAGES = Cfg::PSTAGES;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *ring = smem;                                          // STAGES x (A | B), int8, 128B-swizzled
    uint8_t *pring = ring + STAGES * Cfg::STAGE_BYTES;             // PSTAGES x (A4 | B4), packed, dense rows
    uint8_t *outbuf = pring + PSTAGES * Cfg::PSTAGE_BYTES;         // per epilogue warp: 32 x 32 fp16 box
    uint8_t *recv = outbuf + Cfg::OUT_BYTES;                       // split K: the peers' shares
    uint8_t *after_recv = recv + Cfg::RECV_BYTES;
    float *col_s = reinterpret_cast<float *>(after_recv);                       // [BN] tile column scale
    __half *bias_s = reinterpret_cast<__half *>(col_s + BN);                    // [BN] tile bias (token-major)
    float *act_part = reinterpret_cast<float *>(after_recv + Cfg::SCALE_BYTES);  // activation warps
    uint64_t *bars = reinterpret_cast<uint64_t *>(after_recv + Cfg::SCALE_BYTES + Cfg::ACT_SMEM_BYTES);
    uint64_t *full = bars;                                         // MMA ring: operands ready
    uint64_t *empty = full + STAGES;                               // MMA ring: slot consumed
    uint64_t *pfull = empty + STAGES;                              // packed ring: TMA landed
    uint64_t *pempty = pfull + PSTAGES;                            // packed ring: slot converted
    uint64_t *tmem_full = pempty + PSTAGES;                        // [2] accumulator ready
    uint64_t *tmem_empty = tmem_full + 2;                          // [2] accumulator drained
    uint64_t *drain = tmem_empty + 2;                              // MMA completion at exit
    uint64_t *scale_ready = drain + 1;                             // tile scales staged in smem
    uint64_t *scale_free = scale_ready + 1;                        // tile scales no longer read
    uint64_t *partial_done = scale_free + 1;                       // split K: this slice's partial added
    uint64_t *decided = partial_done + 1;                          // stream-K: role decision made
    uint64_t *red_in = decided + 1;                                // cluster split K: peers' shares copied in
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(red_in + 1);
    volatile int *abort = reinterpret_cast<volatile int *>(tmem_slot + 1);
    volatile int *s_last = reinterpret_cast<volatile int *>(tmem_slot + 2);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int tiles_m = (M + Cfg::TILE_M - 1) / Cfg::TILE_M, tiles_n = (N + BN - 1) / BN;
    const int num_tiles = tiles_m * tiles_n;
    const int num_kb = K / Cfg::BK;
    // CTA pairs: both CTAs of a cluster walk the same tiles; rank 0 issues the MMAs
    const uint32_t rank = Cfg::PAIR ? cluster_ctarank() : 0u;
    const bool leader = rank == 0;
    const int first_unit = Cfg::PAIR ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
    const int unit_stride = Cfg::PAIR ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);
    // split K (feature-major only): work unit u is K slice (u % splits) of tile (u / splits).
    // The host launches one CTA per unit in clusters of `splits` CTAs (a tile's
    // slices), which add their partial accumulators through distributed shared
    // memory: the CTA of rank r sums and stores the r-th of `splits` column
    // shares of every epilogue warp's piece.
    const bool csplit = Cfg::SWAP && splits > 1;
    const uint32_t crank = csplit ? cluster_ctarank() : 0u;
    const int num_units = num_tiles * splits;
    auto unit_tile = [&](int u) { return u / splits; };
    auto unit_kb0 = [&](int u) { return (u - (u / splits) * splits) * num_kb / splits; };
    auto unit_kb1 = [&](int u) { return (u - (u / splits) * splits + 1) * num_kb / splits; };
    // Stream-K (token-major, single CTAs): the tile-major sequence of (tile, K
    // step) pairs, num_tiles * num_kb long, is cut into gridDim.x equal ranges
    // (each at least num_kb long, so a tile is shared by at most two CTAs).  A
    // range falls into segments: the last steps of a tile, whole tiles, the
    // first steps of a tile.  Otherwise a segment is one work unit.
    // (The host keeps num_tiles * num_kb below 2^31.)
    const bool sk = Cfg::SK && streamk != 0;
    const int64_t sk_total = static_cast<int64_t>(num_tiles) * num_kb;
    const int sk_lo = sk ? static_cast<int>(sk_total * blockIdx.x / gridDim.x) : 0;
    const int sk_hi = sk ? static_cast<int>(sk_total * (blockIdx.x + 1) / gridDim.x) : 0;
    struct Seg {
        int u;               // unit, or the range position of the segment's first step
        int tile, kb0, kb1;  // tile < 0: no more work
    };
    auto seg_at = [&](int u) {
        Seg g{u, -1, 0, 0};
        if (sk) {
            if (u < sk_hi) {
                g.tile = u / num_kb;
                g.kb0 = u - g.tile * num_kb;
                g.kb1 = sk_hi - u < num_kb - g.kb0 ? g.kb0 + (sk_hi - u) : num_kb;
            }
        } else if (u < num_units) {
            g.tile = unit_tile(u);
            g.kb0 = unit_kb0(u);
            g.kb1 = unit_kb1(u);
        }
        return g;
    };
    auto seg_first = [&]() { return seg_at(sk ? sk_lo : first_unit); };
    auto seg_next = [&](const Seg &g) { return seg_at(sk ? g.u + (g.kb1 - g.kb0) : g.u + unit_stride); };

    if (threadIdx.x == 0) {
        for (int i = 0; i < STAGES; ++i) {
            mbar_init(&full[i], Cfg::FULL_COUNT);
            mbar_init(&empty[i], 1);
        }
        for (int i = 0; i < PSTAGES; ++i) {
            mbar_init(&pfull[i], 1);
            mbar_init(&pempty[i], Cfg::CONV_THREADS);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&tmem_full[i], 1);
            mbar_init(&tmem_empty[i], Cfg::CTAS * 32 * Cfg::EPI_WARPS);  // every epilogue thread of the tile
        }
        mbar_init(drain, 1);
        mbar_init(scale_ready, 32 * Cfg::EPI_WARPS);
        mbar_init(scale_free, 32 * Cfg::EPI_WARPS);
        mbar_init(partial_done, 32 * Cfg::EPI_WARPS);
        mbar_init(decided, 1);
        // one arrival (with the expected bytes of the peers' copies) by this CTA
        mbar_init(red_in, 1u);
        *abort = 0;
        fence_mbarrier_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
        if (!Cfg::SWAP) tma_prefetch_desc(&tmY);
    }
    if (warp == 1) {
        if (Cfg::PAIR) {
            tmem_alloc_pair(tmem_slot, Cfg::TMEM_COLS);
            tmem_relinquish_pair();
        } else {
            tmem_alloc(tmem_slot, Cfg::TMEM_COLS);
            tmem_relinquish();
        }
    }
    tc_fence_before_sync();
    __syncthreads();
    // the peers' barriers are initialised before any remote use (split K: only
    // the epilogue's reduction, long after; its warps wait for this barrier there)
    if (Cfg::PAIR) cluster_sync();
    else if (csplit) cluster_arrive_release();
    bool cl_waited = !csplit;
    tc_fence_after_sync();
    const uint32_t tmem_base = *tmem_slot;
    // Weight codes that the previous kernel does not write (w_early): the first
    // segment's weight tiles are prefetched into L2 while that kernel still runs
    // (feature-major: the whole K slice, the few-token GEMM's entire stream;
    // token-major: one ring's worth).
    if (w_early != 0 && threadIdx.x == 0) {
        const Seg g = seg_first();
        if (g.tile >= 0) {
            const int tm = g.tile / tiles_n, tn = g.tile - tm * tiles_n;
            const int span = g.kb1 - g.kb0, cap = Cfg::SWAP ? kMaxEarlyBoxes : STAGES;
            const int n = span < cap ? span : cap;
            for (int i = 0; i < n; ++i) {
                const int kb = g.kb0 + i;
                if (Cfg::SWAP) tma_prefetch_l2_2d(&tmA, kb * (Cfg::A4 ? Cfg::BK / 2 : Cfg::BK), tm * BM);
                else tma_prefetch_l2_2d(&tmB, kb * (Cfg::B4 ? Cfg::BK / 2 : Cfg::BK), tn * BN + rank * Cfg::B_ROWS);
            }
        }
    }
    pdl_wait();  // the codes, scales and split-K buffers may come from the previous kernel
    pdl_launch_dependents();
    [[maybe_unused]] const int act_rpr = FUSED ? fuse_unit_rows(Cfg::ACT_THREADS, K) : 1;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            // MMA ring (s, ph): int8 operands loaded straight by TMA; packed ring
            // (ps, pph): int4 operands for the converters
            int s = 0, ps = 0;
            uint32_t ph = 0, pph = 0;
            uint32_t last_parity[STAGES > PSTAGES ? STAGES : PSTAGES];
            uint32_t plast_parity[PSTAGES > 0 ? PSTAGES : 1];
            bool filled[STAGES > PSTAGES ? STAGES : PSTAGES], pfilled[PSTAGES > 0 ? PSTAGES : 1];
            for (int i = 0; i < STAGES; ++i) filled[i] = false;
            for (int i = 0; i < PSTAGES; ++i) pfilled[i] = false;
            bool ok = true;
            [[maybe_unused]] int ready_tm = -1;  // fused: the last panel seen complete
            for (Seg g = seg_first(); ok && g.tile >= 0; g = seg_next(g)) {
                const int tile = g.tile;
                const int tm = tile / tiles_n, tn = tile - tm * tiles_n;
                for (int kb = g.kb0; kb < g.kb1; ++kb) {
                    if (Cfg::TMA_RING) {
                        if (!mbar_wait(&empty[s], ph ^ 1, abort)) {
                            ok = false;
                            break;
                        }
                        uint8_t *dst = ring + s * Cfg::STAGE_BYTES;
                        if (Cfg::PAIR) {
                            // both CTAs' bytes land on the even CTA's barrier
                            if (leader) mbar_arrive_expect_tx(&full[s], 2 * Cfg::STAGE_BYTES);
                            const uint32_t bar = cluster_addr(&full[s], 0);
                            tma_load_2d_pair(dst + Cfg::A_BYTES, &tmB, bar, kb * Cfg::BK,
                                             tn * BN + rank * Cfg::B_ROWS);
                            if constexpr (FUSED) {
                                // this CTA's 128 rows of the pair's tile are panel 2 tm + rank
                                if (tm != ready_tm) {
                                    const int64_t pn = 2 * static_cast<int64_t>(tm) + rank;
                                    if (pn * 128 >= M || fuse_panel_wait(panels, M, act_rpr, pn, abort)) {
                                        fence_proxy_async_global();
                                        ready_tm = tm;
                                    } else {
                                        ok = false;
                                    }
                                }
                            }
                            tma_load_2d_pair(dst, &tmA, bar, kb * Cfg::BK, tm * Cfg::TILE_M + rank * BM);
                        } else {
                            mbar_arrive_expect_tx(&full[s],
                                                  (Cfg::A4 ? 0 : Cfg::A_BYTES) + (Cfg::B4 ? 0 : Cfg::B_BYTES));
                            if (!Cfg::B4) tma_load_2d(dst + Cfg::A_BYTES, &tmB, &full[s], kb * Cfg::BK, tn * BN);
                            if constexpr (FUSED) {
                                // the panel's codes: wait for its units (the weight tile is already on
                                // its way).  After a timeout the A tile is still loaded, so that the
                                // stage completes and drains; the launch is abandoned anyway.
                                if (tm != ready_tm) {
                                    if (fuse_panel_wait(panels, M, act_rpr, tm, abort)) {
                                        fence_proxy_async_global();  // the codes were written through the generic proxy
                                        ready_tm = tm;
                                    } else {
                                        ok = false;
                                    }
                                }
                            }
                            if (!Cfg::A4) tma_load_2d(dst, &tmA, &full[s], kb * Cfg::BK, tm * BM);
                        }
                        filled[s] = true;
                        last_parity[s] = ph;
                        if (++s == STAGES) {
                            s = 0;
                            ph ^= 1;
                        }
                        if (!ok) break;
                    }
                    if (Cfg::W4) {
                        if (!mbar_wait(&pempty[ps], pph ^ 1, abort)) {
                            ok = false;
                            break;
                        }
                        uint8_t *dst = pring + ps * Cfg::PSTAGE_BYTES;
                        mbar_arrive_expect_tx(&pfull[ps], Cfg::PSTAGE_BYTES);
                        if (Cfg::A4) tma_load_2d(dst, &tmA, &pfull[ps], kb * (Cfg::BK / 2), tm * BM);
                        if (Cfg::B4)
                            tma_load_2d(dst + Cfg::PA_BYTES, &tmB, &pfull[ps], kb * (Cfg::BK / 2), tn * BN);
                        pfilled[ps] = true;
                        plast_parity[ps] = pph;
                        if (++ps == PSTAGES) {
                            ps = 0;
                            pph ^= 1;
                        }
                    }
                }
            }
            // no bulk copy may still be writing shared memory when the CTA exits
            // (an MMA stage also waits for its converters when an operand is widened;
            // the odd CTA of a pair sees its copies complete when the MMA frees the stage)
            for (int i = 0; i < STAGES; ++i) {
                if (!filled[i]) continue;
                if (Cfg::PAIR && !leader) mbar_wait_drain(&empty[i], last_parity[i]);
                else mbar_wait_drain(&full[i], last_parity[i]);
            }
            for (int i = 0; i < PSTAGES; ++i)
                if (pfilled[i]) mbar_wait_drain(&pfull[i], plast_parity[i]);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (Cfg::PAIR && !leader) {
            // the even CTA issues the pair's MMAs; wait until they have all completed
            // (they read this CTA's shared memory)
            if (lane == 0) mbar_wait_drain(drain, 0);
        } else if (lane == 0) {
            int s = 0;
            uint32_t ph = 0;
            bool ok = true;
            int local = 0;
            for (Seg g = seg_first(); ok && g.tile >= 0; g = seg_next(g), ++local) {
                const int acc = local & 1;
                const uint32_t acc_ph = (local >> 1) & 1;
                if (!mbar_wait(&tmem_empty[acc], acc_ph ^ 1, abort)) break;
                tc_fence_after_sync();
                const uint32_t d_tmem = tmem_base + acc * BN;
                const int kb0 = g.kb0;
                for (int kb = kb0; kb < g.kb1; ++kb) {
                    if (!mbar_wait(&full[s], ph, abort)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after_sync();
                    const uint32_t a_addr = smem_addr(ring + s * Cfg::STAGE_BYTES);
                    const uint32_t b_addr = a_addr + Cfg::A_BYTES;
#pragma unroll
                    for (int kk = 0; kk < Cfg::BK / 32; ++kk) {
                        if (Cfg::PAIR)
                            umma_i8_pair(d_tmem, smem_desc_k_sw128(a_addr + 32 * kk),
                                         smem_desc_k_sw128(b_addr + 32 * kk), Cfg::IDESC, (kb != kb0) || (kk != 0));
                        else
                            umma_i8(d_tmem, smem_desc_k_sw128(a_addr + 32 * kk), smem_desc_k_sw128(b_addr + 32 * kk),
                                    Cfg::IDESC, (kb != kb0) || (kk != 0));
                    }
                    if (Cfg::PAIR) umma_commit_pair(&empty[s], 3);  // frees the stage in both CTAs
                    else umma_commit(&empty[s]);
                    if (++s == STAGES) {
                        s = 0;
                        ph ^= 1;
                    }
                }
                if (ok) {
                    if (Cfg::PAIR) umma_commit_pair(&tmem_full[acc], 3);
                    else umma_commit(&tmem_full[acc]);
                }
            }
            if (Cfg::PAIR) umma_commit_pair(drain, 3);
            else umma_commit(drain);
            mbar_wait_drain(drain, 0);
        }
    } else if (warp < Cfg::FIRST_CONV_WARP) {
        // ------------------------------------------------------------ epilogue
        // Warp w reads TMEM lanes 32*(w%4) .. +31 (its hardware lane quarter)
        // and columns [cg * EPI_COLS, (cg+1) * EPI_COLS) of the accumulator.  The
        // tile's column scales (and, token-major, the bias) are prefetched into
        // registers one tile ahead (one column per thread) and staged in
        // shared memory at tile start.
        const int ew = warp - 2;  // 0 .. EPI_WARPS-1
        const int q = warp & 3;
        const int cg = ew >> 2;   // column group
        const int scol = ew * 32 + lane;  // the tile column this thread stages (valid if < BN)
        const float *col_scale = Cfg::SWAP ? sx : sw;
        auto load_scales = [&](int t, float &wv, __half &bv) {
            wv = 0.0f;
            bv = __float2half_rn(0.0f);
            if (t < num_tiles && scol < BN) {
                const int col = (t - (t / tiles_n) * tiles_n) * BN + scol;
                if (col < N) {
                    wv = __ldg(col_scale + col);
                    if (!Cfg::SWAP && bias != nullptr) bv = bias[col];
                }
            }
        };
        float next_w;
        __half next_b;
        {
            const Seg g0 = seg_first();
            load_scales(g0.tile >= 0 ? g0.tile : num_tiles, next_w, next_b);
        }
        int local = 0;
        int n_split_units = 0;  // stream-K shared tiles handled so far (parity of `decided`)
        int n_partials = 0;     // stream-K partial tiles stored so far (parity of `partial_done`)
        for (Seg g = seg_first(); g.tile >= 0; g = seg_next(g), ++local) {
            const int tile = g.tile;
            const int acc = local & 1;
            const uint32_t acc_ph = (local >> 1) & 1;
            const int tm = tile / tiles_n, tn = tile - tm * tiles_n;
            const int row0 = tm * Cfg::TILE_M + static_cast<int>(rank) * BM + q * 32;
            const int row = row0 + lane;
            const bool row_ok = row < M;
            if constexpr (FUSED) {
                // the scales of these rows: their panel's word (acquired while the tile's main loop still runs)
                int rdy = 1;
                if (lane == 0 && row0 < M) rdy = fuse_panel_wait(panels, M, act_rpr, row0 / 128, abort);
                if (!__shfl_sync(0xffffffffu, rdy, 0)) break;
            }
            // token-major: the row's per-token scale (L2: possibly written by this launch);
            // feature-major: the row's weight scale and bias -- loaded before the
            // accumulator wait, so that their latency is hidden
            const float sxm = (!Cfg::SWAP && row_ok) ? __ldcg(sx + row) : 0.0f;
            const float swf = (Cfg::SWAP && row_ok) ? __ldg(sw + row) : 0.0f;
            const float bf = (Cfg::SWAP && row_ok && bias != nullptr) ? __half2float(bias[row]) : 0.0f;
            if (!mbar_wait_warp(&tmem_full[acc], acc_ph, abort)) break;
            tc_fence_after_sync();
            // every epilogue thread is done with the previous segment's scales
            if (local > 0 && !mbar_wait_warp(scale_free, (local - 1) & 1, abort)) break;
            if (scol < BN) {
                col_s[scol] = next_w;
                bias_s[scol] = next_b;
            }
            mbar_arrive(scale_ready);
            if (!mbar_wait_warp(scale_ready, local & 1, abort)) break;
            {
                const Seg gn = seg_next(g);
                load_scales(gn.tile >= 0 ? gn.tile : num_tiles, next_w, next_b);
            }
            const uint32_t tbase = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * BN;
            constexpr int CH = Cfg::CHUNK;
            constexpr int NCHUNK = Cfg::EPI_COLS / CH;
            if constexpr (!Cfg::SWAP) {
                // ---- token-major: row = token; 32 x 32 boxes through shared memory and TMA
                // Stream-K, a tile shared with the neighbouring CTA (boundary
                // `slot`): the first of the two to get here stores its int32
                // partial (fragment-major: warp, chunk, register, lane) in the
                // boundary's slot and raises the slot's flag; the second waits
                // for the flag (the first is running and only storing), adds the
                // partial to its own and writes Y.  Integer addition is exact, so
                // the result does not depend on which CTA comes first.
                int sk_role = 0;  // 0: whole tile; 1: store the partial; 2: add the partial
                int slot = 0;
                int32_t *sk_part = nullptr;
                if (sk && (g.kb0 != 0 || g.kb1 != num_kb)) {
                    slot = g.kb0 != 0 ? static_cast<int>(blockIdx.x) : static_cast<int>(blockIdx.x) + 1;
                    if (ew == 0 && lane == 0) {
                        int role = 0;
                        const unsigned int before = atomicAdd(&counters[slot], 1u);
                        if (before == 0u) {
                            role = 1;
                        } else if (flag_wait(&counters[kStreamKFlags + slot], abort)) {
                            counters[slot] = 0u;  // both arrived: ready for the next call
                            counters[kStreamKFlags + slot] = 0u;
                            role = 2;
                        }
                        *s_last = role;
                        mbar_arrive(decided);
                    }
                    if (!mbar_wait_warp(decided, n_split_units & 1, abort)) break;
                    ++n_split_units;
                    sk_role = *s_last;
                    if (sk_role == 0) break;  // abandoned after a timeout
                    sk_part = acc_buf + static_cast<int64_t>(slot) * (Cfg::TILE_M * BN) + ew * (NCHUNK * 1024);
                }
                uint8_t *box = outbuf + ew * Cfg::OUT_BOX_BYTES;
                // 64-byte rows, 16-byte chunk g stored at g ^ ((row / 2) & 3) (64B swizzle)
                uint8_t *brow = box + lane * 64;
                const int xr = ((lane >> 1) & 3) << 4;
#pragma unroll 1
                for (int c = 0; c < NCHUNK; ++c) {
                    const int col_local = cg * Cfg::EPI_COLS + c * CH;
                    uint32_t r[32];
                    __syncwarp();  // tcgen05.ld is warp-collective
                    tmem_ld_32x32(tbase + col_local, r);
                    tmem_ld_wait();
                    if (c == NCHUNK - 1) {
                        // every TMEM read of this segment by this thread is complete
                        tc_fence_before_sync();
                        if (Cfg::PAIR) mbar_arrive_cluster(cluster_addr(&tmem_empty[acc], 0));
                        else mbar_arrive(&tmem_empty[acc]);
                    }
                    const int col0 = tn * BN + col_local;
                    if (row0 >= M || col0 >= N) continue;  // whole box outside Y (warp-uniform)
                    if (sk_role == 1) {
                        int32_t *dst = sk_part + c * 1024 + lane;
#pragma unroll
                        for (int j = 0; j < 32; ++j) __stcg(dst + 32 * j, static_cast<int32_t>(r[j]));
                        continue;
                    }
                    if (sk_role == 2) {
                        const int32_t *src = sk_part + c * 1024 + lane;
#pragma unroll
                        for (int j = 0; j < 32; ++j) r[j] += static_cast<uint32_t>(__ldcg(src + 32 * j));
                    }
                    // the store issued from this box last time must have read it
                    if (lane == 0) bulk_wait_group_read<0>();
                    __syncwarp();
                    const float *sw_c = col_s + col_local;
                    const __half *b_c = bias_s + col_local;
                    if (row_ok && col0 + 32 <= N && acc_out == nullptr) {
#pragma unroll
                        for (int g = 0; g < 4; ++g)
                            *reinterpret_cast<uint4 *>(brow + ((g << 4) ^ xr)) =
                                dequant8<Cfg::ACC_SHIFT>(r + 8 * g, sxm, sw_c + 8 * g, b_c + 8 * g);
                    } else {
#pragma unroll
                        for (int g = 0; g < 4; ++g) {  // 8 columns per 16-byte chunk
                            uint4 v = make_uint4(0, 0, 0, 0);
                            if (row_ok && col0 + 8 * g < N) {
                                const uint32_t *rg = r + 8 * g;
                                v = dequant8<Cfg::ACC_SHIFT>(rg, sxm, sw_c + 8 * g, b_c + 8 * g);
                                if (acc_out != nullptr) {
                                    int4 *dst = reinterpret_cast<int4 *>(acc_out + static_cast<int64_t>(row) * N +
                                                                         col0 + 8 * g);
                                    constexpr int SH = Cfg::ACC_SHIFT;
                                    dst[0] = make_int4(static_cast<int32_t>(rg[0]) >> SH, static_cast<int32_t>(rg[1]) >> SH,
                                                       static_cast<int32_t>(rg[2]) >> SH, static_cast<int32_t>(rg[3]) >> SH);
                                    dst[1] = make_int4(static_cast<int32_t>(rg[4]) >> SH, static_cast<int32_t>(rg[5]) >> SH,
                                                       static_cast<int32_t>(rg[6]) >> SH, static_cast<int32_t>(rg[7]) >> SH);
                                }
                            }
                            *reinterpret_cast<uint4 *>(brow + ((g << 4) ^ xr)) = v;
                        }
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        tma_store_2d(&tmY, box, col0, row0);
                        bulk_commit_group();
                    }
                }
                if (sk_role == 1) {
                    // every thread's partial is visible device-wide before the flag goes up
                    __threadfence();
                    mbar_arrive(partial_done);
                    if (ew == 0 && lane == 0 && mbar_wait(partial_done, n_partials & 1, abort)) {
                        __threadfence();
                        flag_raise(&counters[kStreamKFlags + slot]);
                    }
                    ++n_partials;
                }
            } else {
                // ---- feature-major: row = output feature f, columns = tokens
                const int f = row;
                const int tok_base = tn * BN + cg * Cfg::EPI_COLS;
                if (!csplit) {
#pragma unroll 1
                    for (int c = 0; c < NCHUNK; ++c) {
                        uint32_t r[CH];
                        __syncwarp();
                        tmem_ld_chunk<CH>(tbase + cg * Cfg::EPI_COLS + c * CH, r);
                        tmem_ld_wait();
                        if (c == NCHUNK - 1) {
                            tc_fence_before_sync();
                            mbar_arrive(&tmem_empty[acc]);
                        }
                        if (!row_ok) continue;
#pragma unroll
                        for (int j = 0; j < CH; ++j) {
                            const int tok = tok_base + c * CH + j;
                            if (tok >= N) break;
                            const int64_t o = static_cast<int64_t>(tok) * M + f;
                            const int32_t a = static_cast<int32_t>(r[j]) >> Cfg::ACC_SHIFT;
                            Y[o] = dequant1(a, col_s[cg * Cfg::EPI_COLS + c * CH + j], swf, bf);
                            if (acc_out != nullptr) acc_out[o] = a;
                        }
                    }
                } else {
                    // Split K (one unit per CTA, so the MMA ring is idle now): the warp
                    // stages its piece of this slice's partial in its ring slot as
                    // [column pair][lane][2] int32, where the share of cluster rank d
                    // (columns [d * n, (d + 1) * n), n = EPI_COLS / splits) is one
                    // contiguous block.  Lane 0 bulk-copies each peer's block into
                    // that peer's receive area, counted on the peer's red_in; the CTA
                    // expects those bytes on its own red_in and, once they are in,
                    // sums its share (see split_sum_store).  No remote arrival is
                    // needed: the copies' byte counts complete the phase.  Integer
                    // addition is exact: the order does not matter.  (Measured on
                    // B200: summing with distributed-shared-memory loads held the
                    // epilogue 0.8 us at 16 tokens and 2.3 us at 128; every
                    // cluster-scope release arrival or fence cost 0.3-1 us.)
                    uint8_t *piece = ring + ew * Cfg::PIECE_BYTES;
#pragma unroll 1
                    for (int c = 0; c < NCHUNK; ++c) {
                        uint32_t r[CH];
                        __syncwarp();
                        tmem_ld_chunk<CH>(tbase + cg * Cfg::EPI_COLS + c * CH, r);
                        tmem_ld_wait();
#pragma unroll
                        for (int j2 = 0; j2 < CH / 2; ++j2)
                            *reinterpret_cast<uint2 *>(piece + ((c * (CH / 2) + j2) * 32 + lane) * 8) =
                                make_uint2(r[2 * j2], r[2 * j2 + 1]);
                    }
                    fence_proxy_async_smem();  // the staged piece is read by the bulk copies
                    __syncwarp();
                    if (!cl_waited) {
                        cluster_wait_acquire();  // the peers' barriers are initialised
                        cl_waited = true;
                    }
                    const uint32_t share = static_cast<uint32_t>(Cfg::EPI_COLS / splits) * 128u;  // bytes
                    if (lane == 0) {
                        if (ew == 0)
                            mbar_arrive_expect_tx(red_in, static_cast<uint32_t>(splits - 1) * Cfg::EPI_WARPS * share);
                        for (int d = 0; d < splits; ++d) {
                            if (d == static_cast<int>(crank)) continue;
                            const int slot = static_cast<int>(crank) < d ? static_cast<int>(crank) : static_cast<int>(crank) - 1;
                            const uint32_t dst = cluster_addr(recv, static_cast<uint32_t>(d)) +
                                                 static_cast<uint32_t>(slot * Cfg::EPI_WARPS + ew) * share;
                            bulk_copy_to_peer(dst, piece + d * share, share, cluster_addr(red_in, static_cast<uint32_t>(d)));
                        }
                        bulk_commit_group();
                    }
                    if (!mbar_wait_cluster_warp(red_in, 0, abort)) break;
                    const SplitOut out{Y, acc_out, col_s + cg * Cfg::EPI_COLS, M, N, f, tok_base, swf, bf, row_ok};
                    const uint32_t taddr = tbase + cg * Cfg::EPI_COLS;
                    if (splits == 2)
                        split_sum_store<2, Cfg::EPI_COLS, Cfg::EPI_WARPS, Cfg::ACC_SHIFT>(recv, crank, ew, lane, taddr, out);
                    else if (splits == 4)
                        split_sum_store<4, Cfg::EPI_COLS, Cfg::EPI_WARPS, Cfg::ACC_SHIFT>(recv, crank, ew, lane, taddr, out);
                    else
                        split_sum_store<8, Cfg::EPI_COLS, Cfg::EPI_WARPS, Cfg::ACC_SHIFT>(recv, crank, ew, lane, taddr, out);
                    tc_fence_before_sync();
                    mbar_arrive(&tmem_empty[acc]);
                }
            }
            mbar_arrive(scale_free);
        }
        // the output boxes' TMA stores (token-major) or the split-K copies to the
        // peers (feature-major) are complete before the CTA may leave
        if (lane == 0) bulk_wait_group_all();
    } else if (Cfg::W4 && warp < Cfg::FIRST_ACT_WARP) {
        // ------------------------------------------------------------ int4 -> int8 converters
        const int ct = threadIdx.x - 32 * Cfg::FIRST_CONV_WARP;  // 0 .. CONV_THREADS-1
        int ps = 0, us = 0;
        uint32_t pph = 0, uph = 0;
        bool ok = true;
        for (Seg g = seg_first(); ok && g.tile >= 0; g = seg_next(g)) {
            for (int kb = g.kb0; kb < g.kb1; ++kb) {
                if (!mbar_wait_warp(&pfull[ps], pph, abort) || !mbar_wait_warp(&empty[us], uph ^ 1, abort)) {
                    ok = false;
                    break;
                }
                const uint8_t *src = pring + ps * Cfg::PSTAGE_BYTES;
                // widened rows (A if packed, then B if packed) in the MMA ring's layout
                uint8_t *dst = ring + us * Cfg::STAGE_BYTES + (Cfg::A4 ? 0 : Cfg::A_BYTES);
                constexpr int PIECES = Cfg::CONV_ROWS * (Cfg::BK / 16);  // 16 codes per piece
#pragma unroll 4
                for (int idx = ct; idx < PIECES; idx += Cfg::CONV_THREADS) {
                    const int rr = idx >> 3, piece = idx & 7;  // widened row; 16-byte chunk in the row
                    const uint2 p = *reinterpret_cast<const uint2 *>(src + rr * 64 + piece * 8);
                    *reinterpret_cast<uint4 *>(dst + rr * 128 + ((piece ^ (rr & 7)) << 4)) = widen_int4x16(p);
                }
                // the widened bytes are visible to the tensor core before the stage is signalled
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&full[us]);
                mbar_arrive(&pempty[ps]);
                if (++ps == PSTAGES) {
                    ps = 0;
                    pph ^= 1;
                }
                if (++us == STAGES) {
                    us = 0;
                    uph ^= 1;
                }
            }
        }
    }

    if constexpr (FUSED) {
        if (warp >= Cfg::FIRST_ACT_WARP) {
            // ------------------------------------------------------------ activation warps
            fuse_act_worker<FLOG2B < 0 ? 0 : FLOG2B, FBITS, Cfg::ACT_THREADS>(
                threadIdx.x - 32 * Cfg::FIRST_ACT_WARP, X, M, K, qx_out, sx_out, panels, act_part, 1);
        }
    }

    if (!cl_waited) cluster_wait_acquire();  // (warps that did not reach the reduction)
    __syncthreads();
    // no CTA leaves while a peer may still signal it or read its shared memory
    if (Cfg::PAIR || csplit) cluster_sync();
    if (warp == 1) {
        tc_fence_after_sync();
        if (Cfg::PAIR) tmem_dealloc_pair(tmem_base, Cfg::TMEM_COLS);
        else tmem_dealloc(tmem_base, Cfg::TMEM_COLS);
    }
}

}  // namespace convrot
