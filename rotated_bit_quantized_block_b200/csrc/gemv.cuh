// gemv.cuh -- the integer GEMM with its dequantizing epilogue for a handful of
// tokens (the plan uses it up to 4 tokens with int8 weights, 8 with int4; the
// kernel accepts up to 16), as a weight-streaming kernel.
//
//   acc[m,n] = sum_k qx[m,k] * qw[n,k]            (exact int32, dp4a)
//   Y[m,n]   = fp16( fma( fp32(float(acc) * s_x[m]), s_w[n], bias[n] ) )
//
// Method: civarchive.com "SAM 3.1 Multiplex ConvRot" release, "Quantization
// recipe" (W8A8 / W4A4 operations, per-row scales).  With so few tokens the
// product is bound by reading the weights once from HBM, so the tensor core is
// not needed: each block owns 4 output features, its warps split K into
// 512-code chunks (one 16-byte load per lane and feature), int4 weights are
// widened in registers, the activation codes (a few KB) come through L1.
#pragma once

#include "device_utils.cuh"
#include "rotate_quant.cuh"

namespace convrot {

constexpr int kGemvFeatures = 4;     // output features per block
constexpr int kGemvChunk = 512;      // codes per warp step (32 lanes x 16)
constexpr int kGemvMaxTokens = 16;

__device__ __forceinline__ uint2 ld_stream_v2(const void *p) {
    uint2 v;
    asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
    return v;
}

// Sign-extends 16 packed int4 codes (low nibble = even element) to bytes
// holding 16 * code (see the GEMM's converters); products carry a factor 16.
__device__ __forceinline__ uint4 gemv_widen_int4x16(uint2 p) {
    const uint32_t lo0 = (p.x << 4) & 0xf0f0f0f0u, hi0 = p.x & 0xf0f0f0f0u;
    const uint32_t lo1 = (p.y << 4) & 0xf0f0f0f0u, hi1 = p.y & 0xf0f0f0f0u;
    return make_uint4(__byte_perm(lo0, hi0, 0x5140), __byte_perm(lo0, hi0, 0x7362), __byte_perm(lo1, hi1, 0x5140),
                      __byte_perm(lo1, hi1, 0x7362));
}

// Xq: M x K int8 codes; Wq: N x K int8 (W4 = false) or N x K/2 packed int4
// (W4 = true); MT >= M is the compile-time token bound.  Block: nw warps
// (blockDim.x = 32 * nw), grid: ceil(N / 4) blocks.
template <bool W4, int MT>
__global__ void __launch_bounds__(256) gemv_i8_kernel(const int8_t *__restrict__ Xq, const float *__restrict__ sx,
                                                      const uint8_t *__restrict__ Wq, const float *__restrict__ sw,
                                                      const __half *__restrict__ bias, __half *__restrict__ Y,
                                                      int32_t *__restrict__ acc_out, int M, int N, int K) {
    constexpr int R = kGemvFeatures;
    constexpr int SHIFT = W4 ? 4 : 0;
    __shared__ int s_acc[8][R * MT];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nw = blockDim.x >> 5;
    const int n0 = blockIdx.x * R;
    pdl_wait();  // the codes and scales may come from the previous kernel
    pdl_launch_dependents();

    int acc[R][MT];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
        for (int m = 0; m < MT; ++m) acc[r][m] = 0;

    for (int k0 = warp * kGemvChunk; k0 < K; k0 += nw * kGemvChunk) {
        const int k = k0 + lane * 16;
        if (k < K) {
            uint4 w[R];
#pragma unroll
            for (int r = 0; r < R; ++r) {
                const int n = n0 + r;
                if (n < N) {
                    if (W4) w[r] = gemv_widen_int4x16(ld_stream_v2(Wq + static_cast<int64_t>(n) * (K / 2) + k / 2));
                    else w[r] = ld_stream_v4(Wq + static_cast<int64_t>(n) * K + k);
                } else {
                    w[r] = make_uint4(0, 0, 0, 0);
                }
            }
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                if (m < M) {
                    const uint4 a = __ldg(reinterpret_cast<const uint4 *>(Xq + static_cast<int64_t>(m) * K + k));
#pragma unroll
                    for (int r = 0; r < R; ++r) {
                        int t = acc[r][m];
                        t = __dp4a(static_cast<int>(a.x), static_cast<int>(w[r].x), t);
                        t = __dp4a(static_cast<int>(a.y), static_cast<int>(w[r].y), t);
                        t = __dp4a(static_cast<int>(a.z), static_cast<int>(w[r].z), t);
                        t = __dp4a(static_cast<int>(a.w), static_cast<int>(w[r].w), t);
                        acc[r][m] = t;
                    }
                }
            }
        }
    }
    // warp sums (exact), then the block's warps in order
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            const int v = __reduce_add_sync(0xffffffffu, acc[r][m]);
            if (lane == 0) s_acc[warp][r * MT + m] = v;
        }
    __syncthreads();
    for (int t = threadIdx.x; t < R * MT; t += blockDim.x) {
        const int r = t / MT, m = t - (t / MT) * MT;
        const int n = n0 + r;
        if (m < M && n < N) {
            int v = 0;
            for (int wi = 0; wi < nw; ++wi) v += s_acc[wi][t];
            const int32_t a = v >> SHIFT;
            const float bn = bias != nullptr ? __half2float(bias[n]) : 0.0f;
            const int64_t o = static_cast<int64_t>(m) * N + n;
            Y[o] = __float2half_rn(__fmaf_rn(__fmul_rn(__int2float_rn(a), sx[m]), sw[n], bn));
            if (acc_out != nullptr) acc_out[o] = a;
        }
    }
}

// ---------------------------------------------------------------------------
// The whole linear for a handful of tokens in one kernel: rotate + quantize
// fused with the weight-streaming GEMM.  With so few tokens the separate
// activation launch (a few microseconds of launch and ramp for a few KB of
// work) would be the critical path, so every CTA rotates and quantizes the
// M <= MT token rows itself into shared memory (the same butterfly stages, in
// the same order, as the activation kernel: the codes are bit-identical) while
// its first weight loads are in flight, then streams the weights of its share
// of the output features.
//   Grid: persistent CTAs of kGemvFusedThreads threads; CTA b owns features
//   [N b / grid, N (b+1) / grid).  Warp w takes 512-code chunk c = w mod C
//   (C = K / 512 <= 16) of every (w / C)-th of those features, in batches of
//   kGemvFusedBatch features whose loads are issued together; each (feature,
//   chunk) partial is a warp sum (exact int32) kept in shared memory, and the
//   chunks of a feature are added in order before the dequant.
//   CTA 0 also writes the codes and scales to xq_out / x_scale_out (the linear's
//   workspace holds them on return, as with two launches).
// ---------------------------------------------------------------------------
constexpr int kGemvFusedThreads = 512;
constexpr int kGemvFusedWarps = kGemvFusedThreads / 32;
constexpr int kGemvFusedBatch = 8;     // features whose weight loads a warp issues together
constexpr int kGemvFusedFeatBlock = 64;  // features whose partials are kept at once
constexpr int kGemvFusedMaxK = kGemvFusedWarps * kGemvChunk;  // 8192: every chunk has a warp

// Dynamic shared memory of the fused small-M kernel.
__host__ __device__ constexpr int gemv_fused_smem_bytes(int MT, int K) {
    return MT * K                                               // codes
           + 16 * 4                                             // scales (MT <= 16)
           + kGemvFusedFeatBlock * (K / kGemvChunk) * MT * 4    // (feature, chunk, token) partials
           + 2 * (kGemvFusedThreads / 4) * 4;                   // row-segment maxima
}

template <bool W4, int MT, int LOG2B>
__global__ void __launch_bounds__(kGemvFusedThreads, 1)
    gemv_fused_kernel(const __half *__restrict__ X, const uint8_t *__restrict__ Wq, const float *__restrict__ sw,
                      const __half *__restrict__ bias, __half *__restrict__ Y, int8_t *__restrict__ xq_out,
                      float *__restrict__ x_scale_out, int M, int N, int K) {
    constexpr int SHIFT = W4 ? 4 : 0;
    constexpr int BITS = W4 ? 4 : 8;
    extern __shared__ __align__(16) uint8_t gf_smem[];
    int8_t *codes = reinterpret_cast<int8_t *>(gf_smem);                        // [MT][K]
    float *s_x = reinterpret_cast<float *>(gf_smem + MT * K);                   // [MT]
    int *part = reinterpret_cast<int *>(gf_smem + MT * K + 64);                 // [FB][C][MT]
    const int C = K / kGemvChunk;
    float *s_seg = reinterpret_cast<float *>(part + kGemvFusedFeatBlock * C * MT);  // [2][128]
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int n_lo = static_cast<int>(static_cast<int64_t>(N) * blockIdx.x / gridDim.x);
    const int n_hi = static_cast<int>(static_cast<int64_t>(N) * (blockIdx.x + 1) / gridDim.x);
    // this warp's chunk and its place among the warps sharing that chunk
    const int c = warp % C, sub = warp / C, nsub = (kGemvFusedWarps - c + C - 1) / C;
    const int kc = c * kGemvChunk + lane * 16;  // first code of this lane's 16

    pdl_wait();  // X, the weights and the output may belong to the previous kernel
    pdl_launch_dependents();

    auto load_w = [&](int f) -> uint4 {
        if (W4) return gemv_widen_int4x16(ld_stream_v2(Wq + static_cast<int64_t>(f) * (K / 2) + kc / 2));
        return ld_stream_v4(Wq + static_cast<int64_t>(f) * K + kc);
    };
    // the first batch of weights is requested before the rotation
    uint4 wb[kGemvFusedBatch];
    int fb0 = n_lo;  // first feature of the current feature block
    {
#pragma unroll
        for (int i = 0; i < kGemvFusedBatch; ++i) {
            const int f = fb0 + sub + i * nsub;
            wb[i] = (f < n_hi && f < fb0 + kGemvFusedFeatBlock) ? load_w(f) : make_uint4(0, 0, 0, 0);
        }
    }

    // ---- rotate + quantize the token rows into shared memory
    {
        const int L = K / kElemsPerThread;
        const int rp = kGemvFusedThreads / L;  // rows per pass
        const int r = tid / L, l = tid - r * L;
        const int g = l >> 2, p = l & 3;
        const int elem0 = 128 * g + 8 * p;
        const int G = reduce_width(L);
        const int segs = L / G;
        for (int r0 = 0, it = 0; r0 < M; r0 += rp, ++it) {
            const int row = r0 + r;
            const bool act = r < rp && row < M;
            uint4 raw[4];
            if (act) {
                const __half *src = X + static_cast<int64_t>(row) * K + elem0;
#pragma unroll
                for (int j = 0; j < 4; ++j) raw[j] = ld_stream_v4(src + 32 * j);
            } else {
#pragma unroll
                for (int j = 0; j < 4; ++j) raw[j] = make_uint4(0, 0, 0, 0);
            }
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
                float *seg = s_seg + (it & 1) * (kGemvFusedThreads / 4);
                if (r < rp && (l & (G - 1)) == 0) seg[r * segs + l / G] = amax;
                __syncthreads();
                if (r < rp) {
                    amax = seg[r * segs];
                    for (int sg = 1; sg < segs; ++sg) amax = fmaxf(amax, seg[r * segs + sg]);
                }
            }
            if (act) {
                float fac1;
                const float sc = act_row_scale<LOG2B, BITS>(amax, &fac1);
                if (l == 0) {
                    s_x[row] = sc;
                    if (blockIdx.x == 0) x_scale_out[row] = sc;
                }
                const float2 fac = f2(fac1);
#pragma unroll
                for (int h = 0; h < 2; ++h)
#pragma unroll
                    for (int e = 0; e < 8; ++e) v[h][e] = __ffma2_rn(v[h][e], fac, f2(kRoundMagic));
                store_codes<8>(codes + static_cast<int64_t>(row) * K, elem0, v);
                if (blockIdx.x == 0) store_codes<8>(xq_out + static_cast<int64_t>(row) * K, elem0, v);
            }
        }
    }
    __syncthreads();

    // ---- stream the weights of this CTA's features
    uint4 a[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m)
        a[m] = m < M ? *reinterpret_cast<const uint4 *>(codes + m * K + kc) : make_uint4(0, 0, 0, 0);
    for (; fb0 < n_hi; fb0 += kGemvFusedFeatBlock) {
        const int fb1 = fb0 + kGemvFusedFeatBlock < n_hi ? fb0 + kGemvFusedFeatBlock : n_hi;
        {
            for (int i0 = 0;; i0 += kGemvFusedBatch) {
                const int fi0 = fb0 + sub + i0 * nsub;
                if (fi0 >= fb1) break;
                if (i0 > 0) {
#pragma unroll
                    for (int i = 0; i < kGemvFusedBatch; ++i) {
                        const int f = fi0 + i * nsub;
                        wb[i] = f < fb1 ? load_w(f) : make_uint4(0, 0, 0, 0);
                    }
                }
#pragma unroll
                for (int i = 0; i < kGemvFusedBatch; ++i) {
                    const int f = fi0 + i * nsub;
                    if (f >= fb1) break;
#pragma unroll
                    for (int m = 0; m < MT; ++m) {
                        int t = 0;
                        t = __dp4a(static_cast<int>(a[m].x), static_cast<int>(wb[i].x), t);
                        t = __dp4a(static_cast<int>(a[m].y), static_cast<int>(wb[i].y), t);
                        t = __dp4a(static_cast<int>(a[m].z), static_cast<int>(wb[i].z), t);
                        t = __dp4a(static_cast<int>(a[m].w), static_cast<int>(wb[i].w), t);
                        t = __reduce_add_sync(0xffffffffu, t);
                        if (lane == 0) part[((f - fb0) * C + c) * MT + m] = t;
                    }
                }
            }
        }
        __syncthreads();
        // the chunks of a feature, added in order; the dequantizing epilogue
        for (int t = tid; t < (fb1 - fb0) * MT; t += kGemvFusedThreads) {
            const int fl = t / MT, m = t - fl * MT;
            if (m < M) {
                int v = 0;
                for (int cc = 0; cc < C; ++cc) v += part[(fl * C + cc) * MT + m];
                const int n = fb0 + fl;
                const int32_t accv = v >> SHIFT;
                const float bn = bias != nullptr ? __half2float(bias[n]) : 0.0f;
                Y[static_cast<int64_t>(m) * N + n] =
                    __float2half_rn(__fmaf_rn(__fmul_rn(__int2float_rn(accv), s_x[m]), sw[n], bn));
            }
        }
        __syncthreads();  // the partials are read before the next block overwrites them
        // the next block's first batch
        if (fb0 + kGemvFusedFeatBlock < n_hi) {
            const int nb0 = fb0 + kGemvFusedFeatBlock;
            const int nb1 = nb0 + kGemvFusedFeatBlock < n_hi ? nb0 + kGemvFusedFeatBlock : n_hi;
#pragma unroll
            for (int i = 0; i < kGemvFusedBatch; ++i) {
                const int f = nb0 + sub + i * nsub;
                wb[i] = f < nb1 ? load_w(f) : make_uint4(0, 0, 0, 0);
            }
        }
    }
}

}  // namespace convrot
