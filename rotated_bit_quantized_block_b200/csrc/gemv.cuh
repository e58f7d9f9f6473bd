// gemv.cuh -- the integer GEMM with its dequantizing epilogue for a handful of
// tokens (the plan uses it up to 4 tokens with int8 weights, 8 with int4), as
// a weight-streaming kernel.
//
//   acc[m,n] = sum_k qx[m,k] * qw[n,k]            (exact int32, dp4a)
//   Y[m,n]   = fp16( fma( fp32(float(acc) * s_x[m]), s_w[n], bias[n] ) )
//
// Method: civarchive.com "SAM 3.1 Multiplex ConvRot" release, "Quantization
// recipe" (W8A8 / W4A4 operations, per-row scales).  With so few tokens the
// product is bound by reading the weights once from HBM, so the tensor core is
// not needed: each block owns 2, 4 or 8 output features, its warps split K into
// 512-code chunks (one 16-byte load per lane and feature), int4 weights are
// widened in registers, the activation codes (a few KB) come through L1.
#pragma once

#include "device_utils.cuh"

namespace convrot {

constexpr int kGemvChunk = 512;      // codes per warp step (32 lanes x 16)

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
// (W4 = true); MT >= M is the compile-time token bound, R the output features
// per block.  Block: nw <= 8 warps (blockDim.x = 32 * nw), grid: ceil(N / R).
template <bool W4, int MT, int R>
__global__ void __launch_bounds__(256) gemv_i8_kernel(const int8_t *__restrict__ Xq, const float *__restrict__ sx,
                                                      const uint8_t *__restrict__ Wq, const float *__restrict__ sw,
                                                      const __half *__restrict__ bias, __half *__restrict__ Y,
                                                      int32_t *__restrict__ acc_out, int M, int N, int K) {
    constexpr int SHIFT = W4 ? 4 : 0;
    __shared__ int s_acc[8][R * MT];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nw = blockDim.x >> 5;
    const int n0 = blockIdx.x * R;
    auto load_w = [&](int k, uint4 (&w)[R]) {
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
    };
    if (threadIdx.x == 0) {
        // the block's weight rows are contiguous: one bulk prefetch into L2 (TMA)
        // puts them in flight at once, ahead of the lanes' loads.  The weights
        // are not written by the previous kernel in the stream and a prefetch
        // cannot return stale data, so it goes out before the dependency wait
        // and overlaps the activation launch.
        const int rows = N - n0 < R ? N - n0 : R;
        const int64_t rowb = W4 ? K / 2 : K;
        asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(Wq + static_cast<int64_t>(n0) * rowb),
                     "r"(static_cast<uint32_t>(rows * rowb))
                     : "memory");
    }
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
            load_w(k, w);
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

}  // namespace convrot
