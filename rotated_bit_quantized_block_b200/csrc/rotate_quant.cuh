// rotate_quant.cuh -- block-Hadamard rotation fused with symmetric per-row
// quantization, for activations (online, per token) and weights (offline,
// per output row, with the MSE clip search).
//
// Method: civarchive.com "SAM 3.1 Multiplex ConvRot" release, "Quantization
// recipe" (block-Hadamard ConvRot transform, per-row scales, online dynamic
// activation quantization); trellis3d.app "TRELLIS.2 INT8 ConvRot",
// "What ConvRot changes" (grouped, normalized Hadamard rotation of weights and
// the matching rotation of activations).
//
// Register layout.  A row of K elements is split into 128-element groups;
// four consecutive threads own one group, each holding 32 elements as four
// 16-byte chunks: thread l of the row (g = l / 4, p = l % 4) holds, for chunk
// j in 0..3 and e in 0..7, element 128*g + 8*p + 32*j + e.  Index bits 0-2
// (e) and 5-6 (j) are butterflied in registers, bits 3 and 4 (p) between lanes
// l^1 and l^2, and bit 7 (g's low bit, blocks of 256) between lanes l^4.  The
// values are kept as float2 pairs (chunk h, chunk h + 2) so that every stage
// but the one on bit 6 runs on the packed fp32x2 pipe.
#pragma once

#include "device_utils.cuh"

namespace convrot {

constexpr int kThreadsPerRowGroup = 4;  // threads per 128 elements
constexpr int kElemsPerThread = 32;
constexpr int kMaxRowsPerCta = 64;       // 256 threads / 4 threads per row (K = 128)
constexpr float kRoundMagic = 12582912.0f;  // 1.5 * 2^23: x + magic rounds x to an integer (RNE)

// fp32(1 / sqrt(2^L)), L = 0..8 (correctly rounded decimal literals).
__device__ __forceinline__ float rsqrt_block(int log2b) {
    switch (log2b) {
        case 0: return 1.0f;
        case 1: return 0.70710678118654752440f;
        case 2: return 0.5f;
        case 3: return 0.35355339059327376220f;
        case 4: return 0.25f;
        case 5: return 0.17677669529663688110f;
        case 6: return 0.125f;
        case 7: return 0.088388347648318440550f;
        default: return 0.0625f;
    }
}

__device__ __forceinline__ float2 f2(float a) { return make_float2(a, a); }

// a - b on the packed pipe (b * -1 is exact, so this is one rounding).
__device__ __forceinline__ float2 sub2(float2 a, float2 b) { return __ffma2_rn(b, f2(-1.0f), a); }

// One butterfly stage between lanes `lane` and `lane ^ m`: the lower lane keeps
// a + b, the upper one a - b (a = lower lane's value, b = upper lane's).
__device__ __forceinline__ void lane_stage(float2 (&v)[2][8], int lane, int m) {
    const float sgn = (lane & m) ? -1.0f : 1.0f;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            float2 other;
            other.x = __shfl_xor_sync(0xffffffffu, v[h][e].x, m);
            other.y = __shfl_xor_sync(0xffffffffu, v[h][e].y, m);
            v[h][e] = __ffma2_rn(v[h][e], f2(sgn), other);
        }
    }
}

// Unnormalized Walsh-Hadamard transform (Sylvester order) of every block of
// 2^LOG2B elements held by the thread group (see the layout above).
template <int LOG2B>
__device__ __forceinline__ void fwht_block(float2 (&v)[2][8], int lane) {
#pragma unroll
    for (int k = 0; k < 3; ++k) {
        if (k < LOG2B) {
            const int m = 1 << k;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    if (!(e & m)) {
                        const float2 a = v[h][e], b = v[h][e | m];
                        v[h][e] = __fadd2_rn(a, b);
                        v[h][e | m] = sub2(a, b);
                    }
                }
            }
        }
    }
    if (LOG2B > 3) lane_stage(v, lane, 1);
    if (LOG2B > 4) lane_stage(v, lane, 2);
    if (LOG2B > 5) {  // bit 5: chunk pairs (0,1) and (2,3) -> h = 0 vs h = 1
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const float2 a = v[0][e], b = v[1][e];
            v[0][e] = __fadd2_rn(a, b);
            v[1][e] = sub2(a, b);
        }
    }
    if (LOG2B > 6) {  // bit 6: chunk j vs j + 2 -> inside each float2
#pragma unroll
        for (int h = 0; h < 2; ++h) {
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float a = v[h][e].x, b = v[h][e].y;
                v[h][e] = make_float2(__fadd_rn(a, b), __fsub_rn(a, b));
            }
        }
    }
    if (LOG2B > 7) lane_stage(v, lane, 4);
}

// Loads the thread's 32 source elements of one row and upcasts them to fp32.
// dtype: 0 fp16, 1 bf16, 2 fp32.  `elem0` = 128*g + 8*p.
__device__ __forceinline__ void load_row_chunks(const void *row_base, int dtype, int elem0, float2 (&v)[2][8]) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        float f[8];
        if (dtype == 2) {
            const float *src = static_cast<const float *>(row_base) + elem0 + 32 * j;
            const uint4 a = ld_stream_v4(src), b = ld_stream_v4(src + 4);
            f[0] = __uint_as_float(a.x); f[1] = __uint_as_float(a.y);
            f[2] = __uint_as_float(a.z); f[3] = __uint_as_float(a.w);
            f[4] = __uint_as_float(b.x); f[5] = __uint_as_float(b.y);
            f[6] = __uint_as_float(b.z); f[7] = __uint_as_float(b.w);
        } else {
            const uint16_t *src = static_cast<const uint16_t *>(row_base) + elem0 + 32 * j;
            const uint4 a = ld_stream_v4(src);
            const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                if (dtype == 0) {
                    const float2 p = __half22float2(*reinterpret_cast<const __half2 *>(&w[i]));
                    f[2 * i] = p.x;
                    f[2 * i + 1] = p.y;
                } else {
                    f[2 * i] = __uint_as_float(w[i] << 16);
                    f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
                }
            }
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            if (j < 2) v[j][e].x = f[e];
            else v[j - 2][e].y = f[e];
        }
    }
}

__device__ __forceinline__ float chunk_val(const float2 (&v)[2][8], int j, int e) {
    return j < 2 ? v[j][e].x : v[j - 2][e].y;
}

// Low byte of the bit pattern of (t + 1.5*2^23) for an integer-rounded t:
// rne(t) in 8-bit two's complement.
__device__ __forceinline__ uint32_t code_bits(const float2 (&r)[2][8], int j, int e) {
    return __float_as_uint(chunk_val(r, j, e));
}

// Packs the 8 codes of chunk j (low bytes of `r`) as int8: two 32-bit words.
__device__ __forceinline__ uint2 pack_int8_chunk(const float2 (&r)[2][8], int j) {
    const uint32_t a = __byte_perm(code_bits(r, j, 0), code_bits(r, j, 1), 0x0040);
    const uint32_t b = __byte_perm(code_bits(r, j, 2), code_bits(r, j, 3), 0x0040);
    const uint32_t c = __byte_perm(code_bits(r, j, 4), code_bits(r, j, 5), 0x0040);
    const uint32_t d = __byte_perm(code_bits(r, j, 6), code_bits(r, j, 7), 0x0040);
    return make_uint2(__byte_perm(a, b, 0x5410), __byte_perm(c, d, 0x5410));
}

// Packs the 8 codes of chunk j as int4: byte i = code[2i] | code[2i+1] << 4.
__device__ __forceinline__ uint32_t pack_int4_chunk(const float2 (&r)[2][8], int j) {
    const uint32_t e02 = __byte_perm(code_bits(r, j, 0), code_bits(r, j, 2), 0x0040);
    const uint32_t e46 = __byte_perm(code_bits(r, j, 4), code_bits(r, j, 6), 0x0040);
    const uint32_t e13 = __byte_perm(code_bits(r, j, 1), code_bits(r, j, 3), 0x0040);
    const uint32_t e57 = __byte_perm(code_bits(r, j, 5), code_bits(r, j, 7), 0x0040);
    const uint32_t even = __byte_perm(e02, e46, 0x5410);
    const uint32_t odd = __byte_perm(e13, e57, 0x5410);
    return (even & 0x0f0f0f0fu) | ((odd & 0x0f0f0f0fu) << 4);
}

// Stores the thread's 32 codes (already in the low bytes of `r`).
template <int BITS>
__device__ __forceinline__ void store_codes(void *out_row, int elem0, const float2 (&r)[2][8]) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        if (BITS == 8) {
            *reinterpret_cast<uint2 *>(static_cast<int8_t *>(out_row) + elem0 + 32 * j) = pack_int8_chunk(r, j);
        } else {
            *reinterpret_cast<uint32_t *>(static_cast<uint8_t *>(out_row) + (elem0 + 32 * j) / 2) =
                pack_int4_chunk(r, j);
        }
    }
}

// clamp(rne(x * inv), qmin, qmax) as an exact integer-valued float: the fused
// multiply-add rounds the exact product once onto the integer grid of
// [2^23, 2^24), and removing the offset again is exact.
__device__ __forceinline__ float quant_clamped(float x, float inv, int qmin, int qmax) {
    const float r = __fsub_rn(__fmaf_rn(x, inv, kRoundMagic), kRoundMagic);
    return fminf(fmaxf(r, static_cast<float>(qmin)), static_cast<float>(qmax));
}

// Largest power of two dividing L, at most 32: the lanes of one row that a
// shuffle reduction may combine.
__host__ __device__ __forceinline__ int reduce_width(int L) {
    int g = L & (-L);
    return g > 32 ? 32 : g;
}

// ---------------------------------------------------------------------------
// Online activation path: X (fp16, M x K) -> codes + per-token scales.
//
// A row of K elements is handled by L = K/32 threads, each owning 32 elements
// of a 128-element group in two register layouts:
//   layout A: element 8p + 32j + e (chunks j = 0..3 of 8 e; p = thread in the
//             group), packed as float2 (e, e+1): butterflies on bits 1, 2, 5, 6;
//   layout B: element 32p + i (i = 0..31 contiguous), packed as float2
//             (i, i+2): butterflies on bits 0, 3, 4 (bit 7, blocks of 256,
//             between lanes l^4).
// A -> B goes through a swizzled, bank-conflict-free 528-byte buffer per
// group, so every butterfly runs on the packed fp32x2 pipe and each thread
// ends with 32 contiguous codes (16-byte stores).  The 1/sqrt(b) factor is
// folded into the per-row code factor (exact when b is a power of 4).
//
// The fused linear's activation warps (end of this section) run the same
// stages in another register layout.
// ---------------------------------------------------------------------------
constexpr int kXposeGroupBytes = 33 * 16;  // 32 16-byte units + 1 unit of padding

// 16-byte unit u (0..31) of a group's transpose buffer lives at this unit slot.
__device__ __forceinline__ int xpose_slot(int u) { return (u & 24) | ((u & 7) ^ ((u >> 2) & 6)); }

__device__ __forceinline__ void bfly2(float2 &a, float2 &b) {
    const float2 s = __fadd2_rn(a, b);
    b = sub2(a, b);
    a = s;
}

// max(m, |x|, |y|)
__device__ __forceinline__ float absmax3(float m, float x, float y) {
    return fmaxf(m, fmaxf(fabsf(x), fabsf(y)));
}

// Dynamic shared memory of the register-fed activation kernel for a block of `threads`.
__host__ __device__ constexpr int act_smem_bytes(int threads) { return (threads / 4) * kXposeGroupBytes; }

// Layout A from the four loaded 16-byte chunks (8 fp16 each), then the
// butterfly stages on index bits 1, 2, 5, 6.  With `stagger` set, register
// chunk j holds the group's chunk j ^ 1 (a warp's staggered shared-memory
// reads then hit distinct banks); the bit-5 stage puts the pair back in
// natural order (x0 + x1 into chunk 0, x0 - x1 = -(x1 - x0) into chunk 1,
// bit-identical to the unstaggered result).  Below b = 64 there is no bit-5
// stage and the caller undoes the stagger in the transpose.
template <int LOG2B>
__device__ __forceinline__ void act_layout_a(const uint4 (&raw)[4], bool stagger, float2 (&a)[4][4]) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint32_t ww[4] = {raw[j].x, raw[j].y, raw[j].z, raw[j].w};
#pragma unroll
        for (int k = 0; k < 4; ++k) a[j][k] = __half22float2(*reinterpret_cast<const __half2 *>(&ww[k]));
    }
    if (LOG2B > 1) {  // bit 1
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            bfly2(a[j][0], a[j][1]);
            bfly2(a[j][2], a[j][3]);
        }
    }
    if (LOG2B > 2) {  // bit 2
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            bfly2(a[j][0], a[j][2]);
            bfly2(a[j][1], a[j][3]);
        }
    }
    if (LOG2B > 5) {  // bit 5
        const float2 sg = f2(stagger ? -1.0f : 1.0f);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
#pragma unroll
            for (int j = 0; j < 4; j += 2) {
                const float2 s = __fadd2_rn(a[j][k], a[j + 1][k]);
                a[j + 1][k] = __fmul2_rn(sub2(a[j][k], a[j + 1][k]), sg);
                a[j][k] = s;
            }
        }
    }
    if (LOG2B > 6) {  // bit 6
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            bfly2(a[0][k], a[2][k]);
            bfly2(a[1][k], a[3][k]);
        }
    }
}

// A -> B through the group's transpose buffer (jx: register chunk j is the
// group's chunk j ^ jx), then the stages on bits 0, 3, 4 and (b = 256) bit 7.
// Every lane of the warp must call it (bit 7 uses shuffles).
template <int LOG2B>
__device__ __forceinline__ void act_layout_b(const float2 (&a)[4][4], uint8_t *xbuf, int p, int jx, int lane,
                                             float2 (&bv)[8][2]) {
    // unit u = 2p + 8j + h holds elements 4u .. 4u + 3 = a[j][2h], a[j][2h+1]
#pragma unroll
    for (int j = 0; j < 4; ++j) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            *reinterpret_cast<float4 *>(xbuf + 16 * xpose_slot(2 * p + 8 * (j ^ jx) + h)) =
                make_float4(a[j][2 * h].x, a[j][2 * h].y, a[j][2 * h + 1].x, a[j][2 * h + 1].y);
        }
    }
    __syncwarp();
    // layout B: b[m][c] = (x[32p + 4m + c], x[32p + 4m + c + 2])
#pragma unroll
    for (int m = 0; m < 8; ++m) {
        const float4 f = *reinterpret_cast<const float4 *>(xbuf + 16 * xpose_slot(8 * p + m));
        bv[m][0] = make_float2(f.x, f.z);
        bv[m][1] = make_float2(f.y, f.w);
    }
    if (LOG2B > 0) {  // bit 0
#pragma unroll
        for (int m = 0; m < 8; ++m) bfly2(bv[m][0], bv[m][1]);
    }
    if (LOG2B > 3) {  // bit 3
#pragma unroll
        for (int m = 0; m < 8; ++m)
            if (!(m & 2)) {
                bfly2(bv[m][0], bv[m + 2][0]);
                bfly2(bv[m][1], bv[m + 2][1]);
            }
    }
    if (LOG2B > 4) {  // bit 4
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            bfly2(bv[m][0], bv[m + 4][0]);
            bfly2(bv[m][1], bv[m + 4][1]);
        }
    }
    if (LOG2B > 7) {  // bit 7: the neighbouring 128-element group, lane l ^ 4
        const float sgn = (lane & 4) ? -1.0f : 1.0f;
#pragma unroll
        for (int m = 0; m < 8; ++m) {
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                float2 o;
                o.x = __shfl_xor_sync(0xffffffffu, bv[m][c].x, 4);
                o.y = __shfl_xor_sync(0xffffffffu, bv[m][c].y, 4);
                bv[m][c] = __ffma2_rn(bv[m][c], f2(sgn), o);
            }
        }
    }
}

// max |y| over the thread's 32 values (y = unnormalized rotation).
__device__ __forceinline__ float act_local_absmax(const float2 (&bv)[8][2]) {
    float amax = 0.0f;
#pragma unroll
    for (int m = 0; m < 8; ++m)
#pragma unroll
        for (int c = 0; c < 2; ++c) amax = absmax3(amax, bv[m][c].x, bv[m][c].y);
    return amax;
}

// The row's scale and code factor from its max |y|: max|x~| = fp32(max|y| *
// rsqrt(b)) (rounding is monotone), s = fp32(that / qmax); the code of x~ =
// y * rsqrt(b) is rne(x~ * fp32(1/s)), taken as rne(y * fac) with one factor
// per row, fac = fp32(rsqrt(b) * fp32(1/s)).
template <int LOG2B, int BITS>
__device__ __forceinline__ float act_row_scale(float amax, float *fac) {
    constexpr float qmax = BITS == 8 ? 127.0f : 7.0f;
    const float rb = rsqrt_block(LOG2B);
    const float sc = __fdiv_rn(__fmul_rn(amax, rb), qmax);
    *fac = sc == 0.0f ? 0.0f : __fmul_rn(rb, __frcp_rn(sc));
    return sc;
}

// Quantizes the thread's 32 values (one fused multiply-add each onto the
// integer grid, see quant_clamped) and stores them: 32 bytes at element
// 128g + 32p of the row, or 16 bytes of packed int4.
template <int BITS, bool PACKED>
__device__ __forceinline__ void act_store_codes(float2 (&bv)[8][2], float fac1, void *Xq, int64_t row, int K, int g,
                                                int p) {
    const float2 fac = f2(fac1);
#pragma unroll
    for (int m = 0; m < 8; ++m)
#pragma unroll
        for (int c = 0; c < 2; ++c) bv[m][c] = __ffma2_rn(bv[m][c], fac, f2(kRoundMagic));
    // element 4m + q of the run: q = 0 -> b[m][0].x, 1 -> b[m][1].x, 2 -> b[m][0].y, 3 -> b[m][1].y
    uint32_t wd[8];
#pragma unroll
    for (int m = 0; m < 8; ++m) {
        const uint32_t c01 = __byte_perm(__float_as_uint(bv[m][0].x), __float_as_uint(bv[m][1].x), 0x0040);
        const uint32_t c23 = __byte_perm(__float_as_uint(bv[m][0].y), __float_as_uint(bv[m][1].y), 0x0040);
        wd[m] = __byte_perm(c01, c23, 0x5410);
    }
    if (!PACKED) {
        int8_t *dst = static_cast<int8_t *>(Xq) + row * K + 128 * g + 32 * p;
        *reinterpret_cast<uint4 *>(dst) = make_uint4(wd[0], wd[1], wd[2], wd[3]);
        *reinterpret_cast<uint4 *>(dst + 16) = make_uint4(wd[4], wd[5], wd[6], wd[7]);
    } else {
        // int4 byte = code[2i] | code[2i+1] << 4
        uint32_t nb[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint32_t even = __byte_perm(wd[2 * i], wd[2 * i + 1], 0x6420);
            const uint32_t odd = __byte_perm(wd[2 * i], wd[2 * i + 1], 0x7531);
            nb[i] = (even & 0x0f0f0f0fu) | ((odd & 0x0f0f0f0fu) << 4);
        }
        uint8_t *dst = static_cast<uint8_t *>(Xq) + row * (K / 2) + 64 * g + 16 * p;
        *reinterpret_cast<uint4 *>(dst) = make_uint4(nb[0], nb[1], nb[2], nb[3]);
    }
}

// Packed int4 weight codes (a byte holds element 2j in its low nibble and
// 2j+1 in its high nibble, two's complement) to one int8 code per byte, in
// element order: 16 packed bytes in, 32 code bytes out.
__device__ __forceinline__ void widen_int4_to_int8(uint4 p, uint4 &out0, uint4 &out1) {
    const uint32_t w[4] = {p.x, p.y, p.z, p.w};
    uint32_t o[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        // sign-extend each nibble within its byte: (n ^ 8) - 8, bytewise
        const uint32_t lo = __vsub4((w[i] & 0x0f0f0f0fu) ^ 0x08080808u, 0x08080808u);
        const uint32_t hi = __vsub4(((w[i] >> 4) & 0x0f0f0f0fu) ^ 0x08080808u, 0x08080808u);
        o[2 * i] = __byte_perm(lo, hi, 0x5140);
        o[2 * i + 1] = __byte_perm(lo, hi, 0x7362);
    }
    out0 = make_uint4(o[0], o[1], o[2], o[3]);
    out1 = make_uint4(o[4], o[5], o[6], o[7]);
}

// BITS fixes the code range (8: [-127, 127], 4: [-8, 7]); PACKED stores int4
// codes two per byte, otherwise every code takes one byte.
// One CTA handles `rows` consecutive rows with L = K/32 threads each (the
// block is padded to a multiple of 32 threads; padding threads only join the
// barriers).  Every thread issues its four 16-byte loads up front.
template <int LOG2B, int BITS, bool PACKED>
__global__ void __launch_bounds__(1024) act_rotate_quant_kernel(const __half *__restrict__ X, int64_t M, int K,
                                                                int rows, void *__restrict__ Xq,
                                                                float *__restrict__ x_scale,
                                                                uint4 *__restrict__ zero16,
                                                                int64_t n_zero16,
                                                                const uint4 *__restrict__ w_packed,
                                                                uint4 *__restrict__ w_wide, int64_t n_w16,
                                                                int pf_ahead) {
    extern __shared__ __align__(16) uint8_t act_smem[];
    __shared__ unsigned int s_amax[kMaxRowsPerCta];
    __shared__ float s_fac[kMaxRowsPerCta];
    const int L = K / kElemsPerThread;
    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int r = tid / L;
    const int l = tid - r * L;
    const int64_t row = static_cast<int64_t>(blockIdx.x) * rows + r;
    const bool active = (r < rows) && (row < M);
    const int g = l >> 2, p = l & 3;
    uint8_t *xbuf = act_smem + (tid >> 2) * kXposeGroupBytes;

    if (tid == 0 || (tid == 32 && pf_ahead > 0)) {
        // A CTA's rows are contiguous: one bulk prefetch into L2 (TMA, no
        // shared memory) puts all of their bytes in flight at once, ahead of
        // the threads' own loads.  When the grid has more CTAs than fit the
        // GPU at once, the CTA also prefetches the rows of the CTA pf_ahead
        // places later, which runs in the next wave.  (Measured: own rows +6 %
        // to +17 %; one wave ahead another +4 % to +12 % on multi-wave grids.)
        // It goes out before the grid-dependency wait: a prefetch is only a
        // hint and L2 is the point of coherence, so rows that the previous
        // kernel is still writing are read correctly by the loads after the
        // wait, and CTAs that become resident during the previous kernel's
        // last partial round of tiles overlap their reads with it.
        const int64_t cta = static_cast<int64_t>(blockIdx.x) + (tid == 0 ? 0 : pf_ahead);
        const int64_t r0 = cta * rows;
        if (r0 < M) {
            const int64_t nr = M - r0 < rows ? M - r0 : rows;
            asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(X + r0 * K),
                         "r"(static_cast<uint32_t>(nr * K * 2))
                         : "memory");
        }
    }
    pdl_wait();  // X may come from, and Xq may still be read by, the previous kernel
    pdl_launch_dependents();
    uint4 raw[4];
    if (active) {
        const __half *src = X + row * K + 128 * g + 8 * p;
#pragma unroll
        for (int j = 0; j < 4; ++j) raw[j] = ld_stream_v4(src + 32 * j);
    } else {
#pragma unroll
        for (int j = 0; j < 4; ++j) raw[j] = make_uint4(0, 0, 0, 0);
    }
    // (while the row loads are in flight) the linear's counters start at zero for the GEMM that follows
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + tid; i < n_zero16;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x)
        zero16[i] = make_uint4(0u, 0u, 0u, 0u);
    // the W4A4 linear's packed int4 weights, widened once to int8 codes for the
    // GEMM that follows (n_w16 units of 16 packed bytes)
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + tid; i < n_w16;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        uint4 o0, o1;
        widen_int4_to_int8(ld_stream_v4(w_packed + i), o0, o1);
        w_wide[2 * i] = o0;
        w_wide[2 * i + 1] = o1;
    }
    if (tid < rows) s_amax[tid] = 0u;
    float2 a[4][4];
    act_layout_a<LOG2B>(raw, false, a);
    float2 bv[8][2];
    act_layout_b<LOG2B>(a, xbuf, p, 0, lane, bv);
    float amax = act_local_absmax(bv);
    const int G = reduce_width(L);
    for (int mm = 1; mm < G; mm <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, mm));
    float fac1;
    if (G == L) {
        // the whole row lives in this warp: no block-wide step
        if (!active) return;
        const float sc = act_row_scale<LOG2B, BITS>(amax, &fac1);
        if (l == 0) x_scale[row] = sc;
    } else {
        __syncthreads();  // s_amax initialised
        if (r < rows && (l & (G - 1)) == 0) atomicMax(&s_amax[r], __float_as_uint(amax));  // amax >= 0
        __syncthreads();
        if (active && l == 0) {
            float f;
            x_scale[row] = act_row_scale<LOG2B, BITS>(__uint_as_float(s_amax[r]), &f);
            s_fac[r] = f;
        }
        __syncthreads();
        if (!active) return;
        fac1 = s_fac[r];
    }
    act_store_codes<BITS, PACKED>(bv, fac1, Xq, row, K, g, p);
}

// ---- the fused linear's activation warps ------------------------------------
//
// The same rotation in the register layout of fwht_block (thread l of the
// row: element 128g + 8p + 32j + e, v[h][e] = (chunk h, chunk h + 2)), with no
// shared memory: index bits 3 and 4 go between lanes l^1 and l^2.  The stages
// run in the order of the activation kernel above (bits 1, 2, 5, 6, 0, 3, 4,
// 7), so every sum is rounded in the same sequence and the codes are
// bit-identical to that kernel's.
template <int LOG2B>
__device__ __forceinline__ void fwht_act_order(float2 (&v)[2][8], int lane) {
#pragma unroll
    for (int k = 1; k < 3; ++k) {  // bits 1, 2: e ^ m inside a chunk
        if (k < LOG2B) {
            const int m = 1 << k;
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    if (!(e & m)) bfly2(v[h][e], v[h][e | m]);
        }
    }
    if (LOG2B > 5) {  // bit 5: chunk pairs (0,1) and (2,3) -> h = 0 vs h = 1
#pragma unroll
        for (int e = 0; e < 8; ++e) bfly2(v[0][e], v[1][e]);
    }
    if (LOG2B > 6) {  // bit 6: chunk j vs j + 2 -> inside each float2
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float a = v[h][e].x, b = v[h][e].y;
                v[h][e] = make_float2(__fadd_rn(a, b), __fsub_rn(a, b));
            }
    }
    if (LOG2B > 0) {  // bit 0
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int e = 0; e < 8; e += 2) bfly2(v[h][e], v[h][e + 1]);
    }
    if (LOG2B > 3) lane_stage(v, lane, 1);
    if (LOG2B > 4) lane_stage(v, lane, 2);
    if (LOG2B > 7) lane_stage(v, lane, 4);
}

// The thread's 32 fp16 elements (four 16-byte chunks j, 8 each) in fwht_block's layout.
__device__ __forceinline__ void raw_to_v(const uint4 (&raw)[4], float2 (&v)[2][8]) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint32_t ww[4] = {raw[j].x, raw[j].y, raw[j].z, raw[j].w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&ww[k]));
            if (j < 2) {
                v[j][2 * k].x = f.x;
                v[j][2 * k + 1].x = f.y;
            } else {
                v[j - 2][2 * k].y = f.x;
                v[j - 2][2 * k + 1].y = f.y;
            }
        }
    }
}

// ---------------------------------------------------------------------------
// Offline weight path: W (fp16/bf16/fp32, N x K) -> fp32 -> rotation ->
// per-row clip search -> codes + per-row scales.  Same thread layout as the
// activation kernel.  The squared errors are reduced in a fixed order
// (lanes, then row segments in index order), so the choice is deterministic.
// ---------------------------------------------------------------------------
constexpr int kMseGrid = 51;
constexpr int kMseBatch = 4;  // grid points scored per pass (one pair of block barriers per pass)

//
// Tensor-wise scales use the same kernel in three passes (all optional
// pointers null = the row-wise converter):
//   row_amax_out   stats pass: write each row's absmax and stop;
//   row_err_out    error pass: with the tensor's absmax `given_amax`, write each
//                  row's float64 error for every grid point and stop;
//   given_amax / given_alpha   quantize every row with that absmax and grid point.
template <int LOG2B>
__global__ void __launch_bounds__(1024) weight_rotate_quant_kernel(const void *__restrict__ W, int dtype,
                                                                   int64_t N, int K, int rows, int bits,
                                                                   int clip_mode, void *__restrict__ Wq,
                                                                   float *__restrict__ w_scale,
                                                                   const float *__restrict__ given_amax,
                                                                   const int *__restrict__ given_alpha,
                                                                   float *__restrict__ row_amax_out,
                                                                   double *__restrict__ row_err_out) {
    __shared__ unsigned int s_amax[kMaxRowsPerCta];
    __shared__ float s_scale[kMaxRowsPerCta][kMseGrid];
    // one partial sum per (row, segment of G lanes, grid point of the batch): at most 1024 / 4 x batch
    __shared__ double s_part[256 * kMseBatch];
    __shared__ double s_best_err[kMaxRowsPerCta];
    __shared__ int s_best[kMaxRowsPerCta];
    const int L = K / kElemsPerThread;
    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int r = tid / L;
    const int l = tid - r * L;
    const int64_t row = static_cast<int64_t>(blockIdx.x) * rows + r;
    const bool active = (r < rows) && (row < N);
    const int elem0 = 128 * (l >> 2) + 8 * (l & 3);
    const int qmax = bits == 8 ? 127 : 7;
    const int qmin = bits == 8 ? -127 : -8;
    const int G = reduce_width(L);
    const int segs = L / G;

    float2 v[2][8];
    if (active) {
        const size_t esize = dtype == 2 ? 4 : 2;
        load_row_chunks(static_cast<const char *>(W) + row * K * esize, dtype, elem0, v);
    } else {
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int e = 0; e < 8; ++e) v[h][e] = f2(0.0f);
    }
    if (tid < rows) {
        s_amax[tid] = 0u;
        s_best[tid] = 0;
        s_best_err[tid] = __longlong_as_double(0x7ff0000000000000ll);  // +inf
    }
    __syncthreads();
    fwht_block<LOG2B>(v, lane);
    const float2 rb = f2(rsqrt_block(LOG2B));
    float amax = 0.0f;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            v[h][e] = __fmul2_rn(v[h][e], rb);
            amax = fmaxf(amax, fmaxf(fabsf(v[h][e].x), fabsf(v[h][e].y)));
        }
    }
    for (int m = 1; m < G; m <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, m));
    if (r < rows && (l & (G - 1)) == 0) atomicMax(&s_amax[r], __float_as_uint(amax));
    __syncthreads();
    if (row_amax_out != nullptr) {  // stats pass (uniform across the block)
        if (active && l == 0) row_amax_out[row] = __uint_as_float(s_amax[r]);
        return;
    }
    const bool search = clip_mode == 1 && given_alpha == nullptr;
    const int n_alpha = search ? kMseGrid : 1;
    const int alpha0 = given_alpha != nullptr ? *given_alpha : 0;
    // grid point i: alpha = fp32((100 - i) / 100), s = fp32(fp32(alpha * amax) / qmax)
    if (r < rows) {
        const float am = given_amax != nullptr ? *given_amax : __uint_as_float(s_amax[r]);
        for (int i = l; i < n_alpha; i += L) {
            const int ai = search ? i : alpha0;
            const float alpha = __fdiv_rn(static_cast<float>(100 - ai), 100.0f);
            s_scale[r][i] = __fdiv_rn(__fmul_rn(alpha, am), static_cast<float>(qmax));
        }
    }
    __syncthreads();
    if (n_alpha > 1) {
        // kMseBatch grid points per pass; each point's float64 error is summed in
        // the same order as one point at a time (elements, lanes, then segments)
        for (int i0 = 0; i0 < n_alpha; i0 += kMseBatch) {
            float inv[kMseBatch];
            double sd[kMseBatch], err[kMseBatch];
#pragma unroll
            for (int a = 0; a < kMseBatch; ++a) {
                const float s = (r < rows && i0 + a < n_alpha) ? s_scale[r][i0 + a] : 0.0f;
                inv[a] = s == 0.0f ? 0.0f : __frcp_rn(s);
                sd[a] = static_cast<double>(s);
                err[a] = 0.0;
            }
#pragma unroll
            for (int h = 0; h < 2; ++h) {
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float xs[2] = {v[h][e].x, v[h][e].y};
#pragma unroll
                    for (int c = 0; c < 2; ++c) {
#pragma unroll
                        for (int a = 0; a < kMseBatch; ++a) {
                            const float q = quant_clamped(xs[c], inv[a], qmin, qmax);
                            const double d = fma(-sd[a], static_cast<double>(q), static_cast<double>(xs[c]));
                            err[a] = fma(d, d, err[a]);
                        }
                    }
                }
            }
#pragma unroll
            for (int a = 0; a < kMseBatch; ++a)
                for (int m = 1; m < G; m <<= 1) err[a] += __shfl_xor_sync(0xffffffffu, err[a], m);
            if (r < rows && (l & (G - 1)) == 0) {
#pragma unroll
                for (int a = 0; a < kMseBatch; ++a) s_part[(r * segs + l / G) * kMseBatch + a] = err[a];
            }
            __syncthreads();
            if (r < rows && l == 0) {
                for (int a = 0; a < kMseBatch && i0 + a < n_alpha; ++a) {
                    double tot = 0.0;
                    for (int sgi = 0; sgi < segs; ++sgi) tot += s_part[(r * segs + sgi) * kMseBatch + a];
                    if (row_err_out != nullptr && active) row_err_out[row * kMseGrid + i0 + a] = tot;
                    if (tot < s_best_err[r]) {
                        s_best_err[r] = tot;
                        s_best[r] = i0 + a;
                    }
                }
            }
            __syncthreads();
        }
    }
    if (row_err_out != nullptr || !active) return;  // the error pass ends here
    const float s = s_scale[r][s_best[r]];
    const float inv = s == 0.0f ? 0.0f : __frcp_rn(s);
    if (l == 0) w_scale[row] = s;
    float2 q[2][8];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const float a = quant_clamped(v[h][e].x, inv, qmin, qmax);
            const float b = quant_clamped(v[h][e].y, inv, qmin, qmax);
            // re-encode the (exact, small) integers with the rounding magic so
            // that the packers can take their low bytes
            q[h][e] = make_float2(__fadd_rn(a, kRoundMagic), __fadd_rn(b, kRoundMagic));
        }
    }
    if (bits == 8) store_codes<8>(static_cast<int8_t *>(Wq) + row * K, elem0, q);
    else store_codes<4>(static_cast<uint8_t *>(Wq) + row * (K / 2), elem0, q);
}


// Tensor-wise pass helpers (one block each; offline).
// The tensor's absmax: max over the rows' absmax values (order-free).
__global__ void __launch_bounds__(1024) amax_reduce_kernel(const float *__restrict__ row_amax, int64_t N,
                                                           float *__restrict__ out) {
    __shared__ float s_max[32];
    float m = 0.0f;
    for (int64_t i = threadIdx.x; i < N; i += blockDim.x) m = fmaxf(m, row_amax[i]);
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((threadIdx.x & 31) == 0) s_max[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        float t = 0.0f;
        for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) t = fmaxf(t, s_max[w]);
        *out = t;
    }
}

// The clip choice: for every grid point the rows' float64 errors summed in row
// order (thread i owns grid point i), then the first strict minimum.
__global__ void __launch_bounds__(64) err_argmin_kernel(const double *__restrict__ row_err, int64_t N,
                                                        int *__restrict__ alpha_out) {
    __shared__ double s_tot[64];
    const int i = threadIdx.x;
    if (i < kMseGrid) {
        double t = 0.0;
        for (int64_t n = 0; n < N; ++n) t += row_err[n * kMseGrid + i];
        s_tot[i] = t;
    }
    __syncthreads();
    if (i == 0) {
        int best = 0;
        for (int j = 1; j < kMseGrid; ++j)
            if (s_tot[j] < s_tot[best]) best = j;
        *alpha_out = best;
    }
}


}  // namespace convrot
