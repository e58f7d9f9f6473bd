// gemm_tcgen05.cuh -- integer GEMM with the dequantizing epilogue of the
// ConvRot linear, on sm_100a 5th-generation tensor cores.
//
//   acc[m,n] = sum_k qx[m,k] * qw[n,k]                      (tcgen05.mma kind::i8, int32 in TMEM)
//   Y[m,n]   = fp16( (float(acc) * s_x[m]) * s_w[n] + bias[n] )   (fused epilogue)
//
// Method: civarchive.com "SAM 3.1 Multiplex ConvRot" release, "Quantization
// recipe" (W8A8 / W4A4 operations, per-row scales; INT4 multiplication falls
// back to INT8 multiplication where the hardware has no INT4 path -- sm_100
// tcgen05 has no integer-4 kind, so W4A4 tiles are widened to int8 in shared
// memory before the int8 MMA).
//
// Structure: persistent, warp-specialized CTAs (one per SM), output tile
// 128 x BN, K step 128 bytes.
//   warp 0      TMA producer (one elected lane): A and B tiles -> smem ring
//   warp 1      TMEM allocator + MMA issuer (one lane): 4 x tcgen05.mma per K step
//   warps 2-9   epilogue: tcgen05.ld of the accumulator, scale, fp16, staged
//               in shared memory and written by TMA bulk stores
//   warps 10-13 (W4A4 only) nibble -> byte converters between a packed ring
//               and the MMA ring
// Two TMEM accumulators (2 x BN columns) let the epilogue of one tile overlap
// the main loop of the next.  No TMA multicast is used anywhere.
#pragma once

#include "device_utils.cuh"

namespace convrot {

// A4 / B4: the activation / weight operand arrives as packed int4 (two codes
// per byte) and is widened in shared memory; otherwise it is int8 loaded by TMA
// straight into the MMA ring.  Widened bytes hold 16 * code, so the
// accumulator carries a factor 16 per widened operand (ACC_SHIFT undoes it).
template <int BN_, bool A4_, bool B4_>
struct GemmCfg {
    static constexpr int BM = 128;
    static constexpr int BN = BN_;
    static constexpr int BK = 128;  // K elements per stage (= bytes of one int8 row segment)
    static constexpr bool A4 = A4_;
    static constexpr bool B4 = B4_;
    static constexpr bool W4 = A4 || B4;  // some operand is widened by converter warps
    static constexpr int ACC_SHIFT = (A4 ? 4 : 0) + (B4 ? 4 : 0);
    static constexpr int A_BYTES = BM * BK;
    static constexpr int B_BYTES = BN * BK;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    // MMA ring depth and packed ring depth
    static constexpr int STAGES = !W4 ? (BN == 256 ? 4 : 6) : A4 ? (BN == 256 ? 2 : 3) : (BN == 256 ? 3 : 4);
    static constexpr int PSTAGES = !W4 ? 0 : (BN == 256 ? 3 : 4);
    static constexpr int PA_BYTES = A4 ? A_BYTES / 2 : 0;
    static constexpr int PB_BYTES = B_BYTES / 2;
    static constexpr int PSTAGE_BYTES = PA_BYTES + PB_BYTES;
    static constexpr int CONV_ROWS = (A4 ? BM : 0) + BN;  // rows widened per stage
    // arrivals completing an MMA stage: the producer (A bytes by TMA) and/or the converters
    static constexpr int FULL_COUNT = !W4 ? 1 : (A4 ? 128 : 129);
    static constexpr int TMEM_COLS = 2 * BN;
    static constexpr int EPI_WARPS = 8;           // two per TMEM lane quarter, each half of the columns
    static constexpr int EPI_COLS = BN / 2;       // columns per epilogue warp
    static constexpr int CHUNK = 64;              // columns per output box (two 32-column TMEM loads)
    static constexpr int OUT_BOX_BYTES = 32 * CHUNK * 2;  // 32 rows x 64 fp16, 128-byte rows
    static constexpr int OUT_BYTES = EPI_WARPS * OUT_BOX_BYTES;  // one box per epilogue warp
    static constexpr int SCALE_BYTES = BN * 4 + BN * 2;        // the tile's w_scale (fp32) and bias (fp16)
    static constexpr int FIRST_CONV_WARP = 2 + EPI_WARPS;
    static constexpr int NUM_THREADS = 32 * (FIRST_CONV_WARP + (W4 ? 4 : 0));
    static constexpr int NUM_BARRIERS = 2 * STAGES + 2 * PSTAGES + 4 + 1 + 2;
    static constexpr int SMEM_BYTES = 1024 /* alignment slack */ + STAGES * STAGE_BYTES + PSTAGES * PSTAGE_BYTES +
                                      OUT_BYTES + SCALE_BYTES + NUM_BARRIERS * 8 + 16;
    static constexpr uint32_t IDESC = idesc_i8(BM, BN);
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
    static_assert(BN % 64 == 0 && BN >= 64 && BN <= 256, "tile width");
};

// Bounded wait used while draining: ignores the abort flag, still time-limited.
__device__ __forceinline__ void mbar_wait_drain(uint64_t *bar, uint32_t parity) {
    int dummy = 0;
    mbar_wait(bar, parity, &dummy);
}

// Sign-extends 16 packed int4 codes (8 bytes, low nibble = even element) to 16
// bytes holding 16 * code: shifting each nibble into the high half of its byte
// keeps the sign; the products are rescaled by 1/256 in the epilogue.
__device__ __forceinline__ uint4 widen_int4x16(uint2 p) {
    const uint32_t lo0 = (p.x << 4) & 0xf0f0f0f0u, hi0 = p.x & 0xf0f0f0f0u;
    const uint32_t lo1 = (p.y << 4) & 0xf0f0f0f0u, hi1 = p.y & 0xf0f0f0f0u;
    return make_uint4(__byte_perm(lo0, hi0, 0x5140), __byte_perm(lo0, hi0, 0x7362), __byte_perm(lo1, hi1, 0x5140),
                      __byte_perm(lo1, hi1, 0x7362));
}

// Dequantizes 8 accumulators of one row: fp16(fma(fp32(float(acc) * sx), sw[c], bias[c]))
// (the final multiply-add is one explicit fused operation, so it rounds once).
// sw_s / bias_s point at the tile's scales staged in shared memory.
template <int SHIFT>
__device__ __forceinline__ uint4 dequant8(const uint32_t *r, float sxm, const float *sw_s, const __half *bias_s,
                                          int32_t *acc_vals) {
    const float4 w0 = *reinterpret_cast<const float4 *>(sw_s);
    const float4 w1 = *reinterpret_cast<const float4 *>(sw_s + 4);
    const float wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
    const uint4 braw = *reinterpret_cast<const uint4 *>(bias_s);
    const uint32_t bw[4] = {braw.x, braw.y, braw.z, braw.w};
    uint32_t out[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int32_t a0 = static_cast<int32_t>(r[2 * i]) >> SHIFT;
        const int32_t a1 = static_cast<int32_t>(r[2 * i + 1]) >> SHIFT;
        acc_vals[2 * i] = a0;
        acc_vals[2 * i + 1] = a1;
        const float2 b = __half22float2(*reinterpret_cast<const __half2 *>(&bw[i]));
        float2 t = make_float2(__int2float_rn(a0), __int2float_rn(a1));
        t = __fmul2_rn(t, make_float2(sxm, sxm));
        t = __ffma2_rn(t, make_float2(wv[2 * i], wv[2 * i + 1]), b);
        const __half2 h = __floats2half2_rn(t.x, t.y);
        out[i] = *reinterpret_cast<const uint32_t *>(&h);
    }
    return make_uint4(out[0], out[1], out[2], out[3]);
}

template <class Cfg>
__global__ void __launch_bounds__(Cfg::NUM_THREADS, 1)
    gemm_i8_tcgen05_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                           const __grid_constant__ CUtensorMap tmY, int M, int N, int K, const float *__restrict__ sx,
                           const float *__restrict__ sw, const __half *__restrict__ bias,
                           int32_t *__restrict__ acc_out) {
    constexpr int BM = Cfg::BM, BN = Cfg::BN, STAGES = Cfg::STAGES, PSTAGES = Cfg::PSTAGES;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *ring = smem;                                          // STAGES x (A | B), int8, 128B-swizzled
    uint8_t *pring = ring + STAGES * Cfg::STAGE_BYTES;             // PSTAGES x (A4 | B4), packed, dense rows
    uint8_t *outbuf = pring + PSTAGES * Cfg::PSTAGE_BYTES;         // per epilogue warp: 32 x 64 fp16 box
    float *sw_s = reinterpret_cast<float *>(outbuf + Cfg::OUT_BYTES);          // [BN] tile w_scale
    __half *bias_s = reinterpret_cast<__half *>(sw_s + BN);                     // [BN] tile bias
    uint64_t *bars = reinterpret_cast<uint64_t *>(outbuf + Cfg::OUT_BYTES + Cfg::SCALE_BYTES);
    uint64_t *full = bars;                                         // MMA ring: operands ready
    uint64_t *empty = full + STAGES;                               // MMA ring: slot consumed
    uint64_t *pfull = empty + STAGES;                              // packed ring: TMA landed
    uint64_t *pempty = pfull + PSTAGES;                            // packed ring: slot converted
    uint64_t *tmem_full = pempty + PSTAGES;                        // [2] accumulator ready
    uint64_t *tmem_empty = tmem_full + 2;                          // [2] accumulator drained
    uint64_t *drain = tmem_empty + 2;                              // MMA completion at exit
    uint64_t *scale_ready = drain + 1;                             // tile scales staged in smem
    uint64_t *scale_free = scale_ready + 1;                        // tile scales no longer read
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(scale_free + 1);
    volatile int *abort = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int tiles_m = (M + BM - 1) / BM, tiles_n = (N + BN - 1) / BN;
    const int num_tiles = tiles_m * tiles_n;
    const int num_kb = K / Cfg::BK;

    if (threadIdx.x == 0) {
        for (int i = 0; i < STAGES; ++i) {
            mbar_init(&full[i], Cfg::FULL_COUNT);
            mbar_init(&empty[i], 1);
        }
        for (int i = 0; i < PSTAGES; ++i) {
            mbar_init(&pfull[i], 1);
            mbar_init(&pempty[i], 128);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&tmem_full[i], 1);
            mbar_init(&tmem_empty[i], 32 * Cfg::EPI_WARPS);
        }
        mbar_init(drain, 1);
        mbar_init(scale_ready, 32 * Cfg::EPI_WARPS);
        mbar_init(scale_free, 32 * Cfg::EPI_WARPS);
        *abort = 0;
        fence_mbarrier_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
        tma_prefetch_desc(&tmY);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, Cfg::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem_base = *tmem_slot;
    pdl_wait();  // the codes and scales may come from the previous kernel
    pdl_launch_dependents();

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
            for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
                const int tm = tile / tiles_n, tn = tile - tm * tiles_n;
                for (int kb = 0; kb < num_kb; ++kb) {
                    if (!Cfg::A4) {
                        if (!mbar_wait(&empty[s], ph ^ 1, abort)) {
                            ok = false;
                            break;
                        }
                        uint8_t *dst = ring + s * Cfg::STAGE_BYTES;
                        const uint32_t bytes = Cfg::B4 ? Cfg::A_BYTES : Cfg::STAGE_BYTES;
                        mbar_arrive_expect_tx(&full[s], bytes);
                        tma_load_2d(dst, &tmA, &full[s], kb * Cfg::BK, tm * BM);
                        if (!Cfg::B4) tma_load_2d(dst + Cfg::A_BYTES, &tmB, &full[s], kb * Cfg::BK, tn * BN);
                        filled[s] = true;
                        last_parity[s] = ph;
                        if (++s == STAGES) {
                            s = 0;
                            ph ^= 1;
                        }
                    }
                    if (Cfg::W4) {
                        if (!mbar_wait(&pempty[ps], pph ^ 1, abort)) {
                            ok = false;
                            break;
                        }
                        uint8_t *dst = pring + ps * Cfg::PSTAGE_BYTES;
                        mbar_arrive_expect_tx(&pfull[ps], Cfg::PSTAGE_BYTES);
                        if (Cfg::A4) tma_load_2d(dst, &tmA, &pfull[ps], kb * (Cfg::BK / 2), tm * BM);
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
            // (an MMA stage also waits for its converters when B is widened)
            for (int i = 0; i < STAGES; ++i)
                if (filled[i]) mbar_wait_drain(&full[i], last_parity[i]);
            for (int i = 0; i < PSTAGES; ++i)
                if (pfilled[i]) mbar_wait_drain(&pfull[i], plast_parity[i]);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            int s = 0;
            uint32_t ph = 0;
            bool ok = true;
            int local = 0;
            for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x, ++local) {
                const int acc = local & 1;
                const uint32_t acc_ph = (local >> 1) & 1;
                if (!mbar_wait(&tmem_empty[acc], acc_ph ^ 1, abort)) break;
                tc_fence_after_sync();
                const uint32_t d_tmem = tmem_base + acc * BN;
                for (int kb = 0; kb < num_kb; ++kb) {
                    if (!mbar_wait(&full[s], ph, abort)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after_sync();
                    const uint32_t a_addr = smem_addr(ring + s * Cfg::STAGE_BYTES);
                    const uint32_t b_addr = a_addr + Cfg::A_BYTES;
#pragma unroll
                    for (int kk = 0; kk < Cfg::BK / 32; ++kk) {
                        umma_i8(d_tmem, smem_desc_k_sw128(a_addr + 32 * kk), smem_desc_k_sw128(b_addr + 32 * kk),
                                Cfg::IDESC, (kb | kk) != 0);
                    }
                    umma_commit(&empty[s]);
                    if (++s == STAGES) {
                        s = 0;
                        ph ^= 1;
                    }
                }
                if (ok) umma_commit(&tmem_full[acc]);
            }
            umma_commit(drain);
            mbar_wait_drain(drain, 0);
        }
    } else if (warp < Cfg::FIRST_CONV_WARP) {
        // ------------------------------------------------------------ epilogue
        // Warp w reads TMEM lanes 32*(w%4) .. +31 (its hardware lane quarter)
        // and columns [half * BN/2, (half+1) * BN/2) of the accumulator.  The
        // tile's w_scale / bias are prefetched into registers one tile ahead
        // (one column per thread) and staged in shared memory at tile start.
        const int ew = warp - 2;  // 0..7
        const int q = warp & 3;
        const int half = ew >> 2;
        uint8_t *box = outbuf + ew * Cfg::OUT_BOX_BYTES;
        const int scol = ew * 32 + lane;  // the tile column this thread stages (valid if < BN)
        auto load_scales = [&](int t, float &wv, __half &bv) {
            wv = 0.0f;
            bv = __float2half_rn(0.0f);
            if (t < num_tiles && scol < BN) {
                const int col = (t - (t / tiles_n) * tiles_n) * BN + scol;
                if (col < N) {
                    wv = __ldg(sw + col);
                    if (bias != nullptr) bv = bias[col];
                }
            }
        };
        float next_w;
        __half next_b;
        load_scales(blockIdx.x, next_w, next_b);
        int local = 0;
        for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++local) {
            const int acc = local & 1;
            const uint32_t acc_ph = (local >> 1) & 1;
            if (!mbar_wait(&tmem_full[acc], acc_ph, abort)) break;
            tc_fence_after_sync();
            // every epilogue thread is done with the previous tile's scales
            if (local > 0 && !mbar_wait(scale_free, (local - 1) & 1, abort)) break;
            if (scol < BN) {
                sw_s[scol] = next_w;
                bias_s[scol] = next_b;
            }
            mbar_arrive(scale_ready);
            if (!mbar_wait(scale_ready, local & 1, abort)) break;
            load_scales(tile + gridDim.x, next_w, next_b);
            const int tm = tile / tiles_n, tn = tile - tm * tiles_n;
            const int row0 = tm * BM + q * 32;
            const int row = row0 + lane;
            const bool row_ok = row < M;
            const float sxm = row_ok ? sx[row] : 0.0f;
#pragma unroll 1
            for (int c = 0; c < Cfg::EPI_COLS / Cfg::CHUNK; ++c) {
                const int col_local = half * Cfg::EPI_COLS + c * Cfg::CHUNK;
                uint32_t r[2][32];
                __syncwarp();  // tcgen05.ld is warp-collective
                const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * BN + col_local;
                tmem_ld_32x32(taddr, r[0]);
                tmem_ld_32x32(taddr + 32, r[1]);
                tmem_ld_wait();
                if (c == Cfg::EPI_COLS / Cfg::CHUNK - 1) {
                    // every TMEM read of this tile by this thread is complete
                    tc_fence_before_sync();
                    mbar_arrive(&tmem_empty[acc]);
                }
                const int col0 = tn * BN + col_local;
                if (row0 >= M || col0 >= N) continue;  // whole box outside Y (warp-uniform)
                // the store issued from this box last time must have read it
                if (lane == 0) bulk_wait_group_read<0>();
                __syncwarp();
#pragma unroll
                for (int g = 0; g < 8; ++g) {  // 8 columns per 16-byte chunk
                    int32_t av[8];
                    uint4 v = make_uint4(0, 0, 0, 0);
                    if (row_ok && col0 + 8 * g < N) {
                        v = dequant8<Cfg::ACC_SHIFT>(r[g >> 2] + 8 * (g & 3), sxm, sw_s + col_local + 8 * g,
                                              bias_s + col_local + 8 * g, av);
                        if (acc_out != nullptr) {
                            int4 *dst = reinterpret_cast<int4 *>(acc_out + static_cast<int64_t>(row) * N + col0 + 8 * g);
                            dst[0] = make_int4(av[0], av[1], av[2], av[3]);
                            dst[1] = make_int4(av[4], av[5], av[6], av[7]);
                        }
                    }
                    // 128-byte rows, 16-byte chunk g stored at g ^ (row & 7) (128B swizzle)
                    *reinterpret_cast<uint4 *>(box + lane * 128 + ((g ^ (lane & 7)) << 4)) = v;
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    tma_store_2d(&tmY, box, col0, row0);
                    bulk_commit_group();
                }
            }
            mbar_arrive(scale_free);
        }
        if (lane == 0) bulk_wait_group_all();
    } else if (Cfg::W4) {
        // ------------------------------------------------------------ int4 -> int8 converters
        const int ct = threadIdx.x - 32 * Cfg::FIRST_CONV_WARP;  // 0..127
        int ps = 0, us = 0;
        uint32_t pph = 0, uph = 0;
        bool ok = true;
        for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
            for (int kb = 0; kb < num_kb; ++kb) {
                if (!mbar_wait(&pfull[ps], pph, abort) || !mbar_wait(&empty[us], uph ^ 1, abort)) {
                    ok = false;
                    break;
                }
                const uint8_t *src = pring + ps * Cfg::PSTAGE_BYTES;
                // widened rows: A (if packed) then B, in the MMA ring's layout
                uint8_t *dst = ring + us * Cfg::STAGE_BYTES + (Cfg::A4 ? 0 : Cfg::A_BYTES);
                constexpr int PIECES = Cfg::CONV_ROWS * (Cfg::BK / 16);  // 16 codes per piece
#pragma unroll 4
                for (int idx = ct; idx < PIECES; idx += 128) {
                    const int rr = idx >> 3, piece = idx & 7;  // widened row; 16-byte chunk in the row
                    const uint2 p = *reinterpret_cast<const uint2 *>(src + rr * 64 + piece * 8);
                    *reinterpret_cast<uint4 *>(dst + rr * 128 + ((piece ^ (rr & 7)) << 4)) = widen_int4x16(p);
                }
                fence_proxy_async_smem();
                mbar_arrive(&full[us]);
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

    __syncthreads();
    if (warp == 1) {
        tc_fence_after_sync();
        tmem_dealloc(tmem_base, Cfg::TMEM_COLS);
    }
}

}  // namespace convrot
