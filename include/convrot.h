/*
 * convrot.h -- C ABI of the ConvRot-quantized linear layer for NVIDIA B200
 * (sm_100a).
 *
 * The method (source pages):
 *   - civarchive.com, "SAM 3.1 Multiplex ConvRot" release, section
 *     "Quantization recipe": an offline converter upcasts each eligible
 *     linear weight to FP32, applies a block-Hadamard ConvRot transform,
 *     chooses an MSE-optimized clipping scale and stores per-row scales;
 *     the runtime performs W8A8 (or W4A4) operations with online, dynamic
 *     per-operation activation quantization.  Section "Downloads": INT4
 *     multiplication may fall back to INT8 multiplication where the hardware
 *     has no INT4 path (sm_100 tcgen05 has none: int4 codes are widened to
 *     int8 in shared memory ahead of the int8 MMA).
 *   - trellis3d.app, "TRELLIS.2 INT8 ConvRot in ComfyUI", section "What
 *     ConvRot changes": a grouped, normalized Hadamard rotation precedes the
 *     per-row weight quantization and the matching rotation is applied to the
 *     activations at runtime, spreading channel outliers over the grid.
 *
 * Notation.  X is M x K (tokens x in-features), W is N x K (out x in, as in
 * nn.Linear), both row-major.  b ("block") is the Hadamard block size.
 * R = blockdiag(H_b/sqrt(b), ...) with H_b the Sylvester Hadamard matrix.
 *   X~ = X.R,  s_x[m] = max_k |X~[m,k]| / qmax,       qx = rne(X~ * (1/s_x))
 *   W~ = W.R,  s_w[n] = alpha_n max_k |W~[n,k]| / qmax, qw = clamp(rne(W~ * (1/s_w)))
 *   acc[m,n] = sum_k qx[m,k] qw[n,k]             (exact int32)
 *   Y[m,n]   = fp16( fma( fp32(float(acc) * s_x[m]), s_w[n], bias[n] ) )
 * qmax = 127 (int8, codes in [-127, 127]) or 7 (int4, codes in [-8, 7]).
 * Rotation and scales are fp32; every rounding is round-to-nearest-even.
 *
 * Int4 storage: two codes per byte along K, element 2j in bits 0..3 and
 * element 2j+1 in bits 4..7, 4-bit two's complement.  A packed row of K
 * codes takes K/2 bytes.
 *
 * Conventions for every call below:
 *   - All array pointers are DEVICE pointers owned by the caller; the library
 *     keeps no reference after the call returns.  Arrays are dense row-major.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and nothing synchronizes with the host, except
 *     convrot_device_status().  Calls are safe to capture in a CUDA graph.
 *   - Nothing is allocated; scratch space is the caller's `workspace`.
 *   - Argument checks run before any launch.  On failure the call returns a
 *     status other than CONVROT_OK, launches nothing and leaves every output
 *     untouched; convrot_last_error() then describes the failure.
 *   - Shape limits: 128 <= K <= 32768 with K % 128 == 0; b a power of two in
 *     [1, 256] with K % b == 0; 0 <= M, N < 2^31 (M == 0 or N == 0 is a no-op);
 *     the GEMM entry points need N % 8 == 0.  X, Y, Xq, Wq, workspace,
 *     w_scale, bias and acc_out must be 16-byte aligned, x_scale 4-byte aligned.
 *   - Non-finite inputs (inf / NaN in X or W) give unspecified codes.
 *   - Kernels never trap: a device-side wait that exceeds its time limit
 *     abandons the launch and records CONVROT_ERR_TIMEOUT, which
 *     convrot_device_status() reports.
 */
#ifndef CONVROT_H
#define CONVROT_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    CONVROT_OK = 0,
    CONVROT_ERR_INVALID_ARG = 1, /* null pointer, bad enum, shape outside the limits */
    CONVROT_ERR_UNSUPPORTED = 2, /* valid request this build does not handle (e.g. device not sm_100) */
    CONVROT_ERR_ALIGNMENT = 3,   /* a pointer violates the alignment rules above */
    CONVROT_ERR_CUDA = 4,        /* a CUDA runtime/driver call failed (launch, attribute, tensor map) */
    CONVROT_ERR_TIMEOUT = 5,     /* a kernel abandoned a wait after its time limit */
    CONVROT_ERR_WORKSPACE = 6    /* workspace null or smaller than convrot_workspace_bytes() */
} convrot_status_t;

enum { CONVROT_CLIP_ABSMAX = 0, CONVROT_CLIP_MSE = 1 };
enum { CONVROT_DTYPE_F16 = 0, CONVROT_DTYPE_BF16 = 1, CONVROT_DTYPE_F32 = 2 };

/*
 * Offline weight conversion -- "Quantization recipe" steps 1-4 (civarchive
 * ConvRot release page): upcast W to fp32, rotate each row by blockdiag(R_b),
 * pick the per-row clip factor, store per-row scales and codes.
 *   W        [N x K] source weight, element type w_dtype (fp16, bf16 or fp32).
 *   clip_mode CONVROT_CLIP_ABSMAX: alpha = 1.  CONVROT_CLIP_MSE: alpha is the
 *            first minimiser, scanning alpha = 1.00, 0.99, ..., 0.50, of the
 *            float64 squared error sum_k (W~[n,k] - s*q)^2.
 *   bits     8 -> Wq is int8 [N x K]; 4 -> Wq is packed int4 uint8 [N x K/2].
 *   w_scale  [N] fp32 output, s_w[n] (0 for an all-zero row, whose codes are 0).
 */
convrot_status_t convrot_quantize_weight(const void *W, int w_dtype, int64_t N, int64_t K, int block,
                                         int bits, int clip_mode, void *Wq, float *w_scale,
                                         void *stream);

/*
 * Tensor-wise variant of the offline converter (salahadawi.com "Explanation
 * of INT8 ConvRot", "8-bit INT type models" table: Tensor-wise scaling, one
 * scale per weight tensor; civarchive.com release, downloads table: an
 * int8_tensorwise ConvRot file).  Same rotation and code rule as
 * convrot_quantize_weight; the scale is shared by all rows:
 * s = fp32(fp32(alpha * max over the tensor of |W~|) / qmax), alpha = 1 in
 * CONVROT_CLIP_ABSMAX mode or, in CONVROT_CLIP_MSE mode, the grid point with
 * the smallest total squared error of the tensor (the rows' float64 errors
 * summed in row order; first strict minimum from alpha = 1).  w_scale[N]
 * receives s for every row, so the linears and GEMMs take the result as is.
 *   workspace  at least convrot_tensorwise_workspace_bytes(N, clip_mode) bytes
 *              of device memory, 16-byte aligned; its contents on return are
 *              unspecified.
 * Four launches on `stream` (row absmax, tensor absmax, [row errors, clip
 * choice,] quantization); other arguments and errors as convrot_quantize_weight.
 */
size_t convrot_tensorwise_workspace_bytes(int64_t N, int clip_mode);
convrot_status_t convrot_quantize_weight_tensorwise(const void *W, int w_dtype, int64_t N, int64_t K, int block,
                                                    int bits, int clip_mode, void *Wq, float *w_scale,
                                                    void *workspace, size_t workspace_bytes, void *stream);

/*
 * Online activation quantization -- "online 8-bit activation quantization",
 * "dynamic per-operation" (civarchive ConvRot release, "Quantization recipe"),
 * with the matching rotation of "What ConvRot changes" (trellis3d.app):
 * X~ = X.R in fp32, per-token absmax scale, round to nearest.
 *   X        [M x K] fp16.
 *   bits     8 -> Xq is int8 [M x K]; 4 -> Xq is packed int4 uint8 [M x K/2].
 *   x_scale  [M] fp32 output, s_x[m] (0 for an all-zero row).
 */
convrot_status_t convrot_rotate_quant_act(const void *X, int64_t M, int64_t K, int block, int bits,
                                          void *Xq, float *x_scale, void *stream);

/*
 * Bytes of scratch the linear entry points need for M tokens of K features:
 * the activation codes, one byte per code for both widths (M*K; the W4A4
 * linear keeps its transient int4 activation codes unpacked so that only the
 * stored weights are widened inside the GEMM), and the M per-token scales, each
 * rounded up to 256 bytes.  Returns 0 for invalid arguments.
 */
size_t convrot_workspace_bytes(int64_t M, int64_t K, int bits);

/*
 * Workspace size that also lets the linear balance its GEMM across SMs.  For
 * more than 128 tokens, where the 128 x 256 output tiles fill some but not all
 * SMs in their last round (and CTA pairs are not used), the GEMM runs
 * stream-K: every SM takes an equal share of all tiles' K steps, and a tile
 * shared by two SMs is summed from one int32 partial tile (128 x 256) that the
 * first of them stores in a slot of this workspace.  (With at most 128 tokens
 * the GEMM splits K over clusters of CTAs that add their partials through
 * distributed shared memory, which needs no workspace.)
 * Size: convrot_workspace_bytes(M, K, bits) plus 2 KB of counters plus, where
 * stream-K applies, (SMs + 1) partial-tile slots of 128 KB.  For W4A4 over
 * more than 128 tokens it also holds the weights widened to int8 codes (N*K
 * bytes, after the slots of the int8-weight plan): see convrot_linear_w4a4.
 * The activation half of the linear zeroes the counters; the GEMM half leaves
 * them zeroed again (the partial-tile slots are written before they are read).
 * Depends on the current device's SM count.  Returns 0 for invalid arguments.
 */
size_t convrot_linear_workspace_bytes(int64_t M, int64_t K, int64_t N, int bits);

/*
 * W8A8 ConvRot linear (civarchive ConvRot release, "The INT8 file uses W8A8
 * operations"): Y = dequant( int8(rotate(X)) . Wq^T ) + bias.
 *   X         [M x K] fp16 activations (not yet rotated).
 *   Wq        [N x K] int8 codes from convrot_quantize_weight(bits = 8), same block.
 *   w_scale   [N] fp32 per-output-row scales.
 *   bias      [N] fp16 or NULL.
 *   Y         [M x N] fp16 output.
 *   workspace at least convrot_workspace_bytes(M, K, 8) bytes of device memory
 *             (convrot_linear_workspace_bytes(M, K, N, 8) enables stream-K); on
 *             return it holds the activation codes (int8 M x K) followed, at the
 *             next 256-byte boundary, by the scales.
 */
convrot_status_t convrot_linear_w8a8(const void *X, int64_t M, int64_t K, const int8_t *Wq,
                                     const float *w_scale, int64_t N, const void *bias, int block, void *Y,
                                     void *workspace, size_t workspace_bytes, void *stream);

/*
 * W4A4 ConvRot linear (civarchive ConvRot release, "The INT4 file similarly
 * uses W4A4 operations"; INT8 multiplication on hardware without INT4 MMA).
 * As convrot_linear_w8a8 with Wq the packed int4 codes [N x K/2] from
 * convrot_quantize_weight(bits = 4) and workspace >=
 * convrot_workspace_bytes(M, K, 4).  With more than 128 tokens and a workspace
 * of convrot_linear_workspace_bytes(M, K, N, 4), the activation launch also
 * widens the packed weights once to int8 codes in the workspace and the GEMM
 * multiplies those (the same integers, so the same output); otherwise the GEMM
 * widens the packed tiles in shared memory.
 */
convrot_status_t convrot_linear_w4a4(const void *X, int64_t M, int64_t K, const uint8_t *Wq,
                                     const float *w_scale, int64_t N, const void *bias, int block, void *Y,
                                     void *workspace, size_t workspace_bytes, void *stream);

/*
 * How convrot_linear_w8a8 / convrot_linear_w4a4 would run a call of these
 * sizes with a workspace of workspace_bytes on the current device (no launch):
 *   launches   kernels per call (the activation kernel, then the GEMM).
 *   gemm_kind  0: token-major tensor-core tiles (128 tokens x tile_n
 *              features); 1: feature-major tiles (128 features x tile_n
 *              tokens); 2: the weight-streaming kernel (dp4a).
 *   cta_pair / stream_k / k_splits: CTA pairs (cta_group::2), stream-K shares,
 *              K slices of the feature-major split (a cluster of that many
 *              CTAs per tile; fewer at launch if the GPCs cannot hold all the
 *              clusters at once).
 *   fused_available  1 if convrot_linear_w8a8_fused accepts the call (W8A8).
 *   weights_widened  1 if the W4A4 linear widens its weights to int8 codes in
 *              the workspace and runs the int8-weight GEMM (the fields above
 *              then describe that GEMM).
 */
typedef struct {
    int launches;
    int gemm_kind;
    int tile_n;
    int cta_pair;
    int stream_k;
    int k_splits;
    int fused_available;
    int weights_widened;
} convrot_linear_plan_t;
convrot_status_t convrot_linear_plan(int64_t M, int64_t K, int64_t N, int bits, int block, size_t workspace_bytes,
                                     convrot_linear_plan_t *plan);

/*
 * W8A8 ConvRot linear with the rotation fused into the GEMM kernel
 * (civarchive ConvRot release, "Future improvements": fusion of the steps).
 * Same arguments and results as convrot_linear_w8a8 -- the codes, scales and
 * Y are bit-identical -- but the GEMM's CTAs carry eight activation warps that
 * rotate and quantize units of tokens into the workspace beside the
 * tensor-core main loop; the producer loads a 128-token panel's codes once
 * every unit touching it has been counted into the panel's counter.  A tiny
 * kernel zeroing the counters precedes it.  On B200 the two-launch linear
 * measured faster at every shape tried (the activation kernel then has the
 * whole GPU), so convrot_linear_w8a8 does not use this path.
 *   Supported: more than 128 tokens, block 128, K <= 2048, at most 512
 *   panels of 128 tokens; otherwise CONVROT_ERR_UNSUPPORTED.
 *   workspace  at least convrot_workspace_bytes(M, K, 8) + 2048 bytes (the
 *              panel counters follow the scales);
 *              convrot_linear_workspace_bytes(M, K, N, 8) always suffices.
 * The CTAs wait for one another (bounded): every CTA must be co-resident, which
 * the grid (at most one CTA or CTA pair per SM) ensures when no other kernel
 * holds SMs for the whole run of this one.
 */
convrot_status_t convrot_linear_w8a8_fused(const void *X, int64_t M, int64_t K, const int8_t *Wq,
                                           const float *w_scale, int64_t N, const void *bias, int block, void *Y,
                                           void *workspace, size_t workspace_bytes, void *stream);

/*
 * The two launches of convrot_linear_w8a8 / convrot_linear_w4a4, callable
 * separately (same arguments, same workspace layout): first rotate and
 * quantize X into the workspace, then run the integer GEMM + dequant from it.
 * The workspace must not be reused by another linear in between.
 * convrot_linear_quant_act zeroes the 2 KB of counters after the scales where
 * the workspace holds them.
 */
convrot_status_t convrot_linear_quant_act(const void *X, int64_t M, int64_t K, int block, int bits,
                                          void *workspace, size_t workspace_bytes, void *stream);
convrot_status_t convrot_linear_gemm(const void *workspace, size_t workspace_bytes, int64_t M, int64_t K, int bits,
                                     const void *Wq, const float *w_scale, int64_t N, const void *bias, void *Y,
                                     void *stream);

/*
 * The integer GEMM with its dequantizing epilogue alone, on given codes (the
 * last two steps of the linear): Y[m,n] = fp16(fma(fp32(float(acc) *
 * x_scale[m]), w_scale[n], bias[n])) -- one rounding for the product with
 * x_scale, one for the fused multiply-add -- with acc = sum_k Xq[m,k] Wq[n,k].
 *   Xq [M x K] int8, Wq [N x K] int8 (w8a8); packed int4 [M x K/2], [N x K/2] (w4a4).
 *   acc_out  [M x N] int32 or NULL: receives acc (for exact-integer testing).
 */
convrot_status_t convrot_gemm_w8a8(const int8_t *Xq, const float *x_scale, int64_t M, const int8_t *Wq,
                                   const float *w_scale, int64_t N, int64_t K, const void *bias, void *Y,
                                   int32_t *acc_out, void *stream);
convrot_status_t convrot_gemm_w4a4(const uint8_t *Xq, const float *x_scale, int64_t M, const uint8_t *Wq,
                                   const float *w_scale, int64_t N, int64_t K, const void *bias, void *Y,
                                   int32_t *acc_out, void *stream);

/*
 * W8A8 ConvRot linear that allocates nothing and takes no workspace.  The
 * source pages have no counterpart: this exists for callers that cannot
 * allocate device memory (a plugin whose host framework owns the GPU's memory
 * and offers no allocator, or a path where an allocation is not allowed).
 * Arguments and results are those of convrot_linear_w8a8 without
 * workspace / workspace_bytes.
 *   - Scratch (activation codes and scales) lives in one 16 MiB array built
 *     into the library; every GPU that loads the library holds it until the
 *     process exits.  Calls needing more (M*K + 4*M bytes, each rounded up to
 *     256) return CONVROT_ERR_WORKSPACE without launching.
 *   - The first call on a device looks up the array's device address with
 *     that device current; make that first call before any stream capture.
 *   - All calls on a device share the array and leave the last call's codes in
 *     it; nothing needs to start at zero.  Calls whose kernels overlap on the
 *     GPU (different streams, no ordering between them) race on it.
 */
convrot_status_t convrot_linear_w8a8_noalloc(const void *X, int64_t M, int64_t K, const int8_t *Wq,
                                             const float *w_scale, int64_t N, const void *bias, int block,
                                             void *Y, void *stream);

/*
 * Synchronizes `stream`, then returns and clears the sticky device-side
 * status of the current device: CONVROT_OK, CONVROT_ERR_TIMEOUT if a kernel
 * abandoned a wait since the last query, or CONVROT_ERR_CUDA if the stream
 * reported an error.
 */
convrot_status_t convrot_device_status(void *stream);

/*
 * Diagnostics (no counterpart on the source pages): exercises the failure
 * path of the kernels' bounded device-side waits without a fault.  Launches one
 * tiny kernel that waits, through the same wait routines the linear's kernels
 * use, on something that never completes -- kind 0: an mbarrier phase that no
 * thread completes; kind 1: a fused-prologue flag word that no CTA publishes --
 * with a limit of limit_ns nanoseconds (1 us .. 1 s).  The wait gives up, the
 * kernel records CONVROT_ERR_TIMEOUT in the device status word (reported and
 * cleared by the next convrot_device_status) and returns; nothing traps and the
 * context stays usable.
 *   result  16 bytes of device memory, 16-byte aligned: result[0] = 1 if the
 *           wait succeeded (0 expected), result[1] = 1 if it abandoned the
 *           wait; bytes 8..15 serve as the flag word of kind 1.
 */
convrot_status_t convrot_test_abandoned_wait(int kind, uint64_t limit_ns, int32_t *result, void *stream);

/* Static description of a status code (never NULL). */
const char *convrot_status_string(convrot_status_t status);

/* Detail of the most recent failing call on this host thread ("" if none). */
const char *convrot_last_error(void);

/* Library version, major * 10000 + minor * 100 + patch. */
int convrot_version(void);

#ifdef __cplusplus
}
#endif

#endif /* CONVROT_H */
