"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Bars (from the method's statement of the problem):
  * integer codes from the rotation kernels: within 1 code on at most 0.1 % of
    elements (the GPU rotates with an fp32 butterfly, the oracle rounds an fp64
    product), bit-exact where the butterfly is exact;
  * int32 accumulators and fp16 outputs of the GEMM given identical codes and
    scales: bit-exact;
  * the whole linear: relative Frobenius error <= 2e-3 against the oracle.
Inputs are seeded synthetic tensors from ``workloads`` with the shapes and
outlier statistics of the benchmarked configurations.
"""
import numpy as np
import pytest
import torch

import oracle
from rotated_bit_quantized_block_b200 import binding as cr
from rotated_bit_quantized_block_b200 import workloads as wl

pytestmark = pytest.mark.gpu

CODE_FRAC = 1e-3
REL_FRO = 2e-3


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host(t):
    torch.cuda.synchronize()
    return t.cpu().numpy()


def unpack(q, bits):
    return oracle.unpack_int4(q) if bits == 4 else q


def assert_codes_close(got, ref, frac=CODE_FRAC):
    d = np.abs(got.astype(np.int32) - ref.astype(np.int32))
    assert d.max(initial=0) <= 1, f"code difference {d.max()}"
    assert np.count_nonzero(d) <= frac * d.size, f"{np.count_nonzero(d)} of {d.size} codes differ"


def rel_fro(a, b):
    a = a.astype(np.float64)
    b = b.astype(np.float64)
    return np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30)


@pytest.fixture(autouse=True)
def _status_clean():
    yield
    cr.convrot_device_status()


def gpu_act(X, b, bits):
    Xq, s = cr.convrot_rotate_quant_act(dev(X), b, bits)
    return unpack(host(Xq), bits), host(s)


# ----------------------------------------------------------------------------- activations

ACT_CASES = [
    (64, 256, 64, 8), (64, 256, 64, 4),          # the tiny configuration
    (1, 128, 128, 8), (7, 384, 128, 4), (65, 1536, 128, 8), (300, 6144, 128, 4),
    (33, 1024, 256, 8), (130, 4096, 32, 4), (3, 32768, 256, 8), (129, 128, 1, 8),
]


@pytest.mark.parametrize("M,K,b,bits", ACT_CASES)
def test_act_rotate_quant_matches_oracle(M, K, b, bits):
    X = wl.activations(M, K, 0.01, 30.0, seed=M * 7 + K)
    q, s = gpu_act(X, b, bits)
    qr, sr = oracle.rotate_quant_act(X, b, bits)
    assert np.allclose(s, sr, rtol=1e-5, atol=0)
    assert_codes_close(q, qr)


@pytest.mark.parametrize("b", [1, 2, 4, 8, 16, 32, 64, 128, 256])
@pytest.mark.parametrize("bits", [8, 4])
def test_act_every_block_size(b, bits):
    X = wl.activations(37, 1024, 0.02, 20.0, seed=b + bits)
    q, s = gpu_act(X, b, bits)
    qr, sr = oracle.rotate_quant_act(X, b, bits)
    assert np.allclose(s, sr, rtol=1e-5, atol=0)
    assert_codes_close(q, qr)


@pytest.mark.parametrize("b", [1, 4, 16, 64, 256])
@pytest.mark.parametrize("bits", [8, 4])
def test_act_bit_exact_when_butterfly_is_exact(b, bits):
    """Small-integer inputs and b a power of 4 make every butterfly sum and the
    1/sqrt(b) factor exact in fp32, so codes and scales must match bit for bit."""
    rng = np.random.default_rng(b)
    X = rng.integers(-8, 9, size=(70, 1024)).astype(np.float16)
    X[5] = 0  # an all-zero token
    q, s = gpu_act(X, b, bits)
    qr, sr = oracle.rotate_quant_act(X, b, bits)
    assert np.array_equal(s.view(np.uint32), sr.view(np.uint32))
    assert np.array_equal(q, qr)
    assert s[5] == 0 and np.all(q[5] == 0)


@pytest.mark.parametrize("name,idx", [("vit_l_w8a8", 0), ("vit_l_w8a8", 3), ("vit_l_w4a4", 3), ("dit_w8a8", 0), ("dit_w8a8", 2)])
def test_act_full_size_sampled_rows(name, idx):
    w = wl.WORKLOADS[name]
    X, _, _ = wl.linear_inputs(w, idx)
    q, s = gpu_act(X, w.block, w.bits)
    rows = np.unique(np.concatenate([[0, 1, w.M - 1], np.linspace(0, w.M - 1, 61).astype(int)]))
    qr, sr = oracle.rotate_quant_act(X[rows], w.block, w.bits)
    assert np.allclose(s[rows], sr, rtol=1e-5, atol=0)
    assert_codes_close(q[rows], qr)


# ----------------------------------------------------------------------------- weights

def gpu_weight(W, b, bits, clip, dtype=torch.float16):
    Wt = dev(W) if dtype == torch.float16 else dev(W.astype(np.float32)).to(dtype)
    Wq, s = cr.convrot_quantize_weight(Wt, b, bits, clip)
    return unpack(host(Wq), bits), host(s)


@pytest.mark.parametrize("N,K,b,bits", [(256, 256, 64, 8), (24, 384, 128, 4), (72, 1024, 128, 8),
                                        (8, 6144, 256, 4), (100, 1536, 16, 8)])
def test_weight_absmax_matches_oracle(N, K, b, bits):
    W = wl.weight(N, K, 0.02, seed=N + K)
    q, s = gpu_weight(W, b, bits, cr.CLIP_ABSMAX)
    qr, sr, _ = oracle.quantize_weight(W, b, bits, oracle.CLIP_ABSMAX)
    assert np.allclose(s, sr, rtol=1e-5, atol=0)
    assert_codes_close(q, qr)


def _check_mse_rows(W, b, bits, q, s, dtype=oracle.DTYPE_F16, Wsrc=None):
    src = W if Wsrc is None else Wsrc
    qr, sr, aidx, errs = oracle.quantize_weight(src, b, bits, oracle.CLIP_MSE, dtype=dtype, want_errs=True)
    if dtype == oracle.DTYPE_F32:
        x64 = src.astype(np.float64)
    elif dtype == oracle.DTYPE_BF16:
        x64 = oracle.decode(src, oracle.DTYPE_BF16)
    else:
        x64 = src.astype(np.float64)
    _, w32 = oracle.rotate(x64, b)
    same = np.isclose(s, sr, rtol=1e-5, atol=0)
    # rows whose clip choice differs must be near-ties under the oracle's own error
    for n in np.nonzero(~same)[0]:
        e_gpu = oracle.quant_error(w32[n], s[n], bits)
        best = errs[n, aidx[n]]
        assert e_gpu <= best * (1 + 1e-5) + 1e-30, (n, e_gpu, best)
    assert np.count_nonzero(~same) <= max(1, 0.02 * len(s))
    assert_codes_close(q[same], qr[same])


@pytest.mark.parametrize("N,K,b,bits", [(256, 256, 64, 8), (64, 1024, 128, 4), (48, 4096, 128, 8),
                                        (16, 6144, 128, 4), (33, 512, 8, 4)])
def test_weight_mse_clip_matches_oracle(N, K, b, bits):
    W = wl.weight(N, K, 0.02, seed=3 * N + K)
    # heavy-tailed rows so that the clip search has real decisions to make
    W[::3] = (np.random.default_rng(N).standard_t(3, size=W[::3].shape) * 0.02).astype(np.float16)
    q, s = gpu_weight(W, b, bits, cr.CLIP_MSE)
    _check_mse_rows(W, b, bits, q, s)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_weight_source_dtypes(dtype):
    rng = np.random.default_rng(0)
    W32 = (rng.standard_normal((40, 512)) * 0.02).astype(np.float32)
    Wt = dev(W32).to(dtype)
    Wq, s = cr.convrot_quantize_weight(Wt, 128, 8, cr.CLIP_MSE)
    q, s = host(Wq), host(s)
    if dtype == torch.float32:
        _check_mse_rows(None, 128, 8, q, s, oracle.DTYPE_F32, Wsrc=W32)
    else:
        bits16 = Wt.view(torch.int16).cpu().numpy().view(np.uint16)
        _check_mse_rows(None, 128, 8, q, s, oracle.DTYPE_BF16, Wsrc=bits16)


# ----------------------------------------------------------------------------- GEMM (bit-exact)

def oracle_codes(M, N, K, b, bits, seed, full_range=False):
    if full_range:
        rng = np.random.default_rng(seed)
        lo, hi = (-127, 128) if bits == 8 else (-8, 8)
        qx = rng.integers(lo, hi, size=(M, K)).astype(np.int8)
        qw = rng.integers(lo, hi, size=(N, K)).astype(np.int8)
        sx = (rng.random(M) * 0.01 + 1e-4).astype(np.float32)
        sw = (rng.random(N) * 0.01 + 1e-4).astype(np.float32)
        return qx, sx, qw, sw
    X = wl.activations(M, K, 0.01, 30.0, seed)
    W = wl.weight(N, K, 0.02, seed + 1)
    qx, sx = oracle.rotate_quant_act(X, b, bits)
    qw, sw, _ = oracle.quantize_weight(W, b, bits, oracle.CLIP_MSE)
    return qx, sx, qw, sw


def run_gemm(qx, sx, qw, sw, bias, bits):
    if bits == 8:
        args = (dev(qx), dev(sx), dev(qw), dev(sw))
        fn = cr.convrot_gemm_w8a8
    else:
        args = (dev(oracle.pack_int4(qx)), dev(sx), dev(oracle.pack_int4(qw)), dev(sw))
        fn = cr.convrot_gemm_w4a4
    acc = torch.empty((qx.shape[0], qw.shape[0]), dtype=torch.int32, device="cuda")
    y = fn(*args, bias=None if bias is None else dev(bias), acc_out=acc)
    return host(y), host(acc)


GEMM_CASES = [
    (64, 256, 256), (1, 8, 128), (7, 24, 384), (130, 264, 640), (300, 1000, 1024),
    (256, 512, 4096), (129, 3072, 1024), (1000, 1536, 6144), (517, 4096, 256),
    # 256-wide tiles, ragged in M and N, one and several K steps
    (1300, 2000, 384), (2600, 1032, 128),
]


@pytest.mark.parametrize("bits", [8, 4])
@pytest.mark.parametrize("M,N,K", GEMM_CASES)
@pytest.mark.parametrize("with_bias", [False, True])
def test_gemm_bit_exact(M, N, K, bits, with_bias):
    qx, sx, qw, sw = oracle_codes(M, N, K, 128, bits, seed=M + N + K)
    bias = wl.bias(N, seed=N) if with_bias else None
    y, acc = run_gemm(qx, sx, qw, sw, bias, bits)
    yr, accr = oracle.gemm_dequant(qx, sx, qw, sw, bias, want_acc=True)
    assert np.array_equal(acc, accr)
    assert np.array_equal(y.view(np.uint16), yr.view(np.uint16))


@pytest.mark.parametrize("bits", [8, 4])
@pytest.mark.parametrize("M,N,K", [(200, 512, 2048), (64, 256, 32768)])
def test_gemm_bit_exact_full_code_range(M, N, K, bits):
    qx, sx, qw, sw = oracle_codes(M, N, K, 128, bits, seed=K, full_range=True)
    y, acc = run_gemm(qx, sx, qw, sw, None, bits)
    yr, accr = oracle.gemm_dequant(qx, sx, qw, sw, None, want_acc=True)
    assert np.array_equal(acc, accr)
    assert np.array_equal(y.view(np.uint16), yr.view(np.uint16))


@pytest.mark.parametrize("bits", [8, 4])
def test_gemm_full_size_sampled_rows(bits):
    """ViT-L fc1 shape at full M; the oracle recomputes a sample of rows."""
    M, N, K = 5184, 4096, 1024
    qx, sx, qw, sw = oracle_codes(M, N, K, 128, bits, seed=11)
    y, acc = run_gemm(qx, sx, qw, sw, None, bits)
    rows = np.unique(np.concatenate([[0, 127, 128, M - 1], np.linspace(0, M - 1, 40).astype(int)]))
    yr, accr = oracle.gemm_dequant(qx[rows], sx[rows], qw, sw, None, want_acc=True)
    assert np.array_equal(acc[rows], accr)
    assert np.array_equal(y[rows].view(np.uint16), yr.view(np.uint16))


# ----------------------------------------------------------------------------- whole linear

def linear_pair(w, idx, M=None, with_bias=False, sample=None):
    X, W, bias = wl.linear_inputs(w, idx, M=M, with_bias=with_bias)
    bits = w.bits_of(w.linears[idx])
    lin = cr.QuantizedLinear(dev(W), None if bias is None else dev(bias), w.block, bits, cr.CLIP_MSE)
    y = host(lin(dev(X)))
    qw, sw, _ = oracle.quantize_weight(W, w.block, bits, oracle.CLIP_MSE)
    rows = np.arange(X.shape[0]) if sample is None else sample
    yr = oracle.linear(X[rows], qw, sw, w.block, bits, bias)
    ref = X[rows].astype(np.float64) @ W.astype(np.float64).T
    if bias is not None:
        ref += bias.astype(np.float64)
    return y[rows], yr, ref


@pytest.mark.parametrize("bits", [8, 4])
def test_linear_tiny_config(bits):
    w = wl.WORKLOADS["tiny_w8a8"]
    w = wl.Workload(w.name, w.M, w.linears, bits, w.block, w.outlier_frac, w.outlier_factor, w.w_sigma, w.seed)
    y, yr, ref = linear_pair(w, 0, with_bias=True)
    assert rel_fro(y, yr) <= REL_FRO
    assert rel_fro(y, ref) <= (0.02 if bits == 8 else 0.3)


@pytest.mark.parametrize("name", ["vit_l_w8a8", "vit_l_w4a4"])
@pytest.mark.parametrize("idx", [0, 1, 2, 3])
def test_linear_vit_full_size_sampled(name, idx):
    w = wl.WORKLOADS[name]
    rows = np.unique(np.concatenate([[0, w.M - 1], np.linspace(0, w.M - 1, 48).astype(int)]))
    y, yr, ref = linear_pair(w, idx, sample=rows)
    assert rel_fro(y, yr) <= REL_FRO
    assert rel_fro(y, ref) <= (0.02 if w.bits == 8 else 0.3)


@pytest.mark.parametrize("idx", [0, 1, 2, 3])
def test_linear_mixed_widths_full_size_sampled(idx):
    """Per-layer code width (W8A8 attention, W4A4 MLP) at the ViT-L size."""
    w = wl.WORKLOADS["vit_l_mixed"]
    rows = np.unique(np.concatenate([[0, w.M - 1], np.linspace(0, w.M - 1, 32).astype(int)]))
    y, yr, ref = linear_pair(w, idx, sample=rows)
    assert rel_fro(y, yr) <= REL_FRO
    assert rel_fro(y, ref) <= (0.02 if w.bits_of(w.linears[idx]) == 8 else 0.3)


@pytest.mark.parametrize("idx", [0, 1, 2])
def test_linear_dit_full_size_sampled(idx):
    w = wl.WORKLOADS["dit_w8a8"]
    rows = np.linspace(0, w.M - 1, 24).astype(int)
    y, yr, _ = linear_pair(w, idx, sample=rows)
    assert rel_fro(y, yr) <= REL_FRO


@pytest.mark.parametrize("M", wl.MSWEEP_M)
def test_linear_msweep(M):
    w = wl.msweep(M)
    rows = None if M <= 128 else np.linspace(0, M - 1, 24).astype(int)
    y, yr, _ = linear_pair(w, 0, sample=rows)
    assert rel_fro(y, yr) <= REL_FRO


@pytest.mark.parametrize("bits", [8, 4])
def test_linear_two_stage_entry_points_equal_the_linear(bits):
    w = wl.WORKLOADS["vit_l_w8a8"]
    X, W, bias = wl.linear_inputs(w, 3, M=700, with_bias=True)
    Xd, Wd, bd = dev(X), dev(W), dev(bias)
    Wq, sw = cr.convrot_quantize_weight(Wd, w.block, bits, cr.CLIP_MSE)
    ws = torch.empty(cr.convrot_workspace_bytes(700, W.shape[1], bits), dtype=torch.uint8, device="cuda")
    fn = cr.convrot_linear_w8a8 if bits == 8 else cr.convrot_linear_w4a4
    y1 = host(fn(Xd, Wq, sw, w.block, bias=bd, workspace=ws))
    cr.convrot_linear_quant_act(Xd, w.block, bits, ws)
    y2 = host(cr.convrot_linear_gemm(ws, 700, W.shape[1], bits, Wq, sw, bias=bd))
    assert np.array_equal(y1.view(np.uint16), y2.view(np.uint16))


# (M, N, K): the feature-major split (M <= 128); the token-major stream-K plan
# (5184 x 1024 x 4096 with int4 weights; 2500 x 2000 x 8192, ragged M and N,
# with both widths); the whole-tile plan with the larger workspace
SPLIT_CASES = [(1, 4096, 4096), (16, 4096, 4096), (100, 1024, 4096), (700, 1024, 4096), (5184, 1024, 4096),
               (2500, 2000, 8192), (5184, 3072, 1024)]


@pytest.mark.parametrize("bits", [8, 4])
@pytest.mark.parametrize("M,N,K", SPLIT_CASES)
def test_linear_split_k_bit_exact(M, N, K, bits):
    """With the larger workspace the linear may split K across CTAs (feature-major
    K slices, or token-major stream-K shares whose boundary tiles are summed
    from two CTAs' partials); the int32 sums are exact, so the output equals the
    unsplit linear's and the oracle's GEMM of the same codes, bit for bit, on
    every call (the split state resets itself between calls)."""
    X = wl.activations(M, K, 0.01, 30.0, seed=M + 7)
    W = wl.weight(N, K, 0.02, seed=N + 7)
    bias = wl.bias(N, seed=3)
    Xd, bd = dev(X), dev(bias)
    Wq, sw = cr.convrot_quantize_weight(dev(W), 128, bits, cr.CLIP_ABSMAX)
    fn = cr.convrot_linear_w8a8 if bits == 8 else cr.convrot_linear_w4a4
    small = cr.convrot_workspace_bytes(M, K, bits)
    big = cr.convrot_linear_workspace_bytes(M, K, N, bits)
    assert big >= small + 2048
    ws_small = torch.empty(small, dtype=torch.uint8, device="cuda")
    ws_big = torch.empty(big, dtype=torch.uint8, device="cuda")
    y_ref = host(fn(Xd, Wq, sw, 128, bias=bd, workspace=ws_small))
    outs = [host(fn(Xd, Wq, sw, 128, bias=bd, workspace=ws_big)) for _ in range(3)]
    # the two-launch form on the large workspace takes the split plans even where
    # the linear runs fused
    for _ in range(2):
        cr.convrot_linear_quant_act(Xd, 128, bits, ws_big)
        outs.append(host(cr.convrot_linear_gemm(ws_big, M, K, bits, Wq, sw, bias=bd)))
    for y in outs:
        assert np.array_equal(y.view(np.uint16), y_ref.view(np.uint16))
    # the workspace starts with the activation codes (one per byte) and, at the
    # next 256-byte boundary, the per-token scales
    raw = host(ws_big)
    qx = raw[: M * K].view(np.int8).reshape(M, K)
    off = (M * K + 255) // 256 * 256
    sx = raw[off: off + 4 * M].view(np.float32)
    qw = unpack(host(Wq), bits)
    yr = oracle.gemm_dequant(qx, sx, qw, host(sw), bias)
    assert np.array_equal(outs[0].view(np.uint16), yr.view(np.uint16))


def pair_rows(M):
    """Rows to check on a 256-row-tile GEMM: both 128-row halves of the first
    and last tiles, every tile's first row, and the ragged tail."""
    rows = {0, 127, 128, 255, M - 1, M - 2}
    rows |= set(range(0, M, 256)) | set(range(128, M, 256))
    rows |= set(range(max(0, M - 140), M, 7))
    return np.array(sorted(r for r in rows if 0 <= r < M))


@pytest.mark.parametrize("M,N,K", [(2700, 4000, 1536), (4100, 2056, 2048)])
def test_gemm_pair_tiles_bit_exact_sampled(M, N, K):
    """Shapes the plan runs on CTA pairs (deep K, many 256 x 256 tiles), ragged in M and N."""
    qx, sx, qw, sw = oracle_codes(M, N, K, 128, 8, seed=M + K)
    bias = wl.bias(N, seed=5)
    y, acc = run_gemm(qx, sx, qw, sw, bias, 8)
    rows = pair_rows(M)
    yr, accr = oracle.gemm_dequant(qx[rows], sx[rows], qw, sw, bias, want_acc=True)
    assert np.array_equal(acc[rows], accr)
    assert np.array_equal(y[rows].view(np.uint16), yr.view(np.uint16))


@pytest.mark.parametrize("bits", [8, 4])
def test_linear_pair_tiles_bit_exact_sampled(bits):
    """The linear at a shape the plan runs on CTA pairs for int8 weights (and on
    single-CTA 256-wide tiles for int4): the output equals the oracle's GEMM of
    the workspace's codes on sampled rows."""
    M, N, K = 2700, 4000, 1536
    X = wl.activations(M, K, 0.01, 30.0, seed=17)
    W = wl.weight(N, K, 0.02, seed=18)
    bias = wl.bias(N, seed=19)
    Wq, sw = cr.convrot_quantize_weight(dev(W), 128, bits, cr.CLIP_ABSMAX)
    fn = cr.convrot_linear_w8a8 if bits == 8 else cr.convrot_linear_w4a4
    ws = torch.empty(cr.convrot_linear_workspace_bytes(M, K, N, bits), dtype=torch.uint8, device="cuda")
    y = host(fn(dev(X), Wq, sw, 128, bias=dev(bias), workspace=ws))
    raw = host(ws)
    qx = raw[: M * K].view(np.int8).reshape(M, K)
    off = (M * K + 255) // 256 * 256
    sx = raw[off: off + 4 * M].view(np.float32)
    rows = pair_rows(M)
    yr = oracle.gemm_dequant(qx[rows], sx[rows], unpack(host(Wq), bits), host(sw), bias)
    assert np.array_equal(y[rows].view(np.uint16), yr.view(np.uint16))


@pytest.mark.parametrize("bits", [8, 4])
@pytest.mark.parametrize("clip", [0, 1])
@pytest.mark.parametrize("N,K,b", [(300, 1024, 128), (64, 4096, 256), (7, 256, 64)])
def test_weight_tensorwise_matches_oracle(N, K, b, bits, clip):
    """One scale for the tensor: the clip choice is the oracle's (or a near-tie
    under the oracle's own errors), the scale agrees, the codes meet the code bar."""
    W = wl.weight(N, K, 0.02, seed=N + K + bits)
    W[N // 2, ::17] *= 40  # a few large weights, so that clipping matters
    Wq, sw = cr.convrot_quantize_weight_tensorwise(dev(W), b, bits, clip)
    sw = host(sw)
    codes = unpack(host(Wq), bits)
    rc, rs, ra, rerr = oracle.quantize_weight_tensorwise(W, b, bits, clip, want_errs=True)
    assert np.all(sw == sw[0])
    # the oracle's tensor absmax (rotation in float64, rounded to fp32)
    amax_o = float(np.max(np.abs(oracle.rotate(W.astype(np.float64), b)[1])))
    s_gpu = float(sw[0])
    # the GPU's scale is a grid point of (nearly) the same absmax ...
    cand = [i for i in (range(oracle.MSE_GRID) if clip == 1 else [0])
            if abs(float(oracle.scale(amax_o, oracle.alpha(i), bits)) - s_gpu) <= 2e-6 * s_gpu]
    assert cand, "the GPU's scale is not a grid point of the tensor's absmax"
    # ... whose total error is the oracle's minimum or a near-tie with it
    if clip == 1:
        assert min(rerr[i] for i in cand) <= rerr[ra] * (1 + 1e-6)
    if abs(s_gpu - float(rs[0])) <= 2e-6 * float(rs[0]):
        assert_codes_close(codes, rc)


@pytest.mark.parametrize("bits", [8, 4])
def test_linear_with_tensorwise_weights(bits):
    """The linears consume tensor-wise scales unchanged."""
    w = wl.WORKLOADS["vit_l_w8a8"]
    X, W, bias = wl.linear_inputs(w, 0, M=300, with_bias=True)
    Wq, sw = cr.convrot_quantize_weight_tensorwise(dev(W), 128, bits, cr.CLIP_MSE)
    fn = cr.convrot_linear_w8a8 if bits == 8 else cr.convrot_linear_w4a4
    y = host(fn(dev(X), Wq, sw, 128, bias=dev(bias)))
    qw, swr, _ = oracle.quantize_weight_tensorwise(W, 128, bits, oracle.CLIP_MSE)
    yr = oracle.linear(X, qw, swr, 128, bits, bias)
    assert rel_fro(y, yr) <= REL_FRO


@pytest.mark.parametrize("bits", [8, 4])
@pytest.mark.parametrize("M,N,K", [(1, 4096, 4096), (1, 2056, 8192), (1, 3072, 1024), (2, 2056, 8192),
                                   (1, 1000, 16384), (2, 1032, 2048), (6, 4096, 1024), (5, 1024, 4096),
                                   (1, 1024, 4096), (2, 1024, 1024), (1, 1024, 2048), (1, 4096, 16384),
                                   (2, 2056, 16384), (2, 1024, 4096),
                                   (3, 1000, 1024), (4, 2056, 640), (8, 3072, 128), (7, 520, 8192)])
def test_weight_streaming_gemm_bit_exact(M, N, K, bits):
    """For the fewest tokens the linear's GEMM streams the weights (dp4a, exact
    int32): bit-exact against the oracle's GEMM of the workspace's codes, for
    every block width (2, 4 and 8 features for 1-2 tokens, by N and K; 2 for
    3-4 tokens; 2 and 4 for 5-8, by N) and warp count (K from 128 to 16384)."""
    X = wl.activations(M, K, 0.01, 30.0, seed=M + K)
    W = wl.weight(N, K, 0.02, seed=N)
    bias = wl.bias(N, seed=4)
    Wq, sw = cr.convrot_quantize_weight(dev(W), 128, bits, cr.CLIP_MSE)
    fn = cr.convrot_linear_w8a8 if bits == 8 else cr.convrot_linear_w4a4
    ws = torch.empty(cr.convrot_linear_workspace_bytes(M, K, N, bits), dtype=torch.uint8, device="cuda")
    y = host(fn(dev(X), Wq, sw, 128, bias=dev(bias), workspace=ws))
    raw = host(ws)
    qx = raw[: M * K].view(np.int8).reshape(M, K)
    off = (M * K + 255) // 256 * 256
    sx = raw[off: off + 4 * M].view(np.float32)
    yr = oracle.gemm_dequant(qx, sx, unpack(host(Wq), bits), host(sw), bias)
    assert np.array_equal(y.view(np.uint16), yr.view(np.uint16))


@pytest.mark.parametrize("bits", [8, 4])
@pytest.mark.parametrize("M,N,K", [(1, 4096, 4096), (3, 2056, 8192), (64, 1024, 4096), (700, 1024, 1024),
                                   (2700, 4000, 1536)])
def test_linear_reads_weights_written_just_before(M, N, K, bits):
    """Both launches of the linear run with programmatic dependent launch.
    Weights quantized by the kernel launched right before the linear, on the
    same stream with no synchronization, must be the ones the GEMM reads: the
    output equals that of the same linear run after a device sync (every
    weight-streaming, feature-major split, token-major and CTA-pair plan)."""
    X = wl.activations(M, K, 0.01, 30.0, seed=M + 11)
    W = wl.weight(N, K, 0.02, seed=N + 11)
    bias = wl.bias(N, seed=6)
    Xd, Wd, bd = dev(X), dev(W), dev(bias)
    shape = cr.code_shape(N, K, bits)
    Wq = torch.zeros(shape, dtype=cr.code_dtype(bits), device="cuda")
    sw = torch.zeros(N, dtype=torch.float32, device="cuda")
    ws = torch.empty(cr.convrot_linear_workspace_bytes(M, K, N, bits), dtype=torch.uint8, device="cuda")
    fn = cr.convrot_linear_w8a8 if bits == 8 else cr.convrot_linear_w4a4
    torch.cuda.synchronize()
    cr.convrot_quantize_weight(Wd, 128, bits, cr.CLIP_ABSMAX, Wq=Wq, w_scale=sw)
    y_chained = host(fn(Xd, Wq, sw, 128, bias=bd, workspace=ws))
    torch.cuda.synchronize()
    y_after = host(fn(Xd, Wq, sw, 128, bias=bd, workspace=ws))
    assert np.array_equal(y_chained.view(np.uint16), y_after.view(np.uint16))
    # and the weights really changed: the zero codes give bias-only rows
    assert not np.array_equal(y_after.view(np.uint16), np.broadcast_to(bias.astype(np.float16), y_after.shape).view(np.uint16))


@pytest.mark.parametrize("M,N,K", [(5184, 3072, 1024), (700, 1000, 4096), (129, 264, 128)])
def test_w4a4_linear_widens_weights_once(M, N, K):
    """W4A4 over more than 128 tokens with the linear workspace: the activation
    launch widens the packed int4 weights once to int8 codes in the workspace
    (after the int8-weight plan's part) and the int8-weight GEMM multiplies
    them.  The widened codes equal the oracle's unpacking, and the output
    equals the linear that widens tiles in shared memory (minimum workspace)
    and the oracle's GEMM of the workspace's codes, bit for bit."""
    X = wl.activations(M, K, 0.01, 30.0, seed=M)
    W = wl.weight(N, K, 0.02, seed=N)
    bias = wl.bias(N, seed=K)
    Xd, bd = dev(X), dev(bias)
    Wq, sw = cr.convrot_quantize_weight(dev(W), 128, 4, cr.CLIP_MSE)
    big = cr.convrot_linear_workspace_bytes(M, K, N, 4)
    assert cr.convrot_linear_plan(M, K, N, 4, 128, big)["weights_widened"] == 1
    ws = torch.empty(big, dtype=torch.uint8, device="cuda")
    y = host(cr.convrot_linear_w4a4(Xd, Wq, sw, 128, bias=bd, workspace=ws))
    raw = host(ws)
    off = cr.convrot_linear_workspace_bytes(M, K, N, 8)
    wide = raw[off: off + N * K].view(np.int8).reshape(N, K)
    qw = oracle.unpack_int4(host(Wq))
    assert np.array_equal(wide, qw)
    ws_small = torch.empty(cr.convrot_workspace_bytes(M, K, 4), dtype=torch.uint8, device="cuda")
    y_small = host(cr.convrot_linear_w4a4(Xd, Wq, sw, 128, bias=bd, workspace=ws_small))
    assert np.array_equal(y.view(np.uint16), y_small.view(np.uint16))
    qx = raw[: M * K].view(np.int8).reshape(M, K)
    o = (M * K + 255) // 256 * 256
    sx = raw[o: o + 4 * M].view(np.float32)
    rows = np.unique(np.linspace(0, M - 1, 33).astype(int))
    yr = oracle.gemm_dequant(qx[rows], sx[rows], qw, host(sw), bias)
    assert np.array_equal(y[rows].view(np.uint16), yr.view(np.uint16))


@pytest.mark.parametrize("bits", [8, 4])
@pytest.mark.parametrize("M", [40, 300])
def test_degenerate_rows(M, bits):
    """The method's degenerate inputs, on the few-token (M = 40) and token-major
    (M = 300) GEMMs: an all-zero activation row (scale 0, codes 0, output =
    bias), a one-hot outlier (its block rotates to equal magnitudes), a constant
    block (rotates to a single nonzero), a row at the fp16 limit (+-65504), and
    all-zero / one-hot weight rows.  Codes and scales meet the oracle's bar,
    the GEMM of those codes is bit-exact, and the all-zero rows give exactly
    the bias."""
    K, N, b = 1024, 264, 128
    X = wl.activations(M, K, 0.01, 30.0, seed=M + bits).astype(np.float16)
    X[0] = 0.0
    X[1] = 0.0
    X[1, 5] = 1000.0
    X[2] = 0.0
    X[2, 128:256] = 3.0
    X[3] = np.where(np.arange(K) % 3 == 0, -65504.0, 65504.0).astype(np.float16)
    W = wl.weight(N, K, 0.02, seed=N + bits)
    W[0] = 0.0
    W[1] = 0.0
    W[1, 700] = 0.5
    bias = wl.bias(N, seed=bits)
    Wq, sw = cr.convrot_quantize_weight(dev(W), b, bits, cr.CLIP_MSE)
    _check_mse_rows(W, b, bits, unpack(host(Wq), bits), host(sw))
    assert host(sw)[0] == 0.0 and not np.any(unpack(host(Wq), bits)[0])
    ws = torch.empty(cr.convrot_linear_workspace_bytes(M, K, N, bits), dtype=torch.uint8, device="cuda")
    fn = cr.convrot_linear_w8a8 if bits == 8 else cr.convrot_linear_w4a4
    y = host(fn(dev(X), Wq, sw, b, bias=dev(bias), workspace=ws))
    raw = host(ws)
    qx = raw[: M * K].view(np.int8).reshape(M, K)
    off = (M * K + 255) // 256 * 256
    sx = raw[off: off + 4 * M].view(np.float32)
    qx_o, sx_o = oracle.rotate_quant_act(X, b, bits)
    assert np.allclose(sx, sx_o, rtol=1e-5, atol=0)
    assert sx[0] == 0.0 and not np.any(qx[0])
    assert_codes_close(qx, qx_o)
    yr = oracle.gemm_dequant(qx, sx, unpack(host(Wq), bits), host(sw), bias)
    assert np.array_equal(y.view(np.uint16), yr.view(np.uint16))
    assert np.array_equal(y[0].view(np.uint16), bias.astype(np.float16).view(np.uint16))
    # (the fp16-limit row may overflow Y to +-inf, as an fp16 linear would: the
    # bit-exact comparison above covers it)
    assert np.all(np.isfinite(y[:3].astype(np.float32)))
