"""Pins of the CPU oracle to things other than itself.

Each test ties one oracle function to a value the pages print, a closed form,
a textbook/library routine, an invariant or a brute force on tiny inputs, so
that a plausible slip in the oracle (a dropped term, a wrong sign or index, a
transposed operand) fails at least one of them.  No GPU is needed.
"""
import json
import math
import os

import numpy as np
import pytest
import scipy.linalg
import torch

import oracle
from rotated_bit_quantized_block_b200 import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
BLOCKS = [1, 2, 4, 8, 16, 32, 64, 128, 256]


def _popcount(v):
    return bin(v).count("1")


# ---------------------------------------------------------------- number formats

def test_f16_decode_matches_numpy_for_every_bit_pattern():
    bits = np.arange(65536, dtype=np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = oracle.decode(bits, oracle.DTYPE_F16)
    finite = np.isfinite(ref)
    assert np.array_equal(got[finite], ref[finite])
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    assert np.array_equal(got[np.isinf(ref)], ref[np.isinf(ref)])


def test_bf16_and_f32_decode_match_torch():
    g = torch.Generator().manual_seed(5)
    x = torch.randn(4096, generator=g) * 100
    bf = x.to(torch.bfloat16)
    got = oracle.decode(bf.view(torch.int16).numpy().view(np.uint16), oracle.DTYPE_BF16)
    assert np.array_equal(got, bf.to(torch.float64).numpy())
    x32 = x.numpy().astype(np.float32)
    assert np.array_equal(oracle.decode(x32, oracle.DTYPE_F32), x32.astype(np.float64))


def test_f32_to_f16_rounding_matches_numpy():
    rng = np.random.default_rng(0)
    vals = np.concatenate([
        rng.standard_normal(200000).astype(np.float32) * np.float32(3000.0),
        rng.standard_normal(50000).astype(np.float32) * np.float32(1e-5),   # subnormal range
        np.array([0.0, -0.0, 65504.0, 65519.996, 65520.0, 70000.0, -65520.0, 6.1035156e-05,
                  5.9604645e-08, 2.9802322e-08, 2.9802326e-08, 1e-10, np.inf, -np.inf],
                 dtype=np.float32),
    ])
    # exact ties between fp16 neighbours (half-way points) in several binades
    h = np.arange(0x0400, 0x7bff, 97, dtype=np.uint16).view(np.float16).astype(np.float32)
    h_next = (np.arange(0x0400, 0x7bff, 97, dtype=np.uint16) + 1).view(np.float16).astype(np.float32)
    vals = np.concatenate([vals, (h + h_next) / 2, -(h + h_next) / 2])
    got = oracle.f32_to_f16_bits(vals)
    with np.errstate(over="ignore"):
        ref = vals.astype(np.float16).view(np.uint16)
    assert np.array_equal(got, ref)


# ---------------------------------------------------------------- the rotation

@pytest.mark.parametrize("b", BLOCKS)
def test_hadamard_is_orthogonal_and_symmetric(b):
    R = oracle.hadamard(b)
    assert np.max(np.abs(R @ R.T - np.eye(b))) < 1e-12
    assert np.array_equal(R, R.T)


@pytest.mark.parametrize("b", BLOCKS)
def test_hadamard_matches_sylvester_closed_form_and_scipy(b):
    R = oracle.hadamard(b)
    closed = np.array([[(-1) ** _popcount(i & j) for j in range(b)] for i in range(b)], dtype=np.float64)
    assert np.array_equal(np.round(R * math.sqrt(b)), closed)
    assert np.max(np.abs(R - scipy.linalg.hadamard(b) / math.sqrt(b))) < 1e-15


@pytest.mark.parametrize("b", [4, 64, 128])
def test_rotation_is_blockdiag_product(b):
    rng = np.random.default_rng(b)
    K = 4 * b if b < 128 else 512
    X = rng.standard_normal((5, K))
    Rfull = scipy.linalg.block_diag(*([scipy.linalg.hadamard(b) / math.sqrt(b)] * (K // b)))
    r64, r32 = oracle.rotate(X, b)
    ref = X @ Rfull
    assert np.max(np.abs(r64 - ref)) < 1e-12 * np.max(np.abs(ref))
    assert np.array_equal(r32, r64.astype(np.float32))


@pytest.mark.parametrize("b", [1, 16, 64, 128, 256])
def test_product_is_rotation_invariant(b):
    """(XR)(WR)^T == X W^T: the matching rotation of weights and activations."""
    rng = np.random.default_rng(7 + b)
    K = 512
    X = rng.standard_normal((6, K))
    W = rng.standard_normal((9, K))
    xr, _ = oracle.rotate(X, b)
    wr, _ = oracle.rotate(W, b)
    ref = X @ W.T
    assert np.max(np.abs(xr @ wr.T - ref)) < 1e-12 * np.max(np.abs(ref))


@pytest.mark.parametrize("b", [2, 8, 64, 128])
def test_one_hot_outlier_is_spread_evenly(b):
    """An outlier A at one channel becomes b entries of magnitude exactly A/sqrt(b)."""
    K = 2 * b
    for p in (0, b - 1, b // 2 + (b > 2)):
        X = np.zeros((1, K))
        X[0, b + p] = 30.0
        r64, _ = oracle.rotate(X, b)
        assert np.all(r64[0, :b] == 0)
        assert np.allclose(np.abs(r64[0, b:]), 30.0 / math.sqrt(b), rtol=0, atol=1e-13)
        signs = np.sign(r64[0, b:])
        assert np.array_equal(signs, np.array([(-1) ** _popcount(i & p) for i in range(b)]))


@pytest.mark.parametrize("b", [2, 16, 128])
def test_constant_block_maps_to_first_coordinate(b):
    X = np.full((1, b), 0.75)
    r64, _ = oracle.rotate(X, b)
    assert abs(r64[0, 0] - 0.75 * math.sqrt(b)) < 1e-13
    assert np.max(np.abs(r64[0, 1:])) < 1e-13


def test_golden_worked_rotate_quant_examples():
    with open(os.path.join(GOLDEN, "worked_examples.json")) as f:
        gold = json.load(f)
    for ex in gold["rotate_quant"]:
        x = np.array([ex["x"]], dtype=np.float16)
        b = ex["block"]
        r64, _ = oracle.rotate(x.astype(np.float64), b)
        if "x_rot" in ex:
            assert np.allclose(r64[0], ex["x_rot"], rtol=0, atol=1e-12), ex["name"]
        else:
            assert np.allclose(r64[0], np.array(ex["x_rot_over_amax_sign"]) * ex["amax"], atol=1e-12)
        for bits, key in ((8, "int8"), (4, "int4")):
            codes, scales = oracle.rotate_quant_act(x, b, bits)
            assert codes[0].tolist() == ex[key]["codes"], (ex["name"], key)
            amax = ex[key].get("amax", ex.get("amax"))
            assert scales[0] == np.float32(np.float32(amax) / np.float32(ex[key]["qmax"]))


def test_golden_worked_gemm_example():
    with open(os.path.join(GOLDEN, "worked_examples.json")) as f:
        g = json.load(f)["gemm"]
    y, acc = oracle.gemm_dequant(np.array(g["qx"]), np.array(g["sx"]), np.array(g["qw"]), np.array(g["sw"]),
                                 np.array(g["bias"], dtype=np.float16), want_acc=True)
    assert acc.tolist() == g["acc"]
    assert y.astype(np.float64).tolist() == g["y"]
    assert oracle.pack_int4(np.array(g["qw"])).tolist() == g["qw_int4_bytes"]


# ---------------------------------------------------------------- quantization

@pytest.mark.parametrize("bits", [8])
def test_block1_is_textbook_per_row_absmax_rtn(bits):
    """b = 1 means R = I: the method reduces to symmetric per-row absmax RTN
    (the 'none' outlier method), checked against torch's per-channel quantizer."""
    rng = np.random.default_rng(11)
    X = (rng.standard_normal((64, 256)) * 3).astype(np.float16)
    codes, scales = oracle.rotate_quant_act(X, 1, bits)
    x32 = torch.from_numpy(X.astype(np.float32))
    s = torch.from_numpy(scales.astype(np.float64))
    assert np.array_equal(scales, np.abs(X.astype(np.float32)).max(axis=1) / np.float32(127))
    q = torch.quantize_per_channel(x32, s, torch.zeros(64, dtype=torch.long), 0, torch.qint8)
    ref = q.int_repr().numpy()
    t = X.astype(np.float64) / scales[:, None].astype(np.float64)
    near_tie = np.abs(np.abs(t - np.floor(t)) - 0.5) < 1e-5
    assert np.array_equal(codes[~near_tie], ref[~near_tie])
    assert np.all(np.abs(codes.astype(int) - ref) <= 1)


@pytest.mark.parametrize("bits", [8, 4])
@pytest.mark.parametrize("b", [1, 64, 128])
def test_codes_range_rowmax_and_half_step_bound(bits, b):
    w = workloads.WORKLOADS["vit_l_w8a8"]
    X = workloads.activations(48, 512, w.outlier_frac, w.outlier_factor, 3)
    codes, scales = oracle.rotate_quant_act(X, b, bits)
    qmax, qmin = oracle.qmax(bits), oracle.qmin(bits)
    assert codes.min() >= qmin and codes.max() <= qmax
    _, x32 = oracle.rotate(X.astype(np.float64), b)
    amax_idx = np.argmax(np.abs(x32), axis=1)
    assert np.all(np.abs(codes[np.arange(48), amax_idx]) == qmax)
    s = scales[:, None].astype(np.float64)
    err = np.abs(x32.astype(np.float64) - s * codes)
    assert np.all(err <= s * 0.5 * (1 + 1e-5))


def test_zero_row_gives_zero_scale_and_codes():
    X = np.zeros((3, 128), dtype=np.float16)
    X[1, 5] = 2.0
    codes, scales = oracle.rotate_quant_act(X, 128, 8)
    assert scales[0] == 0 and scales[2] == 0 and scales[1] > 0
    assert np.all(codes[0] == 0) and np.all(codes[2] == 0)


@pytest.mark.parametrize("bits", [8, 4])
def test_mse_clip_matches_bruteforce_with_library_quantizer(bits):
    """Brute force on tiny rows: for every grid scale, quantize with torch's
    fake-quant routine and take the float64 error; the oracle's pick must be a
    minimiser and its per-alpha errors must agree."""
    rng = np.random.default_rng(bits)
    W = rng.standard_t(2, size=(4, 64)).astype(np.float16)  # heavy tails
    codes, scales, aidx, errs = oracle.quantize_weight(W, 1, bits, oracle.CLIP_MSE, want_errs=True)
    qmax, qmin = oracle.qmax(bits), oracle.qmin(bits)
    for n in range(4):
        w32 = W[n].astype(np.float32)
        amax = np.float32(np.max(np.abs(w32)))
        brute = []
        for i in range(oracle.MSE_GRID):
            a = np.float32(np.float32(100 - i) / np.float32(100))
            s = np.float32(np.float32(a * amax) / np.float32(qmax))
            deq = torch.fake_quantize_per_tensor_affine(torch.from_numpy(w32), float(s), 0, qmin, qmax)
            brute.append(float(np.sum((w32.astype(np.float64) - deq.numpy().astype(np.float64)) ** 2)))
        brute = np.array(brute)
        assert np.allclose(errs[n], brute, rtol=1e-5, atol=1e-12)
        assert errs[n, aidx[n]] <= brute.min() * (1 + 1e-5) + 1e-12
        assert errs[n, aidx[n]] <= errs[n, 0]  # never worse than plain absmax
        assert np.all(errs[n, : aidx[n]] > errs[n, aidx[n]])  # first strict minimum
        # codes of the chosen scale: clipped values saturate, the rest within half a step
        s = scales[n].astype(np.float64)
        clipped = np.abs(w32) > s * qmax
        assert np.all(np.isin(codes[n][clipped], [qmin, qmax, -qmax]))
        assert np.all(np.abs(w32[~clipped] - s * codes[n][~clipped]) <= s * 0.5 * (1 + 1e-5))
    if bits == 4:
        assert np.any(aidx > 0)  # with 16 levels the heavy-tailed rows really do clip


def test_absmax_mode_equals_alpha_one():
    W = workloads.weight(32, 256, 0.02, 9)
    c0, s0, a0 = oracle.quantize_weight(W, 64, 8, oracle.CLIP_ABSMAX)
    assert np.all(a0 == 0)
    c1, s1, a1, errs = oracle.quantize_weight(W, 64, 8, oracle.CLIP_MSE, want_errs=True)
    _, w32 = oracle.rotate(W.astype(np.float64), 64)
    assert np.array_equal(s0, np.abs(w32).max(axis=1) / np.float32(127))
    for n in range(32):
        assert errs[n, a1[n]] <= errs[n, 0]


def test_weight_error_is_rotation_invariant():
    """||W - deq R^T||_F == ||W~ - deq||_F for the orthogonal R (so minimising the
    error in the rotated domain minimises it for the original weight)."""
    W = workloads.weight(16, 256, 0.02, 4)
    codes, scales, _ = oracle.quantize_weight(W, 64, 8, oracle.CLIP_MSE)
    W64 = W.astype(np.float64)
    r64, r32 = oracle.rotate(W64, 64)
    deq = codes.astype(np.float64) * scales[:, None].astype(np.float64)
    back, _ = oracle.rotate(deq, 64)  # R is symmetric and R.R = I
    e_orig = np.linalg.norm(W64 - back)
    e_rot = np.linalg.norm(r64 - deq)
    assert abs(e_orig - e_rot) <= 1e-9 * e_rot


def test_rotation_spreads_outlier_channels():
    """The purpose stated on the pages: with outlier channels, the rotated
    quantization error is far below plain per-token RTN (b = 1)."""
    w = workloads.WORKLOADS["vit_l_w8a8"]
    X = workloads.activations(64, 1024, w.outlier_frac, w.outlier_factor, 17)
    X64 = X.astype(np.float64)
    errs = {}
    for b in (1, 128):
        codes, scales = oracle.rotate_quant_act(X, b, 8)
        deq = codes.astype(np.float64) * scales[:, None]
        back, _ = oracle.rotate(deq, b)
        errs[b] = np.linalg.norm(X64 - back) / np.linalg.norm(X64)
    assert errs[128] < 0.25 * errs[1]


# ---------------------------------------------------------------- int4 storage

def test_int4_pack_unpack_roundtrip_and_nibble_order():
    codes = np.arange(-8, 8, dtype=np.int8).repeat(2).reshape(2, 16)
    packed = oracle.pack_int4(codes)
    assert packed.shape == (2, 8)
    assert np.array_equal(oracle.unpack_int4(packed), codes)
    assert oracle.pack_int4(np.array([[3, -2]], dtype=np.int8)).tolist() == [[0xE3]]
    rng = np.random.default_rng(3)
    c = rng.integers(-8, 8, size=(7, 64)).astype(np.int8)
    assert np.array_equal(oracle.unpack_int4(oracle.pack_int4(c)), c)


def test_page_printed_sizes_pin_the_storage_density():
    with open(os.path.join(GOLDEN, "page_sizes.json")) as f:
        v = json.load(f)["values_as_printed"]
    r8 = v["int8_smaller_than_fp16_pct"] / 100
    r4 = v["int4_smaller_than_fp16_pct"] / 100
    N, K = 1024, 1024
    c8 = oracle.weight_bytes(N, K, 8) / (N * K * 2)   # bytes per fp16 byte (codes + scales)
    c4 = oracle.weight_bytes(N, K, 4) / (N * K * 2)
    # reduction = f * (1 - c) - e, solved for the share f and overhead e
    A = np.array([[1 - c8, -1.0], [1 - c4, -1.0]])
    f, e = np.linalg.solve(A, np.array([r8, r4]))
    assert 0.3 < f < 0.8 and -0.002 < e < 0.01
    # the printed INT4-vs-INT8 figure follows from the same model
    pred = 1 - (1 - r4) / (1 - r8)
    assert abs(pred - v["int4_smaller_than_int8_pct"] / 100) < 0.002
    # the FP16 and INT8 sizes themselves agree with the printed reduction
    assert abs(1 - v["int8_w8a8_gib"] / v["fp16_gib"] - r8) < 0.005
    # with one byte per int4 code (c4 == c8) the two printed reductions would
    # have to be equal; the oracle stores two codes per byte
    assert oracle.weight_bytes(N, K, 4) * 2 == N * K + 8 * N
    assert r4 - r8 > 0.1


# ---------------------------------------------------------------- GEMM + epilogue

@pytest.mark.parametrize("M,N,K", [(1, 1, 128), (7, 13, 256), (33, 20, 384)])
def test_accumulator_is_exact_integer_matmul(M, N, K):
    rng = np.random.default_rng(M * N)
    qx = rng.integers(-127, 128, size=(M, K)).astype(np.int8)
    qw = rng.integers(-127, 128, size=(N, K)).astype(np.int8)
    _, acc = oracle.gemm_dequant(qx, np.ones(M, np.float32), qw, np.ones(N, np.float32), want_acc=True)
    assert np.array_equal(acc, qx.astype(np.int64) @ qw.astype(np.int64).T)


def test_epilogue_scale_indexing_with_power_of_two_scales():
    """Per-token scale indexes rows (m), per-output-row weight scale indexes
    columns (n); with power-of-two scales every product is exact."""
    rng = np.random.default_rng(2)
    M, N, K = 5, 6, 256
    qx = rng.integers(-127, 128, size=(M, K)).astype(np.int8)
    qw = rng.integers(-127, 128, size=(N, K)).astype(np.int8)
    ex = rng.integers(-12, -4, size=M)
    ew = rng.integers(-10, -2, size=N)
    sx = (2.0 ** ex).astype(np.float32)
    sw = (2.0 ** ew).astype(np.float32)
    y = oracle.gemm_dequant(qx, sx, qw, sw)
    acc = qx.astype(np.int64) @ qw.astype(np.int64).T
    ref = (acc.astype(np.float32) * (2.0 ** (ex[:, None] + ew[None, :])).astype(np.float32)).astype(np.float16)
    assert np.array_equal(y.view(np.uint16), ref.view(np.uint16))
    y1 = oracle.gemm_dequant(qx, np.ones(M, np.float32), qw, np.ones(N, np.float32))
    assert np.array_equal(y1.view(np.uint16), acc.astype(np.float32).astype(np.float16).view(np.uint16))


def test_w4a4_equals_w8a8_on_unpacked_codes():
    rng = np.random.default_rng(4)
    qx = rng.integers(-8, 8, size=(9, 256)).astype(np.int8)
    qw = rng.integers(-8, 8, size=(11, 256)).astype(np.int8)
    sx = rng.random(9).astype(np.float32)
    sw = rng.random(11).astype(np.float32)
    y8 = oracle.gemm_dequant(qx, sx, qw, sw)
    y4 = oracle.gemm_dequant(oracle.unpack_int4(oracle.pack_int4(qx)), sx,
                             oracle.unpack_int4(oracle.pack_int4(qw)), sw)
    assert np.array_equal(y8.view(np.uint16), y4.view(np.uint16))


def test_int32_overflow_is_reported():
    K = 140000
    q = np.full((1, K), 127, dtype=np.int8)
    with pytest.raises(ValueError):
        oracle.gemm_dequant(q, np.ones(1, np.float32), q, np.ones(1, np.float32))


@pytest.mark.parametrize("bits,b", [(8, 64), (8, 128), (4, 128), (8, 1)])
def test_end_to_end_error_bound(bits, b):
    """|y - X W^T| <= sum_k(|x~_k| s_w/2 + |w~_k| s_x/2 + s_x s_w/4) + rounding,
    for absmax scales on both sides."""
    w = workloads.WORKLOADS["tiny_w8a8"]
    X, W, bias = workloads.linear_inputs(w, 0, with_bias=True)
    qw, sw, _ = oracle.quantize_weight(W, b, bits, oracle.CLIP_ABSMAX)
    qx, sx = oracle.rotate_quant_act(X, b, bits)
    y = oracle.gemm_dequant(qx, sx, qw, sw, bias).astype(np.float64)
    ref = X.astype(np.float64) @ W.astype(np.float64).T + bias.astype(np.float64)
    _, xr = oracle.rotate(X.astype(np.float64), b)
    _, wr = oracle.rotate(W.astype(np.float64), b)
    sx64, sw64 = sx.astype(np.float64)[:, None], sw.astype(np.float64)[None, :]
    K = X.shape[1]
    # sum_k |x~_k| s_w / 2  (per m, n) and sum_k |w~_k| s_x / 2
    term_x = np.abs(xr.astype(np.float64)).sum(axis=1)[:, None] * sw64 / 2
    term_w = np.abs(wr.astype(np.float64)).sum(axis=1)[None, :] * sx64 / 2
    term_xw = K * sx64 * sw64 / 4
    rounding = np.abs(ref) * 2.0 ** -10 + 1e-3 * (sx64 * sw64) + 1e-6
    bound = (term_x + term_w + term_xw) * (1 + 1e-4) + rounding
    assert np.all(np.abs(y - ref) <= bound)
    rel = np.linalg.norm(y - ref) / np.linalg.norm(ref)
    assert rel < (0.5 if bits == 4 else 0.02 if b > 1 else 0.05)


# ---------------------------------------------------------------- single roundings, checked exactly

def _nearest_int_even(fr):
    """Nearest integer to a Fraction, ties to even."""
    from fractions import Fraction
    f = fr.numerator // fr.denominator
    rem = fr - f
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and f % 2 == 1):
        f += 1
    return f


def _is_nearest_f32(exact, r32):
    """r32 is the float32 nearest to the Fraction `exact` (ties to even mantissa)."""
    from fractions import Fraction
    r = np.float32(r32)
    lo = np.nextafter(r, np.float32(-np.inf))
    hi = np.nextafter(r, np.float32(np.inf))
    d = abs(Fraction(float(r)) - exact)
    for nb in (lo, hi):
        dn = abs(Fraction(float(nb)) - exact)
        if dn < d:
            return False
        if dn == d and (int(r.view(np.uint32)) & 1):
            return False
    return True


def test_quantizer_rounds_the_exact_product_once():
    from fractions import Fraction
    rng = np.random.default_rng(21)
    xs = (rng.standard_normal(3000) * 20).astype(np.float32)
    invs = (rng.random(3000) * 10 + 0.01).astype(np.float32)
    # plus the half-way cases where fp32(x * inv) lands on k + 0.5
    xs = np.concatenate([xs, np.float32([9.0, 6.25, 1.25, 7.75, -7.375])])
    invs = np.concatenate([invs, np.float32([7.0555553, 0.4, 0.4, 8.193548, 8.610169])])
    for x, inv in zip(xs, invs):
        ref = _nearest_int_even(Fraction(float(x)) * Fraction(float(inv)))
        ref = max(-127, min(127, ref))
        assert oracle.quantize_value(x, inv, 8) == ref, (x, inv)
    assert oracle.quantize_value(np.float32(9.0), np.float32(7.0555553), 8) == 63  # fp32(x*inv) would say 63.5 -> 64


def test_epilogue_multiply_add_rounds_once():
    from fractions import Fraction
    rng = np.random.default_rng(22)
    for _ in range(3000):
        acc = int(rng.integers(-2**24, 2**24))
        sx = np.float32(rng.random() * 0.1)
        sw = np.float32(rng.random() * 0.01)
        bias = np.float32(np.float16(rng.standard_normal() * 0.05))
        got = np.float32(oracle.epilogue_value(acc, sx, sw, bias))
        t = np.float32(np.float32(acc) * sx)  # IEEE fp32 product
        exact = Fraction(float(t)) * Fraction(float(sw)) + Fraction(float(bias))
        assert _is_nearest_f32(exact, got), (acc, sx, sw, bias)


# ----------------------------------------------------------------------------- tensor-wise variant

@pytest.mark.parametrize("bits", [8, 4])
def test_tensorwise_mse_matches_bruteforce_with_library_quantizer(bits):
    """One scale for the tensor: brute force over the grid with torch's
    fake-quant routine on the whole (unrotated, b = 1) tensor; the oracle's
    pick is the first strict minimiser and its per-alpha errors agree."""
    rng = np.random.default_rng(10 + bits)
    W = rng.standard_t(2, size=(5, 64)).astype(np.float16)
    codes, scales, aidx, errs = oracle.quantize_weight_tensorwise(W, 1, bits, oracle.CLIP_MSE, want_errs=True)
    qmax, qmin = oracle.qmax(bits), oracle.qmin(bits)
    w32 = W.astype(np.float32)
    amax = np.float32(np.max(np.abs(w32)))
    brute = []
    for i in range(oracle.MSE_GRID):
        a = np.float32(np.float32(100 - i) / np.float32(100))
        s = np.float32(np.float32(a * amax) / np.float32(qmax))
        deq = torch.fake_quantize_per_tensor_affine(torch.from_numpy(w32), float(s), 0, qmin, qmax)
        brute.append(float(np.sum((w32.astype(np.float64) - deq.numpy().astype(np.float64)) ** 2)))
    brute = np.array(brute)
    assert np.allclose(errs, brute, rtol=1e-5, atol=1e-12)
    assert errs[aidx] <= brute.min() * (1 + 1e-5) + 1e-12
    assert np.all(errs[:aidx] > errs[aidx])
    s = scales[0].astype(np.float64)
    assert np.all(scales == scales[0])
    clipped = np.abs(w32) > s * qmax
    assert np.all(np.isin(codes[clipped], [qmin, qmax, -qmax]))
    assert np.all(np.abs(w32[~clipped] - s * codes[~clipped]) <= s * 0.5 * (1 + 1e-5))


def test_tensorwise_absmax_scale_and_codes_from_a_dense_rotation():
    """Absmax mode against a dense float64 rotation (scipy's Hadamard): the
    scale is the tensor's max |W R| / qmax and the codes are rne(x * (1/s))."""
    b, K = 64, 256
    W = workloads.weight(8, K, 0.02, 21)
    R = scipy.linalg.block_diag(*([scipy.linalg.hadamard(b) / math.sqrt(b)] * (K // b)))
    WR = (W.astype(np.float64) @ R).astype(np.float32)
    s_ref = np.float32(np.float32(1.0 * np.max(np.abs(WR))) / np.float32(127))
    codes, scales, aidx = oracle.quantize_weight_tensorwise(W, b, 8, oracle.CLIP_ABSMAX)
    assert aidx == 0
    assert np.all(scales == scales[0])
    assert abs(float(scales[0]) - float(s_ref)) <= 1e-6 * float(s_ref)
    inv = np.float64(np.float32(1.0) / scales[0])
    ref = np.clip(np.rint(WR.astype(np.float64) * inv), -127, 127)
    d = np.abs(codes.astype(np.int32) - ref.astype(np.int32))
    assert d.max() <= 1 and np.count_nonzero(d) <= 1e-3 * d.size


@pytest.mark.parametrize("bits", [8, 4])
@pytest.mark.parametrize("clip", [0, 1])
def test_tensorwise_single_row_is_rowwise(bits, clip):
    """With one row the tensor is the row: both converters agree exactly."""
    W = workloads.weight(1, 512, 0.02, 5)
    c1, s1, a1 = oracle.quantize_weight(W, 128, bits, clip)
    c2, s2, a2 = oracle.quantize_weight_tensorwise(W, 128, bits, clip)
    assert np.array_equal(c1, c2) and np.array_equal(s1, s2) and int(a1[0]) == a2


def test_tensorwise_absmax_scale_is_the_largest_row_scale():
    """Rounding is monotone, so max_n fp32(amax_n / qmax) = fp32(max_n amax_n / qmax)."""
    W = workloads.weight(16, 256, 0.02, 23)
    _, s_rows, _ = oracle.quantize_weight(W, 64, 4, oracle.CLIP_ABSMAX)
    _, s_t, _ = oracle.quantize_weight_tensorwise(W, 64, 4, oracle.CLIP_ABSMAX)
    assert np.all(s_t == s_rows.max())
