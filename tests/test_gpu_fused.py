"""The W8A8 linear as one launch: rotate + quantize fused into the integer GEMM.

With a workspace of at least convrot_linear_workspace_bytes, a W8A8 linear over
more than 128 tokens (block 128, K <= 2048) runs as a single kernel: extra
activation warps in every CTA rotate and quantize units of tokens into the
workspace while the tensor core works, and the producer loads a 128-token
panel only once every unit touching it has been counted into the panel's counter.
The rotation runs the same butterfly stages in the same order as the separate
activation kernel, so the fused linear must equal the two-launch linear
(convrot_linear_quant_act + convrot_linear_gemm) bit for bit: codes, scales and
output.  Both must meet the oracle's bars: codes within 1 on at most 0.1 % of
elements, scales within 1e-5 relative, and the output bit-exact against the
oracle's GEMM + dequant of the workspace's codes.  The panel counters are
zeroed by a small kernel launched just before the fused kernel, which makes
repeated calls and CUDA-graph replays on one workspace safe.  Source: civarchive "SAM
3.1 Multiplex ConvRot" release, "Quantization recipe" (online activation
quantization) and "Future improvements" (fusion).
"""
import numpy as np
import pytest
import torch

import oracle
from rotated_bit_quantized_block_b200 import binding as cr
from rotated_bit_quantized_block_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host(t):
    torch.cuda.synchronize()
    return t.cpu().numpy()


@pytest.fixture(autouse=True)
def _status_clean():
    yield
    cr.convrot_device_status()


def unpack(q, bits):
    return oracle.unpack_int4(q) if bits == 4 else q


def ws_parts(raw, M, K):
    qx = raw[: M * K].view(np.int8).reshape(M, K)
    off = (M * K + 255) // 256 * 256
    sx = raw[off: off + 4 * M].view(np.float32)
    flags_off = off + (4 * M + 255) // 256 * 256
    return qx, sx, flags_off


def assert_codes_close(got, ref):
    d = np.abs(got.astype(np.int32) - ref.astype(np.int32))
    assert d.max(initial=0) <= 1
    assert np.count_nonzero(d) <= 1e-3 * d.size


def sample_rows(M):
    rows = {0, 1, 127, 128, M - 1, M - 2}
    rows |= set(np.linspace(0, M - 1, 40).astype(int).tolist())
    return np.array(sorted(r for r in rows if 0 <= r < M))


# (M, N, K): ViT-L qkv (256-wide tiles), proj (192-wide) and fc1, DiT qkv
# (CTA pairs, rows spanning 1.5 warps), ragged token and feature counts, K =
# 128 and 384 (rows shorter than a warp, and not a power of two), K = 2048
FUSED_CASES = [(5184, 3072, 1024), (5184, 1024, 1024), (5184, 4096, 1024), (8192, 4608, 1536),
               (300, 520, 1024), (1000, 264, 2048), (129, 1024, 128), (2049, 4096, 384), (4100, 2056, 2048)]


@pytest.mark.parametrize("M,N,K", FUSED_CASES)
def test_fused_linear_equals_two_launches_and_oracle(M, N, K):
    X = wl.activations(M, K, 0.01, 30.0, seed=M + K)
    W = wl.weight(N, K, 0.02, seed=N + K)
    bias = wl.bias(N, seed=N)
    Xd, bd = dev(X), dev(bias)
    Wq, sw = cr.convrot_quantize_weight(dev(W), 128, 8, cr.CLIP_MSE)
    big = cr.convrot_linear_workspace_bytes(M, K, N, 8)
    plan = cr.convrot_linear_plan(M, K, N, 8, 128, big)
    assert plan["fused"] == 1, plan
    # whatever the counter area held before (here: all ones) must not count
    ws = torch.full((big,), 0xFF, dtype=torch.uint8, device="cuda")
    y = host(cr.convrot_linear_w8a8(Xd, Wq, sw, 128, bias=bd, workspace=ws))
    raw = host(ws)
    qx, sx, _ = ws_parts(raw, M, K)
    # the two-launch linear on its own (minimum) workspace
    ws2 = torch.empty(cr.convrot_workspace_bytes(M, K, 8), dtype=torch.uint8, device="cuda")
    assert cr.convrot_linear_plan(M, K, N, 8, 128, ws2.numel())["fused"] == 0
    cr.convrot_linear_quant_act(Xd, 128, 8, ws2)
    y2 = host(cr.convrot_linear_gemm(ws2, M, K, 8, Wq, sw, bias=bd))
    qx2, sx2, _ = ws_parts(host(ws2), M, K)
    assert np.array_equal(qx, qx2)
    assert np.array_equal(sx.view(np.uint32), sx2.view(np.uint32))
    assert np.array_equal(y.view(np.uint16), y2.view(np.uint16))
    # against the oracle on sampled rows
    rows = sample_rows(M)
    qr, sr = oracle.rotate_quant_act(X[rows], 128, 8)
    assert np.allclose(sx[rows], sr, rtol=1e-5, atol=0)
    assert_codes_close(qx[rows], qr)
    yr = oracle.gemm_dequant(qx[rows], sx[rows], host(Wq), host(sw), bias)
    assert np.array_equal(y[rows].view(np.uint16), yr.view(np.uint16))


def test_fused_linear_repeated_calls_fresh_inputs():
    """Back-to-back calls on one workspace with different inputs: every call
    reads its own codes."""
    M, N, K = 3000, 2048, 1024
    W = wl.weight(N, K, 0.02, seed=5)
    Wq, sw = cr.convrot_quantize_weight(dev(W), 128, 8, cr.CLIP_ABSMAX)
    ws = torch.empty(cr.convrot_linear_workspace_bytes(M, K, N, 8), dtype=torch.uint8, device="cuda")
    ws2 = torch.empty(cr.convrot_workspace_bytes(M, K, 8), dtype=torch.uint8, device="cuda")
    Xs = [dev(wl.activations(M, K, 0.01, 30.0, seed=s)) for s in range(4)]
    Ys = [cr.convrot_linear_w8a8(X, Wq, sw, 128, workspace=ws) for X in Xs]
    for X, Y in zip(Xs, Ys):
        cr.convrot_linear_quant_act(X, 128, 8, ws2)
        y2 = host(cr.convrot_linear_gemm(ws2, M, K, 8, Wq, sw))
        assert np.array_equal(host(Y).view(np.uint16), y2.view(np.uint16))


def test_fused_linear_in_cuda_graph_replays():
    """Each replay of a captured fused linear zeroes its panel counters first,
    so each replay's output equals the two-launch linear of the input it saw."""
    M, N, K = 2600, 3072, 1024
    W = wl.weight(N, K, 0.02, seed=9)
    Wq, sw = cr.convrot_quantize_weight(dev(W), 128, 8, cr.CLIP_MSE)
    X = dev(wl.activations(M, K, 0.01, 30.0, seed=21))
    Y = torch.empty((M, N), dtype=torch.float16, device="cuda")
    ws = torch.empty(cr.convrot_linear_workspace_bytes(M, K, N, 8), dtype=torch.uint8, device="cuda")
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        cr.convrot_linear_w8a8(X, Wq, sw, 128, Y=Y, workspace=ws, stream=s)  # per-device set-up outside capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        cr.convrot_linear_w8a8(X, Wq, sw, 128, Y=Y, workspace=ws, stream=s)
    ws2 = torch.empty(cr.convrot_workspace_bytes(M, K, 8), dtype=torch.uint8, device="cuda")
    for seed in (22, 23, 24):
        X.copy_(dev(wl.activations(M, K, 0.01, 30.0, seed=seed)))
        torch.cuda.synchronize()
        g.replay()
        torch.cuda.synchronize()
        cr.convrot_linear_quant_act(X, 128, 8, ws2)
        y2 = host(cr.convrot_linear_gemm(ws2, M, K, 8, Wq, sw))
        assert np.array_equal(host(Y).view(np.uint16), y2.view(np.uint16))


def test_plan_query_matches_the_paths():
    """The plan query: fused for token-major W8A8 with the linear workspace and
    for the fewest tokens with any workspace; two launches with the minimum
    workspace for more tokens, for token-major W4A4, for the feature-major
    tiles, and for block sizes the fused kernels are not built for."""
    M, K, N = 5184, 1024, 3072
    big = cr.convrot_linear_workspace_bytes(M, K, N, 8)
    assert cr.convrot_linear_plan(M, K, N, 8, 128, big)["fused"] == 1
    assert cr.convrot_linear_plan(M, K, N, 8, 64, big)["fused"] == 0
    assert cr.convrot_linear_plan(M, K, N, 4, 128, cr.convrot_linear_workspace_bytes(M, K, N, 4))["fused"] == 0
    assert cr.convrot_linear_plan(M, K, N, 8, 128, cr.convrot_workspace_bytes(M, K, 8))["fused"] == 0
    small = cr.convrot_linear_plan(1, 4096, 4096, 8, 128, cr.convrot_workspace_bytes(1, 4096, 8))
    assert small["fused"] == 1 and small["gemm_kind"] == 2 and small["launches"] == 1
    assert cr.convrot_linear_plan(1, 4096, 4096, 8, 64, cr.convrot_workspace_bytes(1, 4096, 8))["fused"] == 0
    mid = cr.convrot_linear_plan(16, 4096, 4096, 8, 128, cr.convrot_linear_workspace_bytes(16, 4096, 4096, 8))
    assert mid["fused"] == 0 and mid["gemm_kind"] == 1 and mid["k_splits"] > 1


# (M, N, K, bits): the weight-streaming plan's token counts (up to 4 tokens
# with int8 weights, 8 with int4), K from one to sixteen 512-code chunks
# (including three, which does not divide the sixteen warps), ragged N
SMALL_CASES = [(1, 4096, 4096, 8), (4, 2056, 1024, 8), (3, 1000, 1536, 8), (2, 4104, 2048, 8),
               (8, 520, 8192, 4), (7, 64, 512, 4), (1, 3072, 4096, 4), (4, 1024, 6144, 8)]


@pytest.mark.parametrize("M,N,K,bits", SMALL_CASES)
def test_fused_small_m_linear_equals_two_launches_and_oracle(M, N, K, bits):
    """The fewest tokens: every CTA rotates and quantizes the token rows into
    shared memory, then streams its share of the weights.  Codes, scales (left
    in the workspace) and output equal the two-launch linear bit for bit and
    meet the oracle's bars."""
    X = wl.activations(M, K, 0.01, 30.0, seed=M + K + bits)
    W = wl.weight(N, K, 0.02, seed=N + K + 1)
    bias = wl.bias(N, seed=N + 2)
    Xd, bd = dev(X), dev(bias)
    Wq, sw = cr.convrot_quantize_weight(dev(W), 128, bits, cr.CLIP_MSE)
    ws = torch.empty(cr.convrot_workspace_bytes(M, K, bits), dtype=torch.uint8, device="cuda")
    plan = cr.convrot_linear_plan(M, K, N, bits, 128, ws.numel())
    assert plan["fused"] == 1 and plan["gemm_kind"] == 2 and plan["launches"] == 1, plan
    fn = cr.convrot_linear_w8a8 if bits == 8 else cr.convrot_linear_w4a4
    y = host(fn(Xd, Wq, sw, 128, bias=bd, workspace=ws))
    qx, sx, _ = ws_parts(host(ws), M, K)
    ws2 = torch.empty_like(ws)
    cr.convrot_linear_quant_act(Xd, 128, bits, ws2)
    y2 = host(cr.convrot_linear_gemm(ws2, M, K, bits, Wq, sw, bias=bd))
    qx2, sx2, _ = ws_parts(host(ws2), M, K)
    assert np.array_equal(qx, qx2)
    assert np.array_equal(sx.view(np.uint32), sx2.view(np.uint32))
    assert np.array_equal(y.view(np.uint16), y2.view(np.uint16))
    qr, sr = oracle.rotate_quant_act(X, 128, bits)
    assert np.allclose(sx, sr, rtol=1e-5, atol=0)
    assert_codes_close(qx, qr)
    yr = oracle.gemm_dequant(qx, sx, unpack(host(Wq), bits), host(sw), bias)
    assert np.array_equal(y.view(np.uint16), yr.view(np.uint16))
