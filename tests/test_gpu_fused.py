"""The W8A8 linear with the rotation fused into the GEMM kernel
(convrot_linear_w8a8_fused).

The GEMM's CTAs carry activation warps that rotate and quantize units of
tokens into the workspace beside the tensor-core main loop; the producer loads
a 128-token panel only once every unit touching it has been counted into the
panel's counter (zeroed by a small kernel launched just before).  The rotation
runs the same butterfly stages in the same order as the separate activation
kernel, so the fused linear must equal the two-launch linear
(convrot_linear_quant_act + convrot_linear_gemm) bit for bit: codes, scales and
output.  Both must meet the oracle's bars: codes within 1 on at most 0.1 % of
elements, scales within 1e-5 relative, and the output bit-exact against the
oracle's GEMM + dequant of the workspace's codes.  Zeroing the counters before
each launch makes repeated calls and CUDA-graph replays on one workspace safe.
Source: civarchive "SAM 3.1 Multiplex ConvRot" release, "Quantization recipe"
(online activation quantization) and "Future improvements" (fusion).
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
    assert plan["fused_available"] == 1, plan
    # whatever the counter area held before (here: all ones) must not count
    ws = torch.full((big,), 0xFF, dtype=torch.uint8, device="cuda")
    y = host(cr.convrot_linear_w8a8_fused(Xd, Wq, sw, 128, bias=bd, workspace=ws))
    raw = host(ws)
    qx, sx, _ = ws_parts(raw, M, K)
    # the two-launch linear on its own (minimum) workspace
    ws2 = torch.empty(cr.convrot_workspace_bytes(M, K, 8), dtype=torch.uint8, device="cuda")
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
    Ys = [cr.convrot_linear_w8a8_fused(X, Wq, sw, 128, workspace=ws) for X in Xs]
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
        cr.convrot_linear_w8a8_fused(X, Wq, sw, 128, Y=Y, workspace=ws, stream=s)  # per-device set-up outside capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        cr.convrot_linear_w8a8_fused(X, Wq, sw, 128, Y=Y, workspace=ws, stream=s)
    ws2 = torch.empty(cr.convrot_workspace_bytes(M, K, 8), dtype=torch.uint8, device="cuda")
    for seed in (22, 23, 24):
        X.copy_(dev(wl.activations(M, K, 0.01, 30.0, seed=seed)))
        torch.cuda.synchronize()
        g.replay()
        torch.cuda.synchronize()
        cr.convrot_linear_quant_act(X, 128, 8, ws2)
        y2 = host(cr.convrot_linear_gemm(ws2, M, K, 8, Wq, sw))
        assert np.array_equal(host(Y).view(np.uint16), y2.view(np.uint16))


def test_plan_query_and_unsupported_shapes():
    """The plan query tells where the fused entry point applies; elsewhere it
    refuses with CONVROT_ERR_UNSUPPORTED (or a workspace error) before any launch."""
    M, K, N = 5184, 1024, 3072
    big = cr.convrot_linear_workspace_bytes(M, K, N, 8)
    p = cr.convrot_linear_plan(M, K, N, 8, 128, big)
    assert p["fused_available"] == 1 and p["launches"] == 2 and p["gemm_kind"] == 0 and p["tile_n"] == 256
    assert cr.convrot_linear_plan(M, K, N, 8, 64, big)["fused_available"] == 0
    assert cr.convrot_linear_plan(M, 4096, N, 8, 128, cr.convrot_linear_workspace_bytes(M, 4096, N, 8))[
        "fused_available"] == 0
    p4 = cr.convrot_linear_plan(M, K, N, 4, 128, cr.convrot_linear_workspace_bytes(M, K, N, 4))
    assert p4["fused_available"] == 0 and p4["weights_widened"] == 1
    assert cr.convrot_linear_plan(M, K, N, 4, 128, cr.convrot_workspace_bytes(M, K, 4))["weights_widened"] == 0
    assert cr.convrot_linear_plan(64, K, N, 4, 128, cr.convrot_linear_workspace_bytes(64, K, N, 4))[
        "weights_widened"] == 0
    assert cr.convrot_linear_plan(M, K, N, 8, 128, cr.convrot_workspace_bytes(M, K, 8))["fused_available"] == 0
    small = cr.convrot_linear_plan(1, 4096, 4096, 8, 128, cr.convrot_linear_workspace_bytes(1, 4096, 4096, 8))
    assert small["gemm_kind"] == 2 and small["fused_available"] == 0
    mid = cr.convrot_linear_plan(16, 4096, 4096, 8, 128, cr.convrot_linear_workspace_bytes(16, 4096, 4096, 8))
    assert mid["gemm_kind"] == 1 and mid["k_splits"] > 1
    X = torch.zeros((M, 4096), dtype=torch.float16, device="cuda")
    Wq = torch.zeros((N, 4096), dtype=torch.int8, device="cuda")
    sw = torch.ones(N, dtype=torch.float32, device="cuda")
    Y = torch.full((M, N), 3.0, dtype=torch.float16, device="cuda")
    with pytest.raises(cr.ConvRotError) as err:
        cr.convrot_linear_w8a8_fused(X, Wq, sw, 128, Y=Y)
    assert err.value.status == cr.ERR_UNSUPPORTED
    X1 = torch.zeros((M, K), dtype=torch.float16, device="cuda")
    ws = torch.empty(cr.convrot_workspace_bytes(M, K, 8), dtype=torch.uint8, device="cuda")
    with pytest.raises(cr.ConvRotError) as err:
        cr.convrot_linear_w8a8_fused(X1, Wq[:, :K].contiguous(), sw, 128, Y=Y, workspace=ws)
    assert err.value.status == cr.ERR_WORKSPACE
    torch.cuda.synchronize()
    assert torch.all(Y == 3.0)
