"""Feature-major split K over thread-block clusters (few tokens).

With at most 128 tokens the GEMM runs feature-major: a tile is 128 output
features by all the tokens (32, 64 or 128 columns), so every weight byte is
read once.  Where the tiles alone leave SMs idle, the K loop of a tile is split
over a cluster of 2, 4 or 8 CTAs whose int32 partial accumulators are added
through distributed shared memory.  Integer sums are exact, so the int32
accumulators and the fp16 outputs must equal the oracle's bit for bit for
every cluster size and tile width, through the codes entry points and through
the linear, on repeated calls and in CUDA-graph replays.
Source: civarchive "SAM 3.1 Multiplex ConvRot" release, "Quantization recipe"
(integer GEMM over the quantized codes, per-row dequantization).
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


def sms():
    return torch.cuda.get_device_properties(0).multi_processor_count


# (M, N, K, tile_n, k_splits on a 148-SM B200): every cluster size and token
# tile width, ragged N (1000, 520) and ragged M, a split limited by K (16 steps
# of 128: two slices of 8) and shapes whose slices would be too short to split
CASES = [
    (16, 4096, 4096, 32, 4),
    (5, 4096, 2048, 32, 2),
    (24, 1024, 16384, 32, 8),
    (40, 9472, 2048, 64, 2),
    (64, 1000, 4096, 64, 4),
    (100, 1024, 8192, 128, 8),
    (90, 2048, 2048, 128, 2),
    (128, 2048, 8192, 128, 8),
    (33, 520, 640, 64, 1),
    (128, 3072, 1024, 128, 1),
]


def codes(M, N, K, bits, seed):
    rng = np.random.default_rng(seed)
    lo, hi = (-127, 128) if bits == 8 else (-8, 8)
    qx = rng.integers(lo, hi, size=(M, K)).astype(np.int8)
    qw = rng.integers(lo, hi, size=(N, K)).astype(np.int8)
    sx = (rng.random(M) * 0.01 + 1e-4).astype(np.float32)
    sw = (rng.random(N) * 0.01 + 1e-4).astype(np.float32)
    return qx, sx, qw, sw


def gemm_args(qx, sx, qw, sw, bits):
    if bits == 8:
        return (dev(qx), dev(sx), dev(qw), dev(sw)), cr.convrot_gemm_w8a8
    return (dev(oracle.pack_int4(qx)), dev(sx), dev(oracle.pack_int4(qw)), dev(sw)), cr.convrot_gemm_w4a4


@pytest.mark.parametrize("bits", [8, 4])
@pytest.mark.parametrize("M,N,K,tile_n,splits", CASES)
def test_split_gemm_bit_exact(M, N, K, tile_n, splits, bits):
    plan = cr.convrot_linear_plan(M, K, N, bits, 128, cr.convrot_linear_workspace_bytes(M, K, N, bits))
    if plan["gemm_kind"] == 1:
        assert plan["tile_n"] == tile_n
        if sms() == 148:
            assert plan["k_splits"] == splits
    qx, sx, qw, sw = codes(M, N, K, bits, seed=M * 7 + N + K)
    bias = wl.bias(N, seed=M)
    args, fn = gemm_args(qx, sx, qw, sw, bits)
    acc = torch.empty((M, N), dtype=torch.int32, device="cuda")
    y = host(fn(*args, bias=dev(bias), acc_out=acc))
    yr, accr = oracle.gemm_dequant(qx, sx, qw, sw, bias, want_acc=True)
    assert np.array_equal(host(acc), accr)
    assert np.array_equal(y.view(np.uint16), yr.view(np.uint16))
    # again, into the same output: nothing carries over between calls
    y2 = host(fn(*args, bias=dev(bias)))
    assert np.array_equal(y2.view(np.uint16), yr.view(np.uint16))


@pytest.mark.parametrize("bits", [8, 4])
@pytest.mark.parametrize("M,N,K", [(16, 4096, 4096), (100, 4096, 1024), (40, 9472, 2048)])
def test_split_linear_equals_oracle_gemm_of_its_codes(M, N, K, bits):
    X = wl.activations(M, K, 0.01, 30.0, seed=M + 3)
    W = wl.weight(N, K, 0.02, seed=N + 3)
    bias = wl.bias(N, seed=5)
    Wq, sw = cr.convrot_quantize_weight(dev(W), 128, bits, cr.CLIP_ABSMAX)
    fn = cr.convrot_linear_w8a8 if bits == 8 else cr.convrot_linear_w4a4
    for ws_bytes in (cr.convrot_workspace_bytes(M, K, bits), cr.convrot_linear_workspace_bytes(M, K, N, bits)):
        ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
        y = host(fn(dev(X), Wq, sw, 128, bias=dev(bias), workspace=ws))
        raw = host(ws)
        qx = raw[: M * K].view(np.int8).reshape(M, K)
        off = (M * K + 255) // 256 * 256
        sx = raw[off: off + 4 * M].view(np.float32)
        qw = host(Wq)
        if bits == 4:
            qw = oracle.unpack_int4(qw)
        yr = oracle.gemm_dequant(qx, sx, qw, host(sw), bias)
        assert np.array_equal(y.view(np.uint16), yr.view(np.uint16))


@pytest.mark.parametrize("M,N,K", [(16, 4096, 4096), (100, 4096, 1024)])
def test_split_gemm_in_cuda_graph_replays(M, N, K):
    """The cluster launches are captured and replayed like any other launch;
    each replay computes the product of the codes it finds."""
    qx, sx, qw, sw = codes(M, N, K, 8, seed=K)
    Xq, Sx, Wq, Sw = dev(qx), dev(sx), dev(qw), dev(sw)
    Y = torch.empty((M, N), dtype=torch.float16, device="cuda")
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        cr.convrot_gemm_w8a8(Xq, Sx, Wq, Sw, Y=Y, stream=s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        cr.convrot_gemm_w8a8(Xq, Sx, Wq, Sw, Y=Y, stream=s)
    for seed in (1, 2, 3):
        qx2, sx2, _, _ = codes(M, N, K, 8, seed=seed)
        Xq.copy_(dev(qx2))
        Sx.copy_(dev(sx2))
        torch.cuda.synchronize()
        g.replay()
        yr = oracle.gemm_dequant(qx2, sx2, qw, sw, None)
        assert np.array_equal(host(Y).view(np.uint16), yr.view(np.uint16))
