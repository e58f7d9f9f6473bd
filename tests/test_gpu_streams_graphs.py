"""Linears under concurrency and graph capture.

Every launch of a linear is enqueued on the caller's stream with programmatic
dependent launch, and all its state lives in the caller's workspace, so
(a) linears of different shapes and plans (weight-streaming, feature-major
split K over clusters, token-major tiles, CTA pairs, W4A4 with widened
weights) running at the same time on independent streams and workspaces must
each give exactly what they give alone, (b) a chain of such linears
captured once in a CUDA graph must give, on every replay, exactly what the
same chain gives when launched eagerly, and (c) a linear fed the previous
linear's output must quantize the finished rows although its launch may
start during the previous GEMM.  Integer sums are exact and the epilogue
rounds identically, so the comparisons are bit for bit.
Source: civarchive "SAM 3.1 Multiplex ConvRot" release, "Quantization recipe"
(online activation quantization, integer GEMM, per-row dequantization).
"""
import numpy as np
import pytest
import torch

from rotated_bit_quantized_block_b200 import binding as cr
from rotated_bit_quantized_block_b200 import workloads as wl

pytestmark = pytest.mark.gpu

# (M, K, N, bits): one of each plan
SHAPES = [(1, 4096, 4096, 8), (16, 4096, 2048, 8), (100, 2048, 1024, 4), (700, 1024, 3072, 8),
          (2304, 1536, 4608, 8), (1300, 1024, 2000, 4)]


@pytest.fixture(autouse=True)
def _status_clean():
    yield
    cr.convrot_device_status()


def make(M, K, N, bits, seed):
    X = torch.from_numpy(wl.activations(M, K, 0.01, 30.0, seed=seed)).cuda()
    W = torch.from_numpy(wl.weight(N, K, 0.02, seed=seed + 1)).cuda()
    bias = torch.from_numpy(wl.bias(N, seed=seed + 2)).cuda()
    Wq, sw = cr.convrot_quantize_weight(W, 128, bits, cr.CLIP_ABSMAX)
    ws = torch.empty(cr.convrot_linear_workspace_bytes(M, K, N, bits), dtype=torch.uint8, device="cuda")
    Y = torch.empty((M, N), dtype=torch.float16, device="cuda")
    fn = cr.convrot_linear_w8a8 if bits == 8 else cr.convrot_linear_w4a4
    return {"X": X, "Wq": Wq, "sw": sw, "bias": bias, "ws": ws, "Y": Y, "fn": fn}


def run(it, stream=None):
    return it["fn"](it["X"], it["Wq"], it["sw"], 128, bias=it["bias"], Y=it["Y"], workspace=it["ws"], stream=stream)


def test_linears_on_concurrent_streams():
    items = [make(*s, seed=10 * i) for i, s in enumerate(SHAPES)]
    ref = []
    for it in items:
        run(it)
        torch.cuda.synchronize()
        ref.append(it["Y"].clone())
    for it in items:
        it["Y"].fill_(0)
    streams = [torch.cuda.Stream() for _ in items]
    torch.cuda.synchronize()
    for rep in range(3):
        for it, st in zip(items, streams):
            with torch.cuda.stream(st):
                run(it, st)
        torch.cuda.synchronize()
        for it, r in zip(items, ref):
            assert torch.equal(it["Y"].view(torch.int16), r.view(torch.int16))


def test_chain_of_linears_in_one_graph():
    items = [make(*s, seed=7 + 10 * i) for i, s in enumerate(SHAPES)]
    st = torch.cuda.Stream()
    with torch.cuda.stream(st):
        for it in items:
            run(it, st)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=st):
        for it in items:
            run(it, st)
    for seed in (101, 102):
        # new inputs, eager reference first
        for i, it in enumerate(items):
            M, K = it["X"].shape
            it["X"].copy_(torch.from_numpy(wl.activations(M, K, 0.01, 30.0, seed=seed + i)))
        torch.cuda.synchronize()
        ref = []
        for it in items:
            run(it)
            torch.cuda.synchronize()
            ref.append(it["Y"].clone())
            it["Y"].fill_(0)
        torch.cuda.synchronize()
        g.replay()
        torch.cuda.synchronize()
        for it, r in zip(items, ref):
            assert torch.equal(it["Y"].view(torch.int16), r.view(torch.int16))
    del g


# (M, K, N1, N2, bits): an MLP pair at ViT-L width (token-major GEMMs), few
# tokens (feature-major clusters, the weight-streaming kernel), int4 weights
CHAINS = [(5184, 1024, 4096, 1024, 8), (5184, 1024, 4096, 1024, 4), (16, 4096, 4096, 4096, 8),
          (1, 4096, 4096, 4096, 8), (300, 1024, 2048, 1024, 4)]


@pytest.mark.parametrize("shared_ws", [False, True])
@pytest.mark.parametrize("M,K,N1,N2,bits", CHAINS)
def test_linear_consumes_the_previous_linears_output(M, K, N1, N2, bits, shared_ws):
    """The second linear's activation launch may become resident, and start
    fetching its rows, while the first linear's GEMM is still writing them;
    what it quantizes must be the finished rows.  Back-to-back launches, eager
    and replayed from a CUDA graph, equal the same two calls with a device
    synchronisation between them, bit for bit (also when both linears share
    one workspace, so the second's codes overwrite those the first GEMM read)."""
    first = make(M, K, N1, bits, seed=M + 1)
    second = make(M, N1, N2, bits, seed=M + 2)
    second["X"] = first["Y"]
    if shared_ws:
        n = max(first["ws"].numel(), second["ws"].numel())
        first["ws"] = second["ws"] = torch.empty(n, dtype=torch.uint8, device="cuda")
    run(first)
    torch.cuda.synchronize()
    run(second)
    torch.cuda.synchronize()
    ref1, ref2 = first["Y"].clone(), second["Y"].clone()
    assert torch.isfinite(ref2.float()).all()

    def zero():
        first["Y"].fill_(0)
        second["Y"].fill_(0)
        torch.cuda.synchronize()

    def check():
        torch.cuda.synchronize()
        assert torch.equal(first["Y"].view(torch.int16), ref1.view(torch.int16))
        assert torch.equal(second["Y"].view(torch.int16), ref2.view(torch.int16))

    st = torch.cuda.Stream()
    for _ in range(3):
        zero()
        with torch.cuda.stream(st):
            run(first, st)
            run(second, st)
        check()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=st):
        run(first, st)
        run(second, st)
    for _ in range(2):
        zero()
        g.replay()
        check()
    del g
