"""The allocation-free W8A8 linear (convrot_linear_w8a8_noalloc).

It serves callers that may not allocate device memory: a plugin living inside
a framework that owns all of the GPU's memory and hands out no allocator, or a
path where an allocation (and the synchronization it can bring) is not
allowed.  Instead of a caller workspace it keeps the activation codes and
scales in a fixed array built into the library.  These checks call it through
the C ABI twice in a row, on different shapes, and compare each result with
the ordinary workspace-taking entry point; they also check that a request too
large for the built-in array is refused without a launch.  The file is named
so that pytest runs it last.
"""
import numpy as np
import pytest
import torch

from rotated_bit_quantized_block_b200 import binding as cr
from rotated_bit_quantized_block_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def _inputs(name, idx, with_bias):
    w = wl.WORKLOADS[name]
    X, W, b = wl.linear_inputs(w, idx, with_bias=with_bias)
    X, W = torch.from_numpy(X).cuda(), torch.from_numpy(W).cuda()
    b = None if b is None else torch.from_numpy(b).cuda()
    Wq, sw = cr.convrot_quantize_weight(W, w.block, 8, cr.CLIP_MSE)
    return w, X, Wq, sw, b


def test_noalloc_linear_matches_workspace_linear_two_calls_in_a_row():
    for name, idx, with_bias in (("vit_l_w8a8", 0, False), ("tiny_w8a8", 0, True)):
        w, X, Wq, sw, b = _inputs(name, idx, with_bias)
        ws = torch.empty(cr.convrot_workspace_bytes(X.shape[0], X.shape[1], 8), dtype=torch.uint8, device="cuda")
        y_ref = cr.convrot_linear_w8a8(X, Wq, sw, w.block, bias=b, workspace=ws)
        y = cr.convrot_linear_w8a8_noalloc(X, Wq, sw, w.block, bias=b)
        cr.convrot_device_status()
        a = y.cpu().numpy().astype(np.float64)
        r = y_ref.cpu().numpy().astype(np.float64)
        assert np.linalg.norm(a - r) <= 2e-3 * np.linalg.norm(r)
        assert np.array_equal(y.cpu().numpy().view(np.uint16), y_ref.cpu().numpy().view(np.uint16))


@pytest.mark.parametrize("M", [16, 1])
def test_noalloc_linear_few_tokens_two_calls_in_a_row(M):
    """Few tokens: 16 tokens take the feature-major GEMM with its K loop split
    across SMs, whose counters and int32 sum buffer then live in the built-in
    array too; one token takes the weight-streaming GEMM.  Two calls in a row
    (the split state must be zero again for the second) equal the workspace
    linear bit for bit."""
    K = N = 4096
    X = torch.from_numpy(wl.activations(M, K, 0.01, 30.0, seed=M)).cuda()
    W = torch.from_numpy(wl.weight(N, K, 0.01, seed=M + 1)).cuda()
    Wq, sw = cr.convrot_quantize_weight(W, 128, 8, cr.CLIP_MSE)
    plan = cr.convrot_linear_plan(M, K, N, 8, 128, 16 << 20)
    if M == 16:
        assert plan["gemm_kind"] == 1 and plan["k_splits"] > 1, plan
    else:
        assert plan["gemm_kind"] == 2, plan
    y_ref = cr.convrot_linear_w8a8(X, Wq, sw, 128)
    for _ in range(2):
        y = cr.convrot_linear_w8a8_noalloc(X, Wq, sw, 128)
        cr.convrot_device_status()
        assert np.array_equal(y.cpu().numpy().view(np.uint16), y_ref.cpu().numpy().view(np.uint16))


def test_noalloc_linear_refuses_more_than_its_array():
    lib = cr.load_library()
    M, K, N = 16384, 4096, 64  # 64 MiB of codes: beyond the 16 MiB array
    X = torch.zeros((M, K), dtype=torch.float16, device="cuda")
    Wq = torch.zeros((N, K), dtype=torch.int8, device="cuda")
    sw = torch.ones(N, dtype=torch.float32, device="cuda")
    Y = torch.full((M, N), 7.0, dtype=torch.float16, device="cuda")
    with pytest.raises(cr.ConvRotError) as err:
        cr.convrot_linear_w8a8_noalloc(X, Wq, sw, 128, Y=Y)
    assert err.value.status == cr.ERR_WORKSPACE
    assert b"16777216" in lib.convrot_last_error() or b"built-in" in lib.convrot_last_error()
    torch.cuda.synchronize()
    assert torch.all(Y == 7.0)  # nothing was launched
