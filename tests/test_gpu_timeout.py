"""Failure detection without a fault: a bounded device-side wait that runs out.

Every spin in the kernels (mbarrier phases, the fused prologue's flag words,
stream-K flags) is time-limited; when a limit passes, the kernel records a
timeout in the device status word, abandons its work and returns instead of
hanging or trapping.  These checks make such a wait run out on purpose through
a diagnostics entry point (a barrier nobody completes, a flag nobody raises,
with a 1 ms limit) and check that the call returns, that the status reports
CONVROT_ERR_TIMEOUT exactly once, and that the next linear on the device is
exact again.  (The trellis3d guide asks to tell fallback, out-of-memory and
NaN apart; a timeout is reported as its own status.)
"""
import numpy as np
import pytest
import torch

from rotated_bit_quantized_block_b200 import binding as cr
from rotated_bit_quantized_block_b200 import workloads as wl

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("kind", [0, 1])
def test_abandoned_wait_reports_timeout_once(kind):
    cr.convrot_device_status()  # start clean
    result = torch.full((4,), 7, dtype=torch.int32, device="cuda")
    cr.convrot_test_abandoned_wait(kind, 1_000_000, result)
    with pytest.raises(cr.ConvRotError) as err:
        cr.convrot_device_status()
    assert err.value.status == cr.ERR_TIMEOUT
    r = result.cpu().numpy()
    assert r[0] == 0 and r[1] == 1
    cr.convrot_device_status()  # reported once, then cleared
    # the context is usable: the fused linear equals the two-launch linear
    M, N, K = 640, 1024, 1024
    X = torch.from_numpy(wl.activations(M, K, 0.01, 30.0, seed=kind)).cuda()
    W = torch.from_numpy(wl.weight(N, K, 0.02, seed=kind + 1)).cuda()
    Wq, sw = cr.convrot_quantize_weight(W, 128, 8, cr.CLIP_MSE)
    y1 = cr.convrot_linear_w8a8_fused(X, Wq, sw, 128)
    ws = torch.empty(cr.convrot_workspace_bytes(M, K, 8), dtype=torch.uint8, device="cuda")
    cr.convrot_linear_quant_act(X, 128, 8, ws)
    y2 = cr.convrot_linear_gemm(ws, M, K, 8, Wq, sw)
    cr.convrot_device_status()
    assert np.array_equal(y1.cpu().numpy().view(np.uint16), y2.cpu().numpy().view(np.uint16))


def test_abandoned_wait_rejects_bad_arguments():
    result = torch.zeros(4, dtype=torch.int32, device="cuda")
    for kind, limit in ((2, 1_000_000), (0, 10), (1, 5_000_000_000)):
        with pytest.raises(cr.ConvRotError) as err:
            cr.convrot_test_abandoned_wait(kind, limit, result)
        assert err.value.status == cr.ERR_INVALID_ARG
