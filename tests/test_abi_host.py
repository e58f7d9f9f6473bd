"""Host-side checks of the C ABI: the library builds for sm_100a, loads, exports
every entry point that include/convrot.h declares, and rejects bad arguments
before touching the GPU.  No compute call is made here."""
import ctypes
import os
import re
import subprocess

import pytest

from rotated_bit_quantized_block_b200 import _build, binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"\b(convrot_[a-z0-9_]+)\s*\(", text))
    return names


@pytest.fixture(scope="module")
def lib():
    return binding.load_library()


def test_library_builds_for_sm100a_and_loads(lib):
    assert os.path.exists(_build.LIB_PATH)
    assert "arch=compute_100a,code=sm_100a" in " ".join(_build.NVCC_FLAGS)
    assert lib.convrot_version() >= 100


def test_every_declared_symbol_is_exported(lib):
    declared = declared_symbols()
    assert len(declared) >= 11
    out = subprocess.run(["nm", "-D", "--defined-only", _build.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r"\bT (convrot_[a-z0-9_]+)", out))
    assert declared <= exported, declared - exported
    for name in declared:
        assert hasattr(lib, name)
    assert set(binding.EXPORTED) <= declared


def test_status_strings(lib):
    for s in range(7):
        assert lib.convrot_status_string(s)
    assert lib.convrot_status_string(99) == b"unknown status"


def test_workspace_bytes(lib):
    assert lib.convrot_workspace_bytes(5184, 1024, 8) == 5184 * 1024 + ((5184 * 4 + 255) // 256) * 256
    assert lib.convrot_workspace_bytes(5184, 1024, 4) == 5184 * 1024 + ((5184 * 4 + 255) // 256) * 256
    assert lib.convrot_workspace_bytes(3, 128, 8) == 512 + 256
    assert lib.convrot_workspace_bytes(-1, 128, 8) == 0
    assert lib.convrot_workspace_bytes(4, 128, 5) == 0


P = ctypes.c_void_p
A16 = P(0x10000)      # aligned fake address, never dereferenced: validation fails first
MIS = P(0x10001)


@pytest.mark.parametrize("args,status", [
    # (N, K, block, bits, clip, dtype, W, Wq, scale)
    ((16, 100, 64, 8, 0, 0, A16, A16, A16), binding.ERR_INVALID_ARG),   # K not a multiple of 128
    ((16, 128, 3, 8, 0, 0, A16, A16, A16), binding.ERR_INVALID_ARG),    # block not a power of two
    ((16, 128, 512, 8, 0, 0, A16, A16, A16), binding.ERR_INVALID_ARG),  # block > 256
    ((16, 384, 256, 8, 0, 0, A16, A16, A16), binding.ERR_INVALID_ARG),  # block does not divide K
    ((16, 128, 64, 5, 0, 0, A16, A16, A16), binding.ERR_INVALID_ARG),   # bits
    ((16, 128, 64, 8, 7, 0, A16, A16, A16), binding.ERR_INVALID_ARG),   # clip mode
    ((16, 128, 64, 8, 0, 9, A16, A16, A16), binding.ERR_INVALID_ARG),   # dtype
    ((16, 128, 64, 8, 0, 0, None, A16, A16), binding.ERR_INVALID_ARG),  # null W
    ((16, 128, 64, 8, 0, 0, MIS, A16, A16), binding.ERR_ALIGNMENT),     # misaligned W
    ((-1, 128, 64, 8, 0, 0, A16, A16, A16), binding.ERR_INVALID_ARG),   # negative N
    ((16, 65536, 64, 8, 0, 0, A16, A16, A16), binding.ERR_INVALID_ARG),  # K too large
])
def test_quantize_weight_rejects_bad_arguments(lib, args, status):
    N, K, block, bits, clip, dtype, W, Wq, sc = args
    st = lib.convrot_quantize_weight(W, dtype, N, K, block, bits, clip, Wq, sc, None)
    assert st == status
    assert lib.convrot_last_error()


def test_zero_rows_are_a_noop(lib):
    assert lib.convrot_quantize_weight(None, 0, 0, 128, 64, 8, 0, None, None, None) == binding.OK
    assert lib.convrot_rotate_quant_act(None, 0, 128, 64, 8, None, None, None) == binding.OK
    assert lib.convrot_linear_w8a8(None, 0, 128, None, None, 16, None, 64, None, None, 0, None) == binding.OK
    assert lib.convrot_gemm_w4a4(None, None, 8, None, None, 0, 128, None, None, None, None) == binding.OK


def test_linear_rejects_small_workspace_and_bad_n(lib):
    st = lib.convrot_linear_w8a8(A16, 64, 256, A16, A16, 256, None, 64, A16, A16, 100, None)
    assert st == binding.ERR_WORKSPACE
    st = lib.convrot_linear_w8a8(A16, 64, 256, A16, A16, 250, None, 64, A16, A16, 1 << 20, None)
    assert st == binding.ERR_INVALID_ARG
    st = lib.convrot_linear_w4a4(MIS, 64, 256, A16, A16, 256, None, 64, A16, A16, 1 << 20, None)
    assert st == binding.ERR_ALIGNMENT
    st = lib.convrot_gemm_w8a8(A16, A16, 64, A16, A16, 256, 256, MIS, A16, None, None)
    assert st == binding.ERR_ALIGNMENT
    st = lib.convrot_rotate_quant_act(A16, 64, 256, 64, 8, MIS, A16, None)
    assert st == binding.ERR_ALIGNMENT


def test_binding_refuses_cpu_tensors():
    import torch
    with pytest.raises(ValueError):
        binding.convrot_rotate_quant_act(torch.zeros(4, 128, dtype=torch.float16), 64, 8)


def test_linear_workspace_bytes_adds_split_k_room(lib):
    ws, lws = lib.convrot_workspace_bytes, lib.convrot_linear_workspace_bytes
    for bits in (8, 4):
        for M, K, N in [(1, 4096, 4096), (16, 1024, 3072), (5184, 4096, 1024), (16384, 4096, 4096)]:
            assert lws(M, K, N, bits) >= ws(M, K, bits) + 2048
    # few tokens: the feature-major GEMM splits K over clusters of CTAs whose
    # partials meet in distributed shared memory, so only the counters
    assert lws(100, 4096, 1024, 8) == ws(100, 4096, 8) + 2048
    assert lws(16, 1024, 3072, 4) == ws(16, 1024, 4) + 2048
    # the weight-streaming kernel (one token) needs no split state beyond the counters
    assert lws(1, 4096, 4096, 8) == ws(1, 4096, 8) + 2048
    assert lws(8, 4096, 4096, 4) == ws(8, 4096, 4) + 2048
    # thousands of output tiles on CTA pairs: no split, only the counters
    assert lws(16384, 4096, 4096, 8) == ws(16384, 4096, 8) + 2048
    # token-major stream-K (deep K, a partly filled last round of 128 x 256 tiles):
    # one 128 x 256 int32 partial-tile slot per boundary between the 148 shares (+1)
    slots = 149 * 128 * 256 * 4
    assert lws(2500, 8192, 2000, 8) == ws(2500, 8192, 8) + 2048 + slots
    # W4A4 over more than 128 tokens: the int8-weight plan's split state, then
    # the weights widened to one int8 code per byte (N x K)
    assert lws(2500, 8192, 2000, 4) == ws(2500, 8192, 4) + 2048 + slots + 2000 * 8192
    assert lws(5184, 4096, 1024, 4) == ws(5184, 4096, 4) + 2048 + 1024 * 4096
    # shallow K (the shared tiles cost more than the idle SMs): whole tiles, counters only
    for K, N in [(1024, 3072), (1024, 1024), (1024, 4096)]:
        assert lws(5184, K, N, 8) == ws(5184, K, 8) + 2048
    assert lws(5184, 4096, 1024, 8) == ws(5184, 4096, 8) + 2048
    # a whole number of rounds of tiles (148 x 2 = 296 = 37 x 8 tiles): no stream-K
    assert lws(37 * 128, 8192, 8 * 256, 8) == ws(37 * 128, 8192, 8) + 2048
    assert lws(-1, 4096, 4096, 8) == 0
    assert lws(4, 4096, 4096, 5) == 0


def test_tensorwise_workspace_and_validation(lib):
    ws = lib.convrot_tensorwise_workspace_bytes
    assert ws(1000, 0) == 4096 + 256
    assert ws(1000, 1) == 4096 + 256 + ((1000 * 51 * 8 + 255) // 256) * 256
    assert ws(-1, 0) == 0 and ws(10, 7) == 0
    q = lib.convrot_quantize_weight_tensorwise
    assert q(None, 0, 0, 128, 64, 8, 1, None, None, None, 0, None) == binding.OK  # no rows: no-op
    assert q(A16, 0, 64, 256, 64, 8, 1, A16, A16, A16, 100, None) == binding.ERR_WORKSPACE
    assert q(A16, 0, 64, 256, 64, 8, 1, A16, A16, MIS, 1 << 20, None) == binding.ERR_ALIGNMENT
    assert q(A16, 0, 64, 256, 64, 8, 3, A16, A16, A16, 1 << 20, None) == binding.ERR_INVALID_ARG
    assert q(A16, 0, 64, 100, 64, 8, 0, A16, A16, A16, 1 << 20, None) == binding.ERR_INVALID_ARG
