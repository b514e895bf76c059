"""CPU-only checks of the C ABI library: it loads, exports every symbol the
public header declares, and rejects bad arguments before touching a GPU."""
import ctypes
import glob
import os
import re
import subprocess

import pytest

import activation_sparse_gemm_b200 as rl
from activation_sparse_gemm_b200 import build as rl_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    rl_build.build()
    return rl.lib()


def declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names |= set(re.findall(r"\b(rtlynx_\w+)\s*\(", text))
    return names


def test_header_declares_the_binding_names():
    assert declared_functions() == set(rl.ABI_SYMBOLS)


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.check_output(["nm", "-D", "--defined-only", rl.LIB_PATH]).decode()
    exported = set(re.findall(r"\s[TW]\s+(rtlynx_\w+)$", out, flags=re.M))
    for name in declared_functions():
        assert name in exported, name
        assert hasattr(lib, name)


def test_status_strings(lib):
    assert rl.rtlynx_status_string(rl.OK) == "ok"
    assert "timed out" in rl.rtlynx_status_string(rl.ERR_DEVICE_TIMEOUT)
    assert rl.rtlynx_status_string(99) == "unknown status"


@pytest.mark.parametrize("M,K,N,R,mode", [
    (0, 64, 64, 0, 0),      # empty token dimension
    (16, 0, 64, 0, 0),
    (16, 64, 0, 0, 0),
    (16, 60, 64, 0, 0),     # D_in not a multiple of 8
    (16, 64, 60, 0, 0),     # D_out not a multiple of 8
    (16, 64, 64, -1, 0),
    (16, 64, 64, 0, 7),     # unknown mode
])
def test_invalid_sizes_rejected_without_launch(lib, M, K, N, R, mode):
    st = lib.rtlynx_linear(16, 16, 16, 16, 16, M, K, N, R, mode, None)
    assert st == rl.ERR_INVALID_ARG


def test_null_and_misaligned_pointers_rejected(lib):
    assert lib.rtlynx_linear(None, 16, None, None, 16, 4, 64, 64, 0, 0, None) == rl.ERR_INVALID_ARG
    assert lib.rtlynx_linear(24, 16, None, None, 16, 4, 64, 64, 0, 0, None) == rl.ERR_INVALID_ARG
    # sparse mode with a LoRA rank but no LoRA factors
    assert lib.rtlynx_linear(16, 16, None, None, 16, 4, 64, 64, 64, 0, None) == rl.ERR_INVALID_ARG


def test_unsupported_rank_rejected(lib):
    X, W, A, B, Y = 1 << 20, 2 << 20, 3 << 20, 4 << 20, 5 << 20  # distinct, far apart
    assert lib.rtlynx_linear(X, W, A, B, Y, 4, 64, 64, 264, 0, None) == rl.ERR_UNSUPPORTED
    assert lib.rtlynx_linear(X, W, A, B, Y, 4, 64, 64, 12, 0, None) == rl.ERR_UNSUPPORTED


@pytest.mark.parametrize("entry", ["linear", "ws", "noalloc", "host"])
def test_output_overlapping_an_input_rejected(lib, entry):
    """Y sharing a byte with X, W, L_A or L_B is rejected before anything runs
    (the pointers are never dereferenced, so fake addresses do)."""
    M, K, N, R = 4, 64, 32, 16
    base = {"X": 1 << 20, "W": 2 << 20, "L_A": 3 << 20, "L_B": 4 << 20}
    sizes = {"X": 2 * M * K, "W": 2 * N * K, "L_A": 2 * N * R, "L_B": 2 * R * K}

    def call(Y, args):
        if entry == "linear":
            return lib.rtlynx_linear(args["X"], args["W"], args["L_A"], args["L_B"], Y, M, K, N, R, 0, None)
        if entry == "ws":
            return lib.rtlynx_linear_ws(args["X"], args["W"], args["L_A"], args["L_B"], Y, M, K, N, R, 0, 1 << 30,
                                        1 << 20, None)
        if entry == "noalloc":
            return lib.rtlynx_linear_noalloc(args["X"], args["W"], args["L_A"], args["L_B"], Y, M, K, N, R, 0, None,
                                             None)
        return lib.rtlynx_linear_host(1 << 31, args["W"], args["L_A"], args["L_B"], 3 << 30, M, K, N, R, 0,
                                      args["X"], Y, None)

    for name, addr in base.items():
        # Y's last 16 bytes on the input's first 16, and Y starting on the input's last 16
        y_bytes = 2 * M * N
        for Y in (addr - y_bytes + 16, addr + sizes[name] - 16):
            assert call(Y, base) == rl.ERR_INVALID_ARG, (entry, name, Y)


def test_fp8_output_overlapping_an_input_rejected(lib):
    M, K, N, R = 4, 256, 32, 16
    X, W8, qw, A8, B = 1 << 20, 2 << 20, 3 << 20, 4 << 20, 5 << 20
    for Y in (X + 2 * M * K - 16, W8 + N * K - 16, qw, A8 + 16, B):
        assert lib.rtlynx_linear_fp8(X, W8, qw, A8, B, Y, M, K, N, R, None) == rl.ERR_INVALID_ARG


def test_python_binding_raises_on_error(lib):
    with pytest.raises(rl.RtlynxError) as ei:
        rl.rtlynx_linear(16, 16, 16, 16, 16, 0, 64, 64, 0, 0, stream=0)
    assert ei.value.status == rl.ERR_INVALID_ARG


def test_workspace_size_zero_for_dense_and_invalid(lib):
    assert rl.rtlynx_workspace_size(128, 256, 256, 64, rl.MODE_DENSE_SKIP) == 0
    assert rl.rtlynx_workspace_size(128, 250, 256, 64, rl.MODE_SPARSE) == 0


def test_wait_selftest_rejects_bad_limits_without_launch(lib):
    for limit in (0, -1, 2_000_000_000):
        assert lib.rtlynx_wait_selftest(limit, None) == rl.ERR_INVALID_ARG


@pytest.mark.parametrize("M,K,N,R", [
    (0, 256, 64, 0),      # no tokens
    (4, 384, 64, 0),      # D_in not a multiple of 256 (whole FP8 stages)
    (4, 250, 64, 0),
    (4, 256, 60, 0),      # D_out not a multiple of 8
    (4, 256, 64, -8),
])
def test_fp8_invalid_sizes_rejected_without_launch(lib, M, K, N, R):
    assert lib.rtlynx_linear_fp8(16, 16, 16, 16, 16, 16, M, K, N, R, None) == rl.ERR_INVALID_ARG
    if M > 0:  # the weight preparation has no token count
        assert lib.rtlynx_quantize_weight_fp8(16, 16, 16, 16, 16, N, K, R, None) == rl.ERR_INVALID_ARG


def test_fp8_pointers_and_rank_rejected(lib):
    # null, misaligned, and a LoRA rank without the LoRA factors
    assert lib.rtlynx_linear_fp8(None, 16, 16, None, None, 16, 4, 256, 64, 0, None) == rl.ERR_INVALID_ARG
    assert lib.rtlynx_linear_fp8(24, 16, 16, None, None, 16, 4, 256, 64, 0, None) == rl.ERR_INVALID_ARG
    assert lib.rtlynx_linear_fp8(16, 16, 16, None, None, 16, 4, 256, 64, 64, None) == rl.ERR_INVALID_ARG
    assert lib.rtlynx_linear_fp8(16, 16, 16, 16, 16, 16, 4, 256, 64, 12, None) == rl.ERR_UNSUPPORTED
    assert lib.rtlynx_linear_fp8(16, 16, 16, 16, 16, 16, 4, 256, 64, 264, None) == rl.ERR_UNSUPPORTED
    assert lib.rtlynx_quantize_weight_fp8(16, None, 16, 16, None, 64, 256, 8, None) == rl.ERR_INVALID_ARG
    assert lib.rtlynx_sparsify_fp8_debug(16, 4, 384, None, None, None, None) == rl.ERR_INVALID_ARG
