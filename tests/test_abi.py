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
    assert lib.rtlynx_linear(16, 16, 16, 16, 16, 4, 64, 64, 264, 0, None) == rl.ERR_UNSUPPORTED
    assert lib.rtlynx_linear(16, 16, 16, 16, 16, 4, 64, 64, 12, 0, None) == rl.ERR_UNSUPPORTED


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
