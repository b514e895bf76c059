"""rtlynx_linear_noalloc: the entry point for callers that cannot allocate
device memory (their memory belongs to another pool, or the call sits on a
path where cudaMalloc's possible device synchronization is not acceptable).

Its results must equal those of rtlynx_linear on the same inputs, call after
call, even though every call reuses the same static workspace array.  This
file is collected last so that a run stopping at its first failure has run
every other test already; it also passes on its own in a fresh process.
"""
import numpy as np
import pytest

import activation_sparse_gemm_b200 as rl
from activation_sparse_gemm_b200.inputs import WORKLOADS, bf16_bits_to_f32, make_custom, make_inputs

pytestmark = pytest.mark.gpu


def _dev(bits):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _bits(t):
    import torch
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def _both(X, W, L_A, L_B, mode):
    """Y from rtlynx_linear and from rtlynx_linear_noalloc, plus the device status word."""
    import torch
    M, K = X.shape
    N = W.shape[0]
    R = L_B.shape[0] if (mode == rl.MODE_SPARSE and L_B is not None) else 0
    Xd, Wd = _dev(X), _dev(W)
    Ad = _dev(L_A) if R else None
    Bd = _dev(L_B) if R else None
    Y_ref = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    Y_na = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    rl.rtlynx_linear(Xd, Wd, Ad, Bd, Y_ref, M, K, N, R, mode)
    rl.rtlynx_linear_noalloc(Xd, Wd, Ad, Bd, Y_na, M, K, N, R, mode, status)
    torch.cuda.synchronize()
    assert rl.rtlynx_stream_status() == rl.OK
    return _bits(Y_ref), _bits(Y_na), int(status.item())


def test_noalloc_matches_linear_on_consecutive_calls():
    # two different problems back to back, then the first again: the shared
    # static workspace keeps stale data from the previous call
    cases = [make_custom(300, 512, 264, 32, seed=41), make_inputs(WORKLOADS["tiny"]),
             make_custom(300, 512, 264, 32, seed=41)]
    for X, W, L_A, L_B in cases:
        ref, got, status = _both(X, W, L_A, L_B, rl.MODE_SPARSE)
        assert status == 0
        assert np.array_equal(ref, got), "noalloc output differs from rtlynx_linear"
        assert np.isfinite(bf16_bits_to_f32(got)).all()


def test_noalloc_split_tail_tickets_reused():
    """Shapes whose GEMM cuts its last tiles along K, so that the fp32 partials
    and the arrival tickets of the split tiles live in the shared static array:
    two different split shapes back to back, then the first again, each equal
    bit for bit to rtlynx_linear (which uses its own workspace)."""
    import torch
    shapes = [(2560, 1024, 2160, 64), (2560, 2048, 1920, 64), (2560, 1024, 2160, 64)]
    if torch.cuda.get_device_properties(0).multi_processor_count == 148:
        for M, K, N, R in shapes[:2]:
            s = rl.rtlynx_schedule_info(M, K, N, R, 148)
            assert s.tail_units > 0, (M, K, N)  # the shape really splits
    for M, K, N, R in shapes:
        assert rl.rtlynx_workspace_size(M, K, N, R, rl.MODE_SPARSE) <= rl.NOALLOC_MAX_BYTES
        X, W, L_A, L_B = make_custom(M, K, N, R, seed=60 + K + N)
        ref, got, status = _both(X, W, L_A, L_B, rl.MODE_SPARSE)
        assert status == 0
        assert np.array_equal(ref, got), f"noalloc output differs from rtlynx_linear at {M}x{K}x{N}"


def test_noalloc_without_status_word():
    """With no caller status word, a timeout would go to the library's own
    error word: the call still allocates nothing, its output equals
    rtlynx_linear's, and rtlynx_stream_status reports OK."""
    import torch
    X, W, L_A, L_B = make_custom(300, 512, 264, 32, seed=43)
    M, K = X.shape
    N, R = W.shape[0], L_B.shape[0]
    Xd, Wd, Ad, Bd = _dev(X), _dev(W), _dev(L_A), _dev(L_B)
    Y_ref = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    Y_na = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    rl.rtlynx_linear(Xd, Wd, Ad, Bd, Y_ref, M, K, N, R, rl.MODE_SPARSE)
    rl.rtlynx_linear_noalloc(Xd, Wd, Ad, Bd, Y_na, M, K, N, R, rl.MODE_SPARSE, None)
    assert rl.rtlynx_stream_status() == rl.OK
    assert np.array_equal(_bits(Y_ref), _bits(Y_na))


def test_noalloc_dense_skip_and_no_lora():
    X, W, L_A, L_B = make_custom(129, 256, 136, 16, seed=42)
    for mode, la, lb in ((rl.MODE_DENSE_SKIP, None, None), (rl.MODE_SPARSE, None, None)):
        ref, got, status = _both(X, W, la, lb, mode)
        assert status == 0
        assert np.array_equal(ref, got)


def test_noalloc_rejects_workspace_beyond_limit():
    import torch
    M, K, N, R = 8192, 4096, 64, 64
    assert rl.rtlynx_workspace_size(M, K, N, R, rl.MODE_SPARSE) > rl.NOALLOC_MAX_BYTES
    X = torch.zeros((M, K), dtype=torch.bfloat16, device="cuda")
    W = torch.zeros((N, K), dtype=torch.bfloat16, device="cuda")
    A = torch.zeros((N, R), dtype=torch.bfloat16, device="cuda")
    B = torch.zeros((R, K), dtype=torch.bfloat16, device="cuda")
    Y = torch.zeros((M, N), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(rl.RtlynxError) as ei:
        rl.rtlynx_linear_noalloc(X, W, A, B, Y, M, K, N, R, rl.MODE_SPARSE)
    assert ei.value.status == rl.ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert (Y == 0).all()  # nothing was launched
