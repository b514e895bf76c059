"""GPU parity of the FP8 (E4M3) form of the layer against the CPU oracle.

Both sides quantise identically (float32 decisions, nearest even,
saturating), so the codes of W and of the kept entries must agree bit for
bit, and so must the metadata.  q_x = s * max|x| / 448 is float32 on the GPU
and double in the oracle, and s itself may differ by 2 ulp (the single-layer
bar), so q_x is compared within 4 float32 ulp.  Y is compared with the
single-layer bars: the GEMM's products of codes are exact, and what remains
is the fp32 accumulation, the bf16 rounding of T / q_x and of L_A / q_w
(the LoRA term shares the FP8 accumulator) and the bf16 rounding of Y.
"""
import numpy as np
import pytest

import oracle
import activation_sparse_gemm_b200 as rl
from activation_sparse_gemm_b200.inputs import bf16_bits_to_f32, make_custom, make_inputs, to_bf16_bits, WORKLOADS

from tests.test_gpu_parity import assert_y_close, dev, host_bits, ulp_dist_f32

pytestmark = pytest.mark.gpu


def quantize_weight(W, L_A):
    import torch
    N, K = W.shape
    R = 0 if L_A is None else L_A.shape[1]
    W8 = torch.empty((N, K), dtype=torch.uint8, device="cuda")
    qw = torch.empty((N,), dtype=torch.float32, device="cuda")
    L_A8 = torch.empty((N, max(R, 1)), dtype=torch.bfloat16, device="cuda") if R else None
    rl.rtlynx_quantize_weight_fp8(dev(W), dev(L_A) if R else None, W8, qw, L_A8, N, K, R)
    assert rl.rtlynx_stream_status() == rl.OK
    torch.cuda.synchronize()
    return W8, qw, L_A8


def oracle_weights(W, W8_gpu, qw_gpu):
    """The oracle's quantised weights, asserted equal to the GPU's: every Y
    reference below is built from these, never from the GPU's."""
    rW8, rqw = oracle.quantize_weight_fp8(W)
    assert (W8_gpu == rW8).all(), "W8 codes differ from the oracle's"
    assert (qw_gpu == rqw).all(), "qw differs from the oracle's"
    return rW8, rqw


def run_fp8(X, W, L_A, L_B):
    import torch
    M, K = X.shape
    N = W.shape[0]
    R = 0 if L_A is None else L_B.shape[0]
    W8, qw, L_A8 = quantize_weight(W, L_A)
    Y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    rl.rtlynx_linear_fp8(dev(X), W8, qw, L_A8, dev(L_B) if R else None, Y, M, K, N, R)
    assert rl.rtlynx_stream_status() == rl.OK
    torch.cuda.synchronize()
    return host_bits(Y), W8.cpu().numpy(), qw.cpu().numpy(), (None if L_A8 is None else host_bits(L_A8))


def test_fp8_weight_preparation_matches_oracle():
    rng = np.random.default_rng(5)
    N, K, R = 72, 512, 16
    W = to_bf16_bits(rng.standard_normal((N, K)) * np.exp(rng.standard_normal((N, 1))))
    W[3] = 0  # an all-zero channel
    L_A = to_bf16_bits(rng.standard_normal((N, R)) * 0.02)
    W8, qw, L_A8 = quantize_weight(W, L_A)
    rW8, rqw = oracle.quantize_weight_fp8(W)
    assert (W8.cpu().numpy() == rW8).all()
    assert (qw.cpu().numpy() == rqw).all()
    qe = np.where(rqw > 0, rqw, np.float32(1)).astype(np.float32)
    want = to_bf16_bits((bf16_bits_to_f32(L_A) / qe[:, None]).astype(np.float32))
    assert (host_bits(L_A8) == want).all()


@pytest.mark.parametrize("M,K", [(200, 256), (129, 1024), (1, 512), (384, 3072)])
def test_fp8_sparsify_codes_match_oracle(M, K):
    import torch
    X, _, _, _ = make_custom(M, K, 8, 8, seed=900 + M)
    if M > 7:
        X[7] = 0  # an all-zero token
    codes = torch.empty((M, K // 2), dtype=torch.uint8, device="cuda")
    meta = torch.empty((M, K // 4), dtype=torch.uint8, device="cuda")
    qx = torch.empty((M,), dtype=torch.float32, device="cuda")
    rl.rtlynx_sparsify_fp8_debug(dev(X), M, K, codes, meta, qx)
    assert rl.rtlynx_stream_status() == rl.OK
    torch.cuda.synchronize()
    rmeta, rcodes, _, rqx = oracle.sparsify_fp8(X)
    assert (meta.cpu().numpy() == rmeta).all(), "metadata differs"
    assert (codes.cpu().numpy() == rcodes).all(), "codes differ"
    g = qx.cpu().numpy()
    assert (ulp_dist_f32(g, rqx.astype(np.float32)) <= 4).all(), "q_x differs by more than 4 float32 ulp"


@pytest.mark.parametrize("M,K,N,R", [(128, 256, 256, 64), (129, 512, 232, 16), (300, 1024, 520, 32),
                                     (64, 256, 8, 0), (256, 3072, 448, 64), (5000, 256, 224, 8),
                                     (513, 2048, 1000, 64)])
def test_fp8_linear_small(M, K, N, R):
    X, W, L_A, L_B = make_custom(M, K, N, R if R else 8, seed=950 + M + N)
    if R == 0:
        L_A = L_B = None
    Y, W8, qw, _ = run_fp8(X, W, L_A, L_B)
    rW8, rqw = oracle_weights(W, W8, qw)
    Y_ref = oracle.linear_fp8(X, rW8, rqw, L_A, L_B)
    assert_y_close(Y, Y_ref, f"fp8 {M}x{K}x{N} R={R}")


def test_fp8_qkv_shape_sampled():
    """The qkv workload's shape (4096 x 3072 -> 9216, R = 64): the GPU's weight
    codes and scales equal the oracle's on the whole W; Y on a whole 256-row
    band and 65 further tokens, against the oracle on the oracle's codes."""
    wl = WORKLOADS["qkv"]
    X, W, L_A, L_B = make_inputs(wl)
    Y, W8, qw, _ = run_fp8(X, W, L_A, L_B)
    rW8, rqw = oracle_weights(W, W8, qw)
    rng = np.random.default_rng(4)
    rows = sorted(set(list(range(0, 256)) + [4095] + rng.integers(0, wl.M, 64).tolist()))
    Y_ref = oracle.linear_fp8(X, rW8, rqw, L_A, L_B, rows=rows)
    assert_y_close(Y[rows], Y_ref, "fp8 qkv")
    # FP8 against the bf16 layer: the quantisation error itself, for the record
    Y16 = oracle.linear(X, W, L_A, L_B, rows=rows)
    rel = np.linalg.norm(Y_ref - Y16) / np.linalg.norm(Y16)
    assert rel < 0.08, rel


def test_fp8_rejects_bad_arguments():
    import torch
    X, W, L_A, L_B = make_custom(16, 384, 64, 8, seed=7)
    W8 = torch.empty((64, 384), dtype=torch.uint8, device="cuda")
    qw = torch.empty((64,), dtype=torch.float32, device="cuda")
    Y = torch.empty((16, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(rl.RtlynxError) as e:  # D_in not a multiple of 256
        rl.rtlynx_linear_fp8(dev(X), W8, qw, None, None, Y, 16, 384, 64, 0)
    assert e.value.status == rl.ERR_INVALID_ARG
    with pytest.raises(rl.RtlynxError) as e:  # LoRA factors missing for R > 0
        rl.rtlynx_quantize_weight_fp8(dev(W[:, :256].copy()), None, W8, qw, None, 64, 256, 8)
    assert e.value.status == rl.ERR_INVALID_ARG
