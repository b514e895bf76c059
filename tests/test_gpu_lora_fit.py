"""GPU check of the closed-form LoRA fit (activation_sparse_gemm_b200.lora_fit)
against the oracle's reduced-rank regression.

The factors themselves are not unique (any invertible R x R map between them
gives the same product), so the test compares what is: the value of the
objective ||X W^T - S(X) W^T - X (L_A L_B)^T||^2 on the calibration tokens,
evaluated exactly by the oracle.  The fit's residual target comes from the
layer's bf16 outputs and its factors are rounded to bf16, so it may sit a
little above the oracle's float64 optimum, never meaningfully below it."""
import numpy as np
import pytest

import oracle
import activation_sparse_gemm_b200 as rl
from activation_sparse_gemm_b200.inputs import make_custom

from tests.test_gpu_parity import dev, host_bits

pytestmark = pytest.mark.gpu


def f64(bits):
    return oracle.bf16_to_f64(bits)


@pytest.mark.parametrize("M,K,N,R", [(1024, 256, 320, 16), (600, 128, 96, 32)])
def test_fit_reaches_the_closed_form_optimum(M, K, N, R):
    from activation_sparse_gemm_b200.lora_fit import fit_lora
    X, W, _, _ = make_custom(M, K, N, R, seed=1100 + M, p_out=0.05)
    L_A, L_B = fit_lora(dev(X), dev(W), R)
    A, B = f64(host_bits(L_A)), f64(host_bits(L_B))
    A_o, B_o, E = oracle.lora_fit(X, W, R)
    Xf = f64(X)
    obj = float(np.linalg.norm(Xf @ (A @ B).T - E) ** 2)
    opt = float(np.linalg.norm(Xf @ (A_o @ B_o).T - E) ** 2)
    e2 = float(np.linalg.norm(E) ** 2)
    assert opt < e2
    assert obj >= opt - 1e-9 * e2
    assert obj <= opt * (1 + 1e-3) + 1e-6 * e2, (obj, opt, e2)
    # through the layer: the fitted LoRA moves the sparse layer toward the dense one
    Yd = oracle.linear(X, W, mode=oracle.MODE_DENSE_SKIP)
    import torch
    Y0 = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    Y1 = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    rl.rtlynx_linear(dev(X), dev(W), None, None, Y0, M, K, N, 0, rl.MODE_SPARSE)
    rl.rtlynx_linear(dev(X), dev(W), L_A, L_B, Y1, M, K, N, R, rl.MODE_SPARSE)
    assert rl.rtlynx_stream_status() == rl.OK
    e_none = np.linalg.norm(f64(host_bits(Y0)) - Yd)
    e_fit = np.linalg.norm(f64(host_bits(Y1)) - Yd)
    assert e_fit < e_none
