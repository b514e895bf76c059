"""Closed-form LoRA for the RT-Lynx layer (offline weight preparation).

The RT-Lynx summary page (four-step pipeline paragraph, step 2) trains the
rank-R LoRA so that it absorbs the sparsification residual: it minimises
||X W^T - S(X) W^T - X (L_A L_B)^T||^2 over calibration activations X.  For a
fixed calibration set this is a reduced-rank regression with a closed-form
optimum: with E = X W^T - S(X) W^T, the least-squares map B0 = argmin
||X B - E||, and V_R the top-R right singular vectors of X B0, the optimum is
C = V_R V_R^T B0^T, factored as L_A = V_R [D_out, R] and L_B = (B0 V_R)^T
[R, D_in].

This runs once per layer, before inference, and is not part of the layer's
call path.  The residual E comes from the layer itself (its dense-skip and
its sparse mode without LoRA, through the C ABI); the regression is float64
library linear algebra on the device (cuBLAS and cuSOLVER through torch).
"""
from __future__ import annotations

import activation_sparse_gemm_b200 as rl


def fit_lora(X, W, R: int, stream=None):
    """Fit L_A [D_out, R] and L_B [R, D_in] (bf16 device tensors) on the
    calibration tokens X [M, D_in] (bf16, device, M >= D_in so that X has full
    column rank) for the weight W [D_out, D_in] (bf16, device)."""
    import torch
    M, K = X.shape
    N = W.shape[0]
    if M < K:
        raise ValueError("the calibration set needs at least D_in tokens")
    if not 0 < R <= min(K, N):
        raise ValueError("R must be in 1 .. min(D_in, D_out)")
    dev = X.device
    Yd = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    Ys = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    rl.rtlynx_linear(X, W, None, None, Yd, M, K, N, 0, rl.MODE_DENSE_SKIP, stream)
    rl.rtlynx_linear(X, W, None, None, Ys, M, K, N, 0, rl.MODE_SPARSE, stream)
    status = rl.rtlynx_stream_status(stream)
    if status != rl.OK:
        raise rl.RtlynxError(status, "fit_lora")
    E = Yd.double() - Ys.double()
    Xd = X.double()
    G = Xd.T @ Xd                                     # [K, K], positive definite
    B0 = torch.cholesky_solve(Xd.T @ E, torch.linalg.cholesky(G))   # [K, N]
    Yhat = Xd @ B0                                    # [M, N]
    if M <= N:  # right singular vectors through the smaller Gram matrix
        lam, U = torch.linalg.eigh(Yhat @ Yhat.T)
        U = U[:, -R:].flip(1)
        sig = lam[-R:].flip(0).clamp_min(1e-300).sqrt()
        V = (Yhat.T @ U) / sig
    else:
        lam, V = torch.linalg.eigh(Yhat.T @ Yhat)
        V = V[:, -R:].flip(1)
    L_A = V.to(torch.bfloat16).contiguous()
    L_B = (B0 @ V).T.to(torch.bfloat16).contiguous()
    return L_A, L_B
