"""Seeded synthetic inputs shaped like DiT linear layers.

This module holds no arithmetic of the method itself: it only draws X, W, L_A
and L_B.  Both the CPU oracle's tests and the CUDA path consume exactly the
bf16 bit patterns it returns.

Recipe (numpy PCG64; the workload seed feeds a SeedSequence whose five
spawned children drive, in order, the channel scales, Z, W, L_A and L_B, so
the weights do not depend on the token count):

  c_j  ~ LogNormal(0, 1) per input channel; a fraction p_out of the channels,
         chosen without replacement, is multiplied by 10 (outlier channels:
         the RT-Lynx summary observes that only 5-10% of channels per token are
         strongly active)
  Z    ~ N(0, 1) of shape [M, D_in] (float32)
  X    = Z * c   (the MLP down-projection input is GELU(Z * c), exact erf form,
         so it is skewed towards non-negative values, with p_out = 0)
  W    ~ N(0, 1/D_in)  (variance 1/D_in)   [D_out, D_in]
  L_A  ~ 0.02 * N(0, 1)                    [D_out, R]
  L_B  ~ 0.02 * N(0, 1)                    [R, D_in]

Every tensor is rounded to bf16 with round-to-nearest-even.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    M: int          # tokens
    D_in: int       # K
    D_out: int      # N
    R: int          # LoRA rank
    p_out: float    # fraction of outlier channels
    seed: int
    gelu: bool = False

    @property
    def dense_equiv_flop(self) -> int:
        """2*M*D_in*D_out for the main product plus the rank-R LoRA FLOPs."""
        return 2 * self.M * self.D_in * self.D_out + 2 * self.M * self.R * (self.D_in + self.D_out)

    @property
    def dense_flop(self) -> int:
        return 2 * self.M * self.D_in * self.D_out


WORKLOADS = {
    "tiny": Workload("tiny", 128, 256, 256, 64, 0.08, 0),
    "qkv": Workload("qkv", 4096, 3072, 9216, 64, 0.08, 1),
    "mlp_up": Workload("mlp_up", 4608, 3072, 12288, 64, 0.05, 2),
    "mlp_down": Workload("mlp_down", 4608, 12288, 3072, 64, 0.0, 3, gelu=True),
    "video": Workload("video", 32760, 5120, 13824, 64, 0.06, 4),
}


def to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns (uint16), round to nearest even.  NaN is out of contract."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32)
    rounded = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return rounded.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _gelu_erf(v: np.ndarray) -> np.ndarray:
    from scipy.special import erf
    v64 = v.astype(np.float64)
    return (0.5 * v64 * (1.0 + erf(v64 / math.sqrt(2.0)))).astype(np.float32)


def make_inputs(wl: Workload, M: int | None = None, weights: bool = True):
    """Returns (X, W, L_A, L_B) as bf16 bit patterns (numpy uint16), C-contiguous.

    M overrides the token count while keeping the same per-channel scales and
    weights (the first M rows of Z are the same for any M).  With
    weights=False only X is drawn and W, L_A, L_B are None.
    """
    M = wl.M if M is None else M
    K, N, R = wl.D_in, wl.D_out, wl.R
    g_c, g_z, g_w, g_a, g_b = (np.random.Generator(np.random.PCG64(s))
                               for s in np.random.SeedSequence(wl.seed).spawn(5))
    c = g_c.lognormal(0.0, 1.0, size=K)
    n_out = int(round(wl.p_out * K))
    if n_out:
        idx = g_c.choice(K, n_out, replace=False)
        c[idx] *= 10.0
    c = c.astype(np.float32)
    Z = g_z.standard_normal((M, K), dtype=np.float32)
    X = Z * c
    if wl.gelu:
        X = _gelu_erf(X)
    if not weights:
        return to_bf16_bits(X), None, None, None
    W = g_w.standard_normal((N, K), dtype=np.float32) / np.float32(math.sqrt(K))
    L_A = np.float32(0.02) * g_a.standard_normal((N, R), dtype=np.float32)
    L_B = np.float32(0.02) * g_b.standard_normal((R, K), dtype=np.float32)
    return to_bf16_bits(X), to_bf16_bits(W), to_bf16_bits(L_A), to_bf16_bits(L_B)


def make_custom(M: int, K: int, N: int, R: int, seed: int, p_out: float = 0.08, gelu: bool = False):
    """Same recipe at an arbitrary shape (edge cases and ragged tails)."""
    return make_inputs(Workload("custom", M, K, N, R, p_out, seed, gelu))


def make_block_inputs(M: int, D: int, D_ff: int, R: int, seed: int, p_out: float = 0.05):
    """Inputs of a DiT feed-forward block (two layers): the up-projection's X,
    W_up [D_ff, D], LA_up, LB_up with the recipe above (seed), and the
    down-projection's W_down [D, D_ff], LA_down, LB_down drawn from seed + 100.
    The down-projection's input is produced by the block itself."""
    X, W_up, LA_up, LB_up = make_custom(M, D, D_ff, R, seed, p_out=p_out)
    _, W_down, LA_down, LB_down = make_custom(1, D_ff, D, R, seed + 100, p_out=0.0)
    return X, W_up, LA_up, LB_up, W_down, LA_down, LB_down
