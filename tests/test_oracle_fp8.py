"""Pins of the oracle's FP8 form of the layer, independent of the oracle's code.

The reading (the pages name FP8 only as future work that stacks with the
method): E4M3 codes (the OCP 8-bit float without infinities, max 448, ties
to even, saturating), W quantised per output channel with scale
max|W_n| / 448, S(X) per token with scale max|S(X)| / 448 (so the codes are
E4M3(x~ * 448 / max|x|)), the quantisation decisions taken in float32, and
Y = q_x q_w sum(x8 w8) + T L_A^T.

Independent references used here:
  - the E4M3 decoding written out below from the format's definition;
  - torch's float32 -> float8_e4m3fn cast (round to nearest even) for codes
    of magnitudes below 464, where torch does not saturate;
  - numpy float32 arithmetic for the per-channel and per-token scales;
  - a pure-Python brute-force sum on a tiny case;
  - a rigorous bound on the FP8 form's distance from the unquantised layer.
The last test plants mistakes in copies of the oracle's C source and checks
that these pins catch every one.
"""
import math
import os
import types

import numpy as np
import pytest

import oracle
from activation_sparse_gemm_b200.inputs import bf16_bits_to_f32, make_custom, to_bf16_bits

E4M3_MAX = 448.0


def e4m3_decode(c: int) -> float:
    """E4M3 from its definition: sign, 4-bit exponent with bias 7, 3-bit
    mantissa; exponent field 0 holds the subnormals m * 2^-9."""
    sign = -1.0 if c & 0x80 else 1.0
    e, m = (c >> 3) & 0xF, c & 7
    if e == 0:
        return sign * m * 2.0 ** -9
    return sign * (1.0 + m / 8.0) * 2.0 ** (e - 7)


def torch_e4m3(x):
    import torch
    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


FINITE_CODES = [c for c in range(256) if c not in (0x7F, 0xFF)]


def test_e4m3_every_code_roundtrips():
    for c in FINITE_CODES:
        v = e4m3_decode(c)
        assert oracle.e4m3(v) == c, hex(c)
    assert e4m3_decode(0x7E) == E4M3_MAX


def test_e4m3_matches_torch_cast_on_codes_midpoints_and_random_values():
    pos = np.array([e4m3_decode(c) for c in range(0x7F)])
    mids = (pos[:-1] + pos[1:]) / 2  # every tie between neighbouring codes
    rng = np.random.default_rng(11)
    x = np.concatenate([pos, -pos, mids, -mids, rng.uniform(-E4M3_MAX, E4M3_MAX, 20000),
                        rng.standard_normal(20000) * 0.02, rng.standard_normal(5000) * 1e-4]).astype(np.float32)
    ours = np.array([oracle.e4m3(float(v)) for v in x], np.uint8)
    assert (ours == torch_e4m3(x)).all()


def test_e4m3_closed_forms_and_saturation():
    assert oracle.e4m3(1.0) == 0x38 and oracle.e4m3(-1.0) == 0xB8
    assert oracle.e4m3(2.0 ** -6) == 0x08      # smallest normal
    assert oracle.e4m3(2.0 ** -9) == 0x01      # smallest subnormal
    assert oracle.e4m3(2.0 ** -10) == 0x00     # half of it: tie, to the even code 0
    assert oracle.e4m3(3 * 2.0 ** -10) == 0x02  # 1.5 steps: tie, to the even code 2
    assert oracle.e4m3(1 + 1 / 16) == 0x38     # tie between 1 and 1.125: even mantissa 0
    assert oracle.e4m3(1 + 3 / 16) == 0x3A     # tie between 1.125 and 1.25: even mantissa 2
    for v in (448.0, 460.0, 464.0, 470.0, 479.9, 480.0, 1000.0, 3e38):
        assert oracle.e4m3(v) == 0x7E and oracle.e4m3(-v) == 0xFE, v


def test_weight_quantisation_per_channel():
    rng = np.random.default_rng(3)
    N, K = 37, 96
    W = to_bf16_bits(rng.standard_normal((N, K)) * np.exp(rng.standard_normal((N, 1))))
    W[5] = 0  # an all-zero channel
    W8, qw = oracle.quantize_weight_fp8(W)
    Wf = bf16_bits_to_f32(W)
    b = np.abs(Wf).max(axis=1).astype(np.float32)
    with np.errstate(divide="ignore"):
        r = np.where(b > 0, np.float32(E4M3_MAX) / b, np.float32(0)).astype(np.float32)
    t = (Wf * r[:, None]).astype(np.float32)
    assert (W8 == torch_e4m3(t)).all()
    assert (qw == (b / np.float32(E4M3_MAX)).astype(np.float32)).all()
    assert (W8[5] == 0).all() and qw[5] == 0
    n_max = np.abs(Wf).argmax(axis=1)
    for n in range(N):
        if n != 5:
            assert W8[n, n_max[n]] & 0x7F == 0x7E  # the channel's largest entry is +-448


def test_sparsify_fp8_codes_and_token_scale():
    X, _, _, _ = make_custom(64, 128, 8, 8, seed=21)
    X[7] = 0  # an all-zero token
    meta, x8, s, qx = oracle.sparsify_fp8(X)
    rmeta, _, rs = oracle.sparsify(X)
    assert (meta == rmeta).all() and (s == rs).all()
    Xf = bf16_bits_to_f32(X)
    M, K = X.shape
    i0 = (meta & 3).astype(np.int64)
    i1 = (meta >> 2).astype(np.int64)
    base = 4 * np.arange(K // 4)[None, :]
    kept = np.empty((M, K // 2), np.float32)
    kept[:, 0::2] = np.take_along_axis(Xf, base + i0, axis=1)
    kept[:, 1::2] = np.take_along_axis(Xf, base + i1, axis=1)
    A = np.abs(Xf).max(axis=1).astype(np.float32)
    with np.errstate(divide="ignore"):
        r = np.where(A > 0, np.float32(E4M3_MAX) / A, np.float32(0)).astype(np.float32)
    assert (x8 == torch_e4m3((kept * r[:, None]).astype(np.float32))).all()
    assert np.allclose(qx, s.astype(np.float64) * A.astype(np.float64) / E4M3_MAX, rtol=0, atol=0)
    assert (x8[7] == 0).all() and qx[7] == 0
    # the token's largest magnitude is always kept, and lands on +-448
    assert ((x8 & 0x7F).max(axis=1)[A > 0] == 0x7E).all()


def test_linear_fp8_brute_force_tiny():
    M, K, N, R = 3, 16, 5, 4
    X, W, L_A, L_B = make_custom(M, K, N, R, seed=31)
    W8, qw = oracle.quantize_weight_fp8(W)
    meta, x8, s, qx = oracle.sparsify_fp8(X)
    Y = oracle.linear_fp8(X, W8, qw, L_A, L_B)
    Xf, Af, Bf = (bf16_bits_to_f32(a).astype(np.float64) for a in (X, L_A, L_B))
    for m in range(M):
        T = [sum(Xf[m, k] * Bf[r, k] for k in range(K)) for r in range(R)]
        for n in range(N):
            acc = 0.0
            for g in range(K // 4):
                ia, ib = int(meta[m, g]) & 3, int(meta[m, g]) >> 2
                acc += e4m3_decode(int(x8[m, 2 * g])) * e4m3_decode(int(W8[n, 4 * g + ia]))
                acc += e4m3_decode(int(x8[m, 2 * g + 1])) * e4m3_decode(int(W8[n, 4 * g + ib]))
            want = qx[m] * float(qw[n]) * acc + sum(T[r] * Af[n, r] for r in range(R))
            assert math.isclose(Y[m, n], want, rel_tol=1e-12, abs_tol=1e-12), (m, n)


def test_linear_fp8_within_quantisation_bound_of_exact_layer():
    """|Y_fp8 - Y| for Y = S(X) W^T + T L_A^T with S(X) = s x~ unrounded, bounded
    term by term: a normal code is within 2^-4 relative of its scaled value
    (three mantissa bits, nearest), a subnormal within 2^-10 absolute, and the
    float32 scale and product add at most 2^-22 relative."""
    M, K, N, R = 48, 256, 40, 16
    X, W, L_A, L_B = make_custom(M, K, N, R, seed=41)
    W8, qw = oracle.quantize_weight_fp8(W)
    meta, _, s, qx = oracle.sparsify_fp8(X)
    Y8 = oracle.linear_fp8(X, W8, qw, L_A, L_B)
    Xf, Wf = bf16_bits_to_f32(X).astype(np.float64), bf16_bits_to_f32(W).astype(np.float64)
    mask = np.zeros((M, K), bool)
    for g in range(K // 4):
        mask[np.arange(M), 4 * g + (meta[:, g] & 3)] = True
        mask[np.arange(M), 4 * g + (meta[:, g] >> 2)] = True
    S = np.where(mask, Xf * s[:, None].astype(np.float64), 0.0)
    T = Xf @ bf16_bits_to_f32(L_B).astype(np.float64).T
    Y = S @ Wf.T + T @ bf16_bits_to_f32(L_A).astype(np.float64).T
    eps = 2.0 ** -4 + 2.0 ** -22
    qwd = qw.astype(np.float64)
    ex = np.abs(S) * eps + qx[:, None] * 2.0 ** -10 * mask  # [M, K]
    ew = np.abs(Wf) * eps + qwd[:, None] * 2.0 ** -10      # [N, K]
    bound = ex @ (np.abs(Wf) + ew).T + np.abs(S) @ ew.T
    err = np.abs(Y8 - Y)
    assert (err <= bound * (1 + 1e-9) + 1e-12).all()
    rel = np.linalg.norm(Y8 - Y) / np.linalg.norm(Y)
    assert 1e-3 < rel < 0.08, rel  # quantisation happened, and stayed at FP8's precision


MUTANTS = {
    "round_toward_zero": ("(int)nearbyint(ldexp(m, 4)) - 8", "(int)trunc(ldexp(m, 4)) - 8"),
    "exponent_bias_8": ("(uint8_t)(((ex + 7) << 3) | q)", "(uint8_t)(((ex + 8) << 3) | q)"),
    "no_saturation": ("if (a >= 448.0) return sign | 0x7E;", "if (a >= 4480.0) return sign | 0x7E;"),
    "subnormal_step": ("(uint8_t)nearbyint(ldexp(a, 9))", "(uint8_t)nearbyint(ldexp(a, 8))"),
    "weight_scale_dropped": ("double y = qx * (double)qw[n] * acc;", "double y = qx * acc;"),
    "token_scale_without_s": ("*qx = (double)s * (double)A / 448.0;", "*qx = (double)A / 448.0;"),
    "weight_range_240": ("float r = b > 0.0f ? 448.0f / b : 0.0f;", "float r = b > 0.0f ? 240.0f / b : 0.0f;"),
    "second_code_from_first_index": ("x8[2 * g + 1] = e4m3_from_double((double)((float)x[i1] * r));",
                                     "x8[2 * g + 1] = e4m3_from_double((double)((float)x[i0] * r));"),
}

PINS = [
    test_e4m3_every_code_roundtrips,
    test_e4m3_matches_torch_cast_on_codes_midpoints_and_random_values,
    test_e4m3_closed_forms_and_saturation,
    test_weight_quantisation_per_channel,
    test_sparsify_fp8_codes_and_token_scale,
    test_linear_fp8_brute_force_tiny,
    test_linear_fp8_within_quantisation_bound_of_exact_layer,
]


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_fp8_pins_catch_mutant(name, tmp_path, monkeypatch):
    old, new = MUTANTS[name]
    src_path = os.path.join(os.path.dirname(oracle.__file__), "rtlynx_oracle.c")
    src = open(src_path).read()
    assert src.count(old) == 1, f"mutation site for {name} not found"
    mut = tmp_path / "mutant.c"
    mut.write_text(src.replace(old, new))
    o = oracle.Oracle(oracle.build(force=True, src=str(mut), out=str(tmp_path / "libmutant.so")))
    ns = types.SimpleNamespace(e4m3=o.e4m3, quantize_weight_fp8=o.quantize_weight_fp8,
                               sparsify_fp8=o.sparsify_fp8, linear_fp8=o.linear_fp8, sparsify=oracle.sparsify)
    monkeypatch.setitem(globals(), "oracle", ns)
    caught = []
    for pin in PINS:
        try:
            pin()
        except (AssertionError, ValueError, FloatingPointError):
            caught.append(pin.__name__)
    assert caught, f"no pin caught mutant {name}"
