"""Pins for the CPU oracle: facts fixed by the RT-Lynx definition and by mathematics.

The pages (RT-Lynx summary, four-step pipeline paragraph, steps 1-3) print no
worked numbers, so the oracle is pinned by: a hand-worked example, exhaustive
brute force of the 2-of-4 rule against an independent rule, exact-arithmetic
recomputation of s and of the bf16 rounding, closed-form bounds, special cases
that reduce to a textbook GEMM, and symmetries.
"""
import itertools
import json
import math
import os
from decimal import Decimal, getcontext
from fractions import Fraction

import numpy as np
import pytest

import oracle
from activation_sparse_gemm_b200.inputs import (WORKLOADS, bf16_bits_to_f32, make_custom, make_inputs,
                                                to_bf16_bits)

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
VALID_META = {0x4, 0x8, 0xC, 0x9, 0xD, 0xE}
getcontext().prec = 80


# ----------------------------------------------------------------------------- exact helpers
def f32_bits_value(bits: int) -> Fraction:
    return Fraction(float(np.uint32(bits).view(np.float32)))


def bf16_value(bits: int) -> Fraction:
    return Fraction(float(bf16_bits_to_f32(np.array([bits], np.uint16))[0]))


def nearest_bf16_bits(v: Fraction) -> int:
    """Nearest bf16 to an exact rational, ties to an even significand, by search."""
    approx = np.float32(float(v))
    centre = int(approx.view(np.uint32)) >> 16
    cands = []
    for b in range(max(0, centre - 3), centre + 4):
        for sign in (0, 0x8000):
            bits = (b & 0x7FFF) | sign
            if (bits & 0x7F80) == 0x7F80:  # inf / nan
                continue
            cands.append(bits)
    best = min(cands, key=lambda b: (abs(bf16_value(b) - v), b & 1))
    # normalise the sign of a zero result to the sign of v
    if bf16_value(best) == 0:
        return 0x8000 if v < 0 else 0
    return best


def nearest_f32(d: Decimal) -> np.float32:
    """Nearest float32 to a high-precision decimal, ties to even, by search."""
    v = Fraction(d)
    approx = np.float32(float(d))
    bits = int(approx.view(np.uint32))
    cands = [b for b in range(max(0, bits - 3), bits + 4)]
    best = min(cands, key=lambda b: (abs(f32_bits_value(b) - v), b & 1))
    return np.uint32(best).view(np.float32)


def expected_val_bits(s32, x) -> int:
    """bf16 bits of s*x rounded once from the exact product; a zero keeps the
    IEEE sign of the product."""
    s32, x = float(s32), float(x)
    if x == 0.0 or s32 == 0.0:
        neg = math.copysign(1.0, x) * math.copysign(1.0, s32) < 0
        return 0x8000 if neg else 0
    return nearest_bf16_bits(Fraction(s32) * Fraction(x))


def exact_s(xs) -> np.float32:
    """s = ||x|| / (||x~|| + 1e-8) from the exact sums, rounded once to float32."""
    xs = [Fraction(float(x)) for x in xs]
    nx = sum(x * x for x in xs)
    nt = Fraction(0)
    for g in range(len(xs) // 4):
        grp = xs[4 * g:4 * g + 4]
        i0, i1 = energy_rule(grp)
        nt += grp[i0] ** 2 + grp[i1] ** 2
    dn = Decimal(nx.numerator) / Decimal(nx.denominator)
    dt = Decimal(nt.numerator) / Decimal(nt.denominator)
    return nearest_f32(dn.sqrt() / (dt.sqrt() + Decimal(1e-8)))


def energy_rule(grp):
    """Independent 2-of-4 rule: the pair with the largest x_i^2 + x_j^2 (exact
    rationals), lexicographically smallest pair on ties."""
    best = None
    for i, j in itertools.combinations(range(4), 2):
        a = grp[i] if isinstance(grp[i], Fraction) else Fraction(float(grp[i]))
        b = grp[j] if isinstance(grp[j], Fraction) else Fraction(float(grp[j]))
        e = a * a + b * b
        if best is None or e > best[0]:
            best = (e, i, j)
    return best[1], best[2]


def decode_dense(meta, vals, K):
    """Dense S(X) (float64) from metadata nibbles and kept values."""
    M = meta.shape[0]
    G = K // 4
    S = np.zeros((M, G, 4), np.float64)
    v = bf16_bits_to_f32(vals).astype(np.float64).reshape(M, G, 2)
    i0 = (meta & 3).astype(np.int64)[..., None]
    i1 = ((meta >> 2) & 3).astype(np.int64)[..., None]
    np.put_along_axis(S, i0, v[..., 0:1], axis=2)
    np.put_along_axis(S, i1, v[..., 1:2], axis=2)
    return S.reshape(M, K)


def f64(bits):
    return bf16_bits_to_f32(bits).astype(np.float64)


# ----------------------------------------------------------------------------- hand-worked example
def test_worked_example():
    ex = json.load(open(os.path.join(GOLDEN, "worked_example.json")))
    x = np.array(ex["x"], np.float32)
    X = to_bf16_bits(x)[None, :]
    meta, vals, s = oracle.sparsify(X)
    assert meta[0].tolist() == ex["meta"]
    nx = Fraction(ex["nx_num"], ex["nx_den"])
    nt = Fraction(ex["nt_num"], ex["nt_den"])
    assert sum(Fraction(float(v)) ** 2 for v in x) == nx
    s_ref = nearest_f32(Decimal(nx.numerator / nx.denominator).sqrt()
                        / (Decimal(nt.numerator / nt.denominator).sqrt() + Decimal(1e-8)))
    assert s[0] == s_ref
    for i, k in enumerate(ex["kept_unscaled"]):
        assert vals[0, i] == expected_val_bits(s_ref, k)


# ----------------------------------------------------------------------------- mask brute force
ALPHABET = [-2.0, -1.0, -0.0, 0.0, 1.0, 2.0, 2.0 ** -133, 0.5]


def test_mask_bruteforce_small_alphabet():
    groups = list(itertools.product(ALPHABET, repeat=4))
    X = to_bf16_bits(np.array(groups, np.float32))          # [4096, 4], one group per token
    meta, vals, s = oracle.sparsify(X)
    for r, grp in enumerate(groups):
        i0, i1 = energy_rule(grp)
        assert meta[r, 0] == (i0 | (i1 << 2)), (grp, meta[r, 0])
        assert meta[r, 0] in VALID_META
        assert s[r] == exact_s(grp), (grp, s[r])
        for slot, idx in enumerate((i0, i1)):
            want = expected_val_bits(s[r], grp[idx])
            assert vals[r, slot] == want, (grp, slot)


def test_mask_random_rows_exact_s():
    X, _, _, _ = make_custom(24, 64, 8, 16, seed=11)
    meta, vals, s = oracle.sparsify(X)
    xf = bf16_bits_to_f32(X)
    for r in range(X.shape[0]):
        assert s[r] == exact_s(xf[r])
        for g in range(16):
            i0, i1 = energy_rule(list(xf[r, 4 * g:4 * g + 4]))
            assert meta[r, g] == (i0 | (i1 << 2))
            assert vals[r, 2 * g] == expected_val_bits(s[r], xf[r, 4 * g + i0])
            assert vals[r, 2 * g + 1] == expected_val_bits(s[r], xf[r, 4 * g + i1])


# ----------------------------------------------------------------------------- invariants on the workloads
@pytest.mark.parametrize("name", list(WORKLOADS))
def test_invariants_on_workload_distributions(name):
    wl = WORKLOADS[name]
    X, _, _, _ = make_inputs(wl, M=min(wl.M, 48), weights=False)
    meta, vals, s = oracle.sparsify(X)
    M, K = X.shape
    xf = f64(X)
    assert set(np.unique(meta).tolist()) <= VALID_META
    i0 = meta & 3
    i1 = (meta >> 2) & 3
    assert (i0 < i1).all()
    mag = np.abs(xf.reshape(M, K // 4, 4))
    kept = np.zeros_like(mag, dtype=bool)
    np.put_along_axis(kept, i0[..., None].astype(np.int64), True, axis=2)
    np.put_along_axis(kept, i1[..., None].astype(np.int64), True, axis=2)
    assert (kept.sum(axis=2) == 2).all()
    min_kept = np.where(kept, mag, np.inf).min(axis=2)
    max_dropped = np.where(kept, -np.inf, mag).max(axis=2)
    assert (min_kept >= max_dropped).all()
    # closed form: the two largest squares hold at least half of a group's energy
    nz = np.abs(xf).sum(axis=1) > 0
    assert (s[nz] >= np.float32(1.0)).all()
    assert (s[nz] <= np.float32(math.sqrt(2.0)) * np.float32(1 + 2.0 ** -23)).all()
    # norm preservation up to the bf16 rounding of the kept values
    S = decode_dense(meta, vals, K)
    nS = np.linalg.norm(S, axis=1)
    nX = np.linalg.norm(xf, axis=1)
    assert (np.abs(nS - nX) <= 2.0 ** -8 * nX + 1e-8).all()
    if name == "mlp_down":
        assert (xf.mean() > 0) and (xf.min() > -0.2)


def test_zero_groups_and_zero_rows():
    X, W, L_A, L_B = make_custom(6, 32, 16, 16, seed=3)
    xf = bf16_bits_to_f32(X).copy()
    xf[0, 4:8] = 0.0                 # one all-zero group
    xf[1, 8:12] = [0.0, -0.0, 0.0, -0.0]
    xf[2, :] = 0.0                   # an all-zero token
    X = to_bf16_bits(xf)
    meta, vals, s = oracle.sparsify(X)
    assert meta[0, 1] == 0x4 and (f64(vals[0, 2:4]) == 0).all()
    assert meta[1, 2] == 0x4 and (f64(vals[1, 4:6]) == 0).all()
    assert s[2] == 0.0 and (f64(vals[2]) == 0).all()
    Y = oracle.linear(X, W, L_A, L_B)
    assert (Y[2] == 0).all()


# ----------------------------------------------------------------------------- special cases
def test_already_two_of_four_reduces_to_textbook_gemm():
    rng = np.random.default_rng(5)
    X, W, _, _ = make_custom(32, 64, 40, 16, seed=9)
    xf = bf16_bits_to_f32(X).copy()
    for m in range(xf.shape[0]):
        for g in range(16):
            drop = rng.choice(4, 2, replace=False)
            xf[m, 4 * g + drop] = 0.0
    X = to_bf16_bits(xf)
    meta, vals, s = oracle.sparsify(X)
    assert (s == np.float32(1.0)).all()           # ||x|| > 0.34 on every row here
    S = decode_dense(meta, vals, 64)
    assert (S == f64(X)).all()
    Y = oracle.linear(X, W)
    ref = f64(X) @ f64(W).T
    np.testing.assert_allclose(Y, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())


def test_lora_zero_gives_sparse_branch_exactly():
    X, W, L_A, L_B = make_custom(16, 128, 48, 32, seed=4)
    Y0 = oracle.linear(X, W)
    Y1 = oracle.linear(X, W, np.zeros_like(L_A), L_B)
    Y2 = oracle.linear(X, W, L_A, np.zeros_like(L_B))
    assert (Y0 == Y1).all() and (Y0 == Y2).all()


def test_dense_skip_is_textbook_gemm():
    X, W, L_A, L_B = make_custom(20, 96, 56, 16, seed=6)
    Y = oracle.linear(X, W, L_A, L_B, mode=oracle.MODE_DENSE_SKIP)
    ref = f64(X) @ f64(W).T
    np.testing.assert_allclose(Y, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())


def test_brute_force_tiny_against_numpy():
    X, W, L_A, L_B = make_custom(12, 64, 24, 16, seed=7)
    meta, vals, s = oracle.sparsify(X)
    S = decode_dense(meta, vals, 64)
    Y, T = oracle.linear(X, W, L_A, L_B, want_T=True)
    xf, wf, af, bf = f64(X), f64(W), f64(L_A), f64(L_B)
    ref = S @ wf.T + xf @ (af @ bf).T
    np.testing.assert_allclose(Y, ref, rtol=1e-11, atol=1e-12 * np.abs(ref).max())
    np.testing.assert_allclose(T, xf @ bf.T, rtol=1e-12, atol=1e-14)
    # the two LoRA routes agree: (X L_B^T) L_A^T == X (L_A L_B)^T
    np.testing.assert_allclose((xf @ bf.T) @ af.T, xf @ (af @ bf).T, rtol=1e-12, atol=1e-15)


def test_rows_subset_matches_full():
    X, W, L_A, L_B = make_custom(40, 64, 24, 16, seed=8)
    full = oracle.linear(X, W, L_A, L_B)
    rows = [39, 0, 17, 17, 5]
    part = oracle.linear(X, W, L_A, L_B, rows=rows)
    assert (part == full[rows]).all()


# ----------------------------------------------------------------------------- symmetries
def test_scaling_by_power_of_two_and_negation():
    X, W, L_A, L_B = make_custom(16, 64, 24, 16, seed=10)
    meta, vals, s = oracle.sparsify(X)
    Y = oracle.linear(X, W, L_A, L_B)
    for k in (-3, 4):
        Xk = to_bf16_bits(bf16_bits_to_f32(X) * np.float32(2.0 ** k))
        mk, vk, sk = oracle.sparsify(Xk)
        assert (mk == meta).all()
        assert (f64(vk) == f64(vals) * 2.0 ** k).all()
        assert (oracle.linear(Xk, W, L_A, L_B) == Y * 2.0 ** k).all()
    Xn = X ^ np.uint16(0x8000)
    mn, vn, sn = oracle.sparsify(Xn)
    assert (mn == meta).all() and (sn == s).all() and (f64(vn) == -f64(vals)).all()
    assert (oracle.linear(Xn, W, L_A, L_B) == -Y).all()


def test_token_and_group_permutations():
    X, W, L_A, L_B = make_custom(16, 64, 24, 16, seed=12)
    Y = oracle.linear(X, W, L_A, L_B)
    perm = np.random.default_rng(1).permutation(16)
    assert (oracle.linear(X[perm], W, L_A, L_B) == Y[perm]).all()
    gperm = np.random.default_rng(2).permutation(16)
    cols = (4 * gperm[:, None] + np.arange(4)[None, :]).reshape(-1)
    Yg = oracle.linear(X[:, cols], W[:, cols], L_A, L_B[:, cols])
    np.testing.assert_allclose(Yg, Y, rtol=1e-11, atol=1e-12 * np.abs(Y).max())
    # permuting channels inside a group changes which channel survives but not Y
    # when the permutation is applied to W and L_B as well
    inner = np.array([2, 0, 3, 1])
    cols2 = (4 * np.arange(16)[:, None] + inner[None, :]).reshape(-1)
    Yi = oracle.linear(X[:, cols2], W[:, cols2], L_A, L_B[:, cols2])
    ties = False  # equal magnitudes inside a group could legitimately change the kept pair
    xf = np.abs(f64(X)).reshape(16, 16, 4)
    for m in range(16):
        for g in range(16):
            if len(set(xf[m, g].tolist())) < 4:
                ties = True
    if not ties:
        np.testing.assert_allclose(Yi, Y, rtol=1e-11, atol=1e-12 * np.abs(Y).max())


def test_bf16_rounding_helper_is_nearest_even():
    # values exactly between two bf16 neighbours go to the even significand
    one = Fraction(1)
    ulp = Fraction(1, 128)
    assert oracle.bf16_round(float(one + ulp / 2)) == 0x3F80
    assert oracle.bf16_round(float(one + 3 * ulp / 2)) == 0x3F82
    assert oracle.bf16_round(2.0 ** -134) == 0x0000       # half the smallest subnormal: ties to 0
    assert oracle.bf16_round(1.5 * 2.0 ** -133) == 0x0002
    assert oracle.bf16_round(3.5e38) == 0x7F80
    rng = np.random.default_rng(0)
    for v in rng.standard_normal(200) * 10.0 ** rng.integers(-30, 30, 200):
        assert oracle.bf16_round(float(v)) == nearest_bf16_bits(Fraction(float(v)))


def test_tiny_digest_unchanged():
    """The oracle's outputs on the tiny workload match the stored digest
    (written by tests/golden/make_golden.py, which calls only the oracle)."""
    import importlib.util
    spec = importlib.util.spec_from_file_location("make_golden", os.path.join(GOLDEN, "make_golden.py"))
    mg = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mg)
    want = json.load(open(os.path.join(GOLDEN, "tiny_oracle.json")))
    got = mg.digest()
    assert got == want



# ------------------------------------------------------------------ feed-forward block (GELU between two layers)
def test_gelu_closed_forms():
    """GELU(x) = x Phi(x): Phi(1) and Phi(2) from the standard normal table,
    the identity GELU(x) - GELU(-x) = x, GELU(0) = 0, and the scipy routine."""
    from scipy.special import ndtr
    assert abs(oracle.gelu(1.0) - 0.8413447460685429) < 1e-15       # Phi(1)
    assert abs(oracle.gelu(2.0) - 2 * 0.9772498680518208) < 1e-15   # 2 Phi(2)
    assert oracle.gelu(0.0) == 0.0
    rng = np.random.default_rng(7)
    for x in rng.normal(0, 3, 200):
        assert abs(oracle.gelu(x) - oracle.gelu(-x) - x) <= 1e-14 * max(1.0, abs(x))
        assert abs(oracle.gelu(x) - x * ndtr(x)) <= 1e-14 * max(1.0, abs(x))
    assert abs(oracle.gelu(10.0) - 10.0) < 1e-20 and abs(oracle.gelu(-10.0)) < 1e-20


def test_gelu_bf16_is_one_rounding_of_the_exact_value():
    """H = bf16(GELU(y)) rounded once, nearest even: compared with the exact
    nearest bf16 of a 40-digit GELU value (skip values within 1e-12 relative of
    a rounding boundary, where the double evaluation may land either side)."""
    from scipy.special import ndtr
    rng = np.random.default_rng(8)
    y = np.concatenate([rng.normal(0, 2, 3000), rng.normal(0, 40, 1000), [0.0, -0.0, 1e-30, -5.5, 3.25]])
    H = oracle.gelu_bf16(y)
    checked = 0
    for yi, hb in zip(y, H):
        g = Fraction(float(yi)) * Fraction(float(ndtr(yi)))
        lo = nearest_bf16_bits(g * (1 - Fraction(1, 10 ** 12)))
        hi = nearest_bf16_bits(g * (1 + Fraction(1, 10 ** 12)))
        if lo == hi:
            def z(b):  # +0 and -0 are the same value (GELU of a large negative y rounds to a zero)
                return 0 if b == 0x8000 else b
            assert z(int(hb)) == z(lo), (yi, hex(int(hb)), hex(lo))
            checked += 1
    assert checked > 3900


def test_mlp_block_wiring_with_selection_weights():
    """Up-projection dense-skip with W_up selecting input channels (rows of the
    identity): Y_up = X exactly, so H = bf16(GELU(X)).  Down-projection
    dense-skip with W_down = identity: Y = H.  Tokens are independent, so a row
    subset equals the same rows of the whole."""
    M, D = 24, 32
    X, _, _, _ = make_custom(M, D, 8, 8, seed=41)
    eye = to_bf16_bits(np.eye(D, dtype=np.float32))
    Y_up, H, Y = oracle.mlp_block(X, eye, None, None, eye, None, None,
                                  mode_up=oracle.MODE_DENSE_SKIP, mode_down=oracle.MODE_DENSE_SKIP)
    xf = f64(X)
    assert (Y_up == xf).all()
    assert (H == oracle.gelu_bf16(xf)).all()
    assert (Y == f64(H)).all()
    rows = [3, 0, 17]
    Y_up2, H2, Y2 = oracle.mlp_block(X, eye, None, None, eye, None, None,
                                     mode_up=oracle.MODE_DENSE_SKIP, mode_down=oracle.MODE_DENSE_SKIP, rows=rows)
    assert (Y_up2 == Y_up[rows]).all() and (H2 == H[rows]).all() and (Y2 == Y[rows]).all()


def test_mlp_block_sparse_rows_subset():
    from activation_sparse_gemm_b200.inputs import make_block_inputs
    args = make_block_inputs(40, 64, 128, 16, seed=9)
    _, H, Y = oracle.mlp_block(*args)
    rows = [39, 2, 11]
    _, H2, Y2 = oracle.mlp_block(*args, rows=rows)
    assert (H2 == H[rows]).all() and (Y2 == Y[rows]).all()
    # GELU output is never below its minimum, about -0.17
    assert (bf16_bits_to_f32(H) >= -0.1701).all()


# ------------------------------------------------------------------ LoRA fit (reduced-rank regression)
def _objective(X, E, L_A, L_B):
    return float(np.linalg.norm(X @ (L_A @ L_B).T - E) ** 2)


def test_reduced_rank_fit_recovers_a_planted_map():
    """E = X C^T with rank(C) = R: the fit returns C exactly (up to rounding)."""
    rng = np.random.default_rng(11)
    M, K, N, R = 400, 40, 56, 6
    X = rng.standard_normal((M, K)) * rng.lognormal(0, 1, K)
    C = rng.standard_normal((N, R)) @ rng.standard_normal((R, K))
    L_A, L_B, sig = oracle.reduced_rank_fit(X, X @ C.T, R)
    assert np.abs(L_A @ L_B - C).max() <= 1e-9 * np.abs(C).max()
    assert sig[R] <= 1e-9 * sig[0]
    assert np.allclose(L_A.T @ L_A, np.eye(R), atol=1e-12)


def test_reduced_rank_fit_meets_the_eckart_young_optimum():
    """The objective equals the least-squares residual plus the energy of the
    discarded singular values of the least-squares fit (the closed-form
    optimum), falls as R grows, and is below two other rank-R candidates:
    the truncated SVD of E itself mapped back through least squares, and zero."""
    rng = np.random.default_rng(12)
    M, K, N = 300, 32, 48
    X = rng.standard_normal((M, K))
    E = rng.standard_normal((M, N)) + X @ rng.standard_normal((K, N))
    B0 = np.linalg.lstsq(X, E, rcond=None)[0]
    ls_res = float(np.linalg.norm(X @ B0 - E) ** 2)
    prev = None
    for R in (1, 4, 16, 32):
        L_A, L_B, sig = oracle.reduced_rank_fit(X, E, R)
        obj = _objective(X, E, L_A, L_B)
        assert abs(obj - (ls_res + float(np.sum(sig[R:] ** 2)))) <= 1e-9 * obj
        U, s, Vt = np.linalg.svd(E, full_matrices=False)
        Et = (U[:, :R] * s[:R]) @ Vt[:R]
        Bt = np.linalg.lstsq(X, Et, rcond=None)[0]           # a rank-R candidate
        assert obj <= _objective(X, E, Bt.T, np.eye(K)) * (1 + 1e-12)
        assert obj <= float(np.linalg.norm(E) ** 2)
        if prev is not None:
            assert obj <= prev * (1 + 1e-12)
        prev = obj
    assert abs(prev - ls_res) <= 1e-9 * prev  # R = K: the least-squares residual itself


def test_lora_fit_targets_the_sparsification_residual():
    """The fitted LoRA lowers ||X W^T - S(X) W^T - X (L_A L_B)^T||, and with the
    fitted factors the oracle's layer moves toward the dense layer."""
    X, W, _, _ = make_custom(700, 64, 48, 8, seed=13, p_out=0.05)
    R = 8
    L_A, L_B, E = oracle.lora_fit(X, W, R)
    Xf = f64(X)
    assert _objective(Xf, E, L_A, L_B) < 0.95 * float(np.linalg.norm(E) ** 2)
    A16, B16 = to_bf16_bits(L_A.astype(np.float32)), to_bf16_bits(L_B.astype(np.float32))
    Yd = oracle.linear(X, W, mode=oracle.MODE_DENSE_SKIP)
    err_none = np.linalg.norm(oracle.linear(X, W) - Yd)
    err_fit = np.linalg.norm(oracle.linear(X, W, A16, B16) - Yd)
    assert err_fit < 0.975 * err_none
