"""The oracle's pins must catch plausible mistakes.

Each case plants one mistake in a copy of the oracle's C source (on the CPU,
in a temporary directory), builds it, and runs every pin of test_oracle.py
against the mutant.  At least one pin has to fail for every mutant.
"""
import os
import types

import pytest

import oracle
from tests import test_oracle as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "rtlynx_oracle.c")

MUTANTS = {
    "tie_to_higher_index": ("(aj == ai && j < i)", "(aj == ai && j > i)"),
    "signed_topk": ("double aj = fabs(x[j]), ai = fabs(x[i]);", "double aj = x[j], ai = x[i];"),
    "eps_inside_sqrt": ("sqrt(nx) / (sqrt(nt) + RTLYNX_EPS)", "sqrt(nx) / sqrt(nt + RTLYNX_EPS)"),
    "no_norm_compensation": ("float s = (float)(sqrt(nx) / (sqrt(nt) + RTLYNX_EPS));", "float s = 1.0f;"),
    "swapped_meta_nibbles": ("meta[g] = (uint8_t)(i0 | (i1 << 2));", "meta[g] = (uint8_t)(i1 | (i0 << 2));"),
    "unscaled_values": ("double_to_bf16_rne((double)s * x[i0])", "double_to_bf16_rne(x[i0])"),
    "lora_on_sparse_x": ("acc += bf16_to_double(Xrow[k]) * bf16_to_double(L_B[r * K + k]);",
                         "acc += A[k] * bf16_to_double(L_B[r * K + k]);"),
    "lora_up_transposed": ("lr += Trow[r] * bf16_to_double(L_A[n * R + r]);",
                           "lr += Trow[r] * bf16_to_double(L_A[r * N + n]);"),
    "lora_subtracted": ("acc += lr;", "acc -= lr;"),
    "lora_dropped": ("acc += lr;", "acc += 0.0 * lr;"),
    "w_transposed": ("acc += A[k] * bf16_to_double(W[n * K + k]);", "acc += A[k] * bf16_to_double(W[k * N + n]);"),
    "dense_skip_sparsifies": ("if (mode == 0) {\n            sparsify_row", "if (1) {\n            sparsify_row"),
    "nt_over_all_channels": ("nt += x[i0] * x[i0] + x[i1] * x[i1];",
                             "nt += x[0] * x[0] + x[1] * x[1] + x[2] * x[2] + x[3] * x[3];"),
    "round_toward_zero": ("r = ldexp(nearbyint(ldexp(m, 8)), e - 8);", "r = ldexp(trunc(ldexp(m, 8)), e - 8);"),
}

PIN_TESTS = [
    pins.test_worked_example,
    pins.test_mask_bruteforce_small_alphabet,
    pins.test_mask_random_rows_exact_s,
    lambda: pins.test_invariants_on_workload_distributions("tiny"),
    lambda: pins.test_invariants_on_workload_distributions("mlp_down"),
    pins.test_zero_groups_and_zero_rows,
    pins.test_already_two_of_four_reduces_to_textbook_gemm,
    pins.test_lora_zero_gives_sparse_branch_exactly,
    pins.test_dense_skip_is_textbook_gemm,
    pins.test_brute_force_tiny_against_numpy,
    pins.test_scaling_by_power_of_two_and_negation,
    pins.test_token_and_group_permutations,
    pins.test_bf16_rounding_helper_is_nearest_even,
]


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, tmp_path, monkeypatch):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not found or not unique"
    mut_src = tmp_path / "mutant.c"
    mut_src.write_text(src.replace(old, new))
    lib = oracle.build(force=True, src=str(mut_src), out=str(tmp_path / "libmutant.so"))
    o = oracle.Oracle(lib)
    ns = types.SimpleNamespace(sparsify=o.sparsify, linear=o.linear, bf16_round=o.bf16_round,
                               MODE_SPARSE=oracle.MODE_SPARSE, MODE_DENSE_SKIP=oracle.MODE_DENSE_SKIP)
    monkeypatch.setattr(pins, "oracle", ns)
    caught = []
    for pin in PIN_TESTS:
        try:
            pin()
        except (AssertionError, ValueError, FloatingPointError):
            caught.append(getattr(pin, "__name__", "lambda"))
    assert caught, f"no pin caught mutant {name}"
