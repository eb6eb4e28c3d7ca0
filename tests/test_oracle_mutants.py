"""Plant mistakes in a copy of the CPU oracle and check that the pins catch each one.

Every mutant is a plausible slip in the oracle's C source (a dropped term, a
wrong sign, a transposed operand, a lost index, a missed convention).  The
mutant is compiled on the CPU into a temporary library, swapped in for the
real oracle, and the pin tests of ``test_oracle_pins`` are run against it;
at least one must fail.  No GPU is involved.
"""
import os
import subprocess

import numpy as np
import pytest

import oracle
import test_oracle_mask_pins as mpins
import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "ragged_oracle.c")

MUTANTS = {
    "cls_not_forced": ("if (j == 0)\n        return 1;", "if (j < 0)\n        return 1;"),
    "scale_dropped": ("s[j] = J->scale * dot;", "s[j] = dot;"),
    "qk_transposed": ("dot += Q[i * d + c] * K[j * d + c];", "dot += Q[j * d + c] * K[i * d + c];"),
    "last_value_dropped": ("for (int64_t j = 0; j < L; ++j)\n                acc += s[j] * V[j * d + c];",
                           "for (int64_t j = 0; j < L - 1; ++j)\n                acc += s[j] * V[j * d + c];"),
    "not_normalised": ("o[c] = acc / l;", "o[c] = acc;"),
    "exp_sign_flipped": ("s[j] = exp(s[j] - m);", "s[j] = exp(m - s[j]);"),
    "head_offset_lost": ("(start + i) * J->tok_stride + h * J->head_stride + c;",
                         "(start + i) * J->tok_stride + c;"),
    "half_exponent_bias": ("ldexp((double)(0x400 | f), e - 25)", "ldexp((double)(0x400 | f), e - 24)"),
    "cu_off_by_one": ("        cu[b + 1] = (int32_t)t;\n    }\n    return t;\n}\n\n/* Pack",
                      "        cu[b + 1] = (int32_t)t + 1;\n    }\n    return t;\n}\n\n/* Pack"),
    "pack_reads_wrong_row": ("dense + (b * L_full + j) * row_bytes,\n                       (size_t)row_bytes);\n                ++t;\n            }\n        }\n        cu[b + 1]",
                             "dense + (b * L_full + (L_full - 1 - j)) * row_bytes,\n                       (size_t)row_bytes);\n                ++t;\n            }\n        }\n        cu[b + 1]"),
    "topk_tie_to_higher_index": ("    return ia < ib;", "    return ia > ib;"),
    "topk_nan_ranks_first": ("return nb; /* every number ranks before NaN */", "return na; /* every number ranks before NaN */"),
    "topk_ascending": ("        return a > b;", "        return a < b;"),
    "topk_one_too_few": ("for (int64_t r = 0; r < k - 1; ++r)", "for (int64_t r = 0; r < k - 2; ++r)"),
    "l2_strict_threshold": ("            return a[i] > b[i];\n    return 1;", "            return a[i] > b[i];\n    return 0;"),
    "l2_last_element_dropped": ("for (int64_t c = 0; c < C; ++c) {\n            const double v = load_elem(x, dtype, t * tok_stride + c);",
                                "for (int64_t c = 0; c < C - 1; ++c) {\n            const double v = load_elem(x, dtype, t * tok_stride + c);"),
    "l2_cls_not_forced": ("if (t % L_full == 0)\n            kept = 1;", "if (t % L_full == -1)\n            kept = 1;"),
    "l2_square_doubled": ("big_add(S, (unsigned __int128)m * m, 2 * e + L2_UNIT);",
                          "big_add(S, (unsigned __int128)m * m, 2 * e + L2_UNIT + 1);"),
    "l2_carry_lost": ("        carry = sum >> 32;", "        carry = 0;"),
    "l2_tau_rounded_down": ("q = (M2 >> c) + ((M2 & ((((unsigned __int128)1) << c) - 1)) != 0);", "q = (M2 >> c);"),
    "l2_nan_kept": ("        else if (has_nan)\n            kept = 0;", "        else if (has_nan)\n            kept = 1;"),
}


def _pin_calls():
    calls = [pins.test_hand_example_seqlens_and_pack, pins.test_decode_f16_all_bit_patterns,
             pins.test_decode_bf16_all_bit_patterns, pins.test_weights_sum_to_one,
             pins.test_closed_forms, pins.test_hand_example_attention,
             pins.test_brute_force_tiny_lengths, pins.test_attention_no_pruning_equals_dense_sdpa,
             pins.test_key_shift_invariance_and_convex_hull]
    for dt in ("f16", "bf16", "f32"):
        calls.append(lambda dt=dt: pins.test_attention_equals_padded_masked_sdpa(dt))
    for keep in pins._random_masks():
        calls.append(lambda keep=keep: pins.test_seqlens_matches_flatnonzero(keep))
        calls.append(lambda keep=keep: pins.test_pack_unpack_roundtrip(keep))
    calls += [mpins.test_topk_closed_cases, mpins.test_topk_counts_and_cls, mpins.test_l2_boundary_and_closed_cases,
              mpins.test_l2_decides_where_fp64_sums_round, mpins.test_l2_subnormals_nan_and_infinity]
    for ties in (False, True):
        for nans in (False, True):
            calls.append(lambda ties=ties, nans=nans: mpins.test_topk_matches_lexsort(ties, nans))
    for dt in ("f16", "bf16", "f32"):
        calls.append(lambda dt=dt: mpins.test_l2_matches_exact_arithmetic(dt))
        calls.append(lambda dt=dt: mpins.test_l2_exact_at_and_next_to_tau(dt))
    return calls


@pytest.fixture(scope="module")
def source():
    return open(SRC).read()


# Mutant copies are built beside the oracle's own library (a git-ignored folder).
MUTANT_DIR = os.path.join(os.path.dirname(SRC), "_build", "mutants")


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, source):
    old, new = MUTANTS[name]
    assert source.count(old) == 1, f"mutation site for {name} not found exactly once"
    os.makedirs(MUTANT_DIR, exist_ok=True)
    mutant_src = os.path.join(MUTANT_DIR, f"{name}.c")
    with open(mutant_src, "w") as f:
        f.write(source.replace(old, new))
    so = os.path.join(MUTANT_DIR, f"lib{name}.so")
    subprocess.run(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-shared", "-fPIC", "-pthread", mutant_src,
                    "-o", so, "-lm"], check=True)
    real = oracle._load()
    oracle.use_library(oracle.bind(str(so)))
    caught = 0
    try:
        with np.errstate(all="ignore"):
            for call in _pin_calls():
                try:
                    call()
                except AssertionError:
                    caught += 1
    finally:
        oracle.use_library(real)
    assert caught > 0, f"no pin caught mutant {name}"


def test_unmutated_source_passes_all_pins():
    for call in _pin_calls():
        call()
