"""Plant plausible mistakes into copies of the oracle and check that the pins catch each one.

Every mutant is a one-line textual change to oracle.c (a dropped term, a wrong sign, index or
rounding rule, a transposed operand), compiled with gcc into a temporary directory and swapped
in for the real oracle while the pins of tests/test_oracle_pins.py run against it.  A mutant
that no pin rejects would mean the pins leave that part of the oracle unchecked.
"""
import os
import subprocess

import pytest

import oracle
import test_oracle_pins as pins

ORACLE_C = os.path.join(os.path.dirname(oracle.__file__), "oracle.c")

# (name, original text, mutated text)
MUTANTS = [
    ("attend: logits not divided by sqrt(D)", "z[t] = dot / sqrt_d;", "z[t] = dot;"),
    ("attend: wrong sign in the exponent", "l += exp(z[t] - m);", "l += exp(m - z[t]);"),
    ("attend: output not normalised", "og[d] /= l;", "og[d] /= 1.0;"),
    ("attend: lse missing the max", "lse[g] = m + log(l);", "lse[g] = log(l);"),
    ("attend: value channels reversed", "og[d] += w * v[(size_t)t * D + d];",
     "og[d] += w * v[(size_t)t * D + (D - 1 - d)];"),
    ("attend: keys read in reverse token order", "dot += qg[d] * k[(size_t)t * D + d];",
     "dot += qg[d] * k[(size_t)(n - 1 - t) * D + d];"),
    ("merge: weights use the max instead of the merged lse",
     "acc += exp(lse_c[(size_t)c * G + g] - L)", "acc += exp(lse_c[(size_t)c * G + g] - M)"),
    ("merge: lse is the max only", "lse[g] = L;", "lse[g] = M;"),
    ("quantize: round half away from zero", "nearbyint((double)quotient)", "round((double)quotient)"),
    ("quantize: scale divides by 128", "(double)amax / 127.0", "(double)amax / 128.0"),
    ("quantize: clamp at 128", "if (r > 127.0)", "if (r > 128.0)"),
    ("quantize: multiply by a float32 reciprocal", "(float)((double)x / (double)scale)",
     "(float)(x * (1.0f / scale))"),
    ("quantize: amax ignores the sign", "const float a = fabsf(x[i]);", "const float a = x[i];"),
    ("oam: beta dropped", "s[t] = best + beta * log(sqrt(sq) + eps);", "s[t] = best + log(sqrt(sq) + eps);"),
    ("oam: log of the squared norm", "log(sqrt(sq) + eps)", "log(sq + eps)"),
    ("oam: routing not divided by sqrt(D)", "const double z = dot / sqrt_d;", "const double z = dot;"),
    ("oam: last head instead of the max", "if (z > best)\n                best = z;", "best = z;"),
    ("topk: ties prefer the higher index", "return (i > j) - (i < j);\n}\n\nstatic int ascending",
     "return (i < j) - (i > j);\n}\n\nstatic int ascending"),
    ("topk: keeps the lowest scores", "if (si > sj)\n        return -1;\n    if (si < sj)\n        return 1;",
     "if (si > sj)\n        return 1;\n    if (si < sj)\n        return -1;"),
    ("plan: chunk size not rounded to the granule", "S = (S + granule - 1) / granule * granule;", ""),
    ("plan: segment start in stream coordinates", "seg_start[count] = lo - pos[r];", "seg_start[count] = lo;"),
    ("plan: the per-row charge dropped", "/ granule * granule + row_cost;", "/ granule * granule;"),
]

# pins re-run against each mutant (call -> raises on a caught mistake)
PIN_CALLS = [
    lambda g: pins.test_attend_matches_torch_sdpa(4, 8, 16),
    lambda g: pins.test_attend_matches_torch_sdpa(3, 16, 37),
    lambda g: pins.test_attend_identical_keys_gives_mean_of_v(),
    lambda g: pins.test_attend_one_token_returns_its_value(),
    lambda g: pins.test_attend_two_tokens_closed_form(),
    lambda g: pins.test_decode_matches_sdpa_with_repeat_interleave(4),
    lambda g: pins.test_merge_of_every_chunking_equals_unsplit(7),
    lambda g: pins.test_quantize_worked_cases(g),
    lambda g: pins.test_quantize_clamps_to_127(g),
    lambda g: pins.test_quantize_matches_numpy_float32_route(),
    lambda g: pins.test_quantize_amax_element_maps_to_127_and_bounds(),
    lambda g: pins.test_quantize_integers_reproduce_and_ties_go_to_even(),
    lambda g: pins.test_scheme_a_partitions_start_at_each_sequence(),
    lambda g: pins.test_oam_hand_example(g),
    lambda g: pins.test_oam_scores_match_torch_route(),
    lambda g: pins.test_topk_matches_brute_force_sort(),
    lambda g: pins.test_topk_all_equal_keeps_lowest_indices_and_keep_all(),
    lambda g: pins.test_beta_zero_is_classic_qk_ranking_and_q_zero_is_norm_ranking(),
    lambda g: pins.test_plan_hand_example(g),
    lambda g: pins.plan_coverage(3),
    lambda g: pins.plan_coverage(5, 256),
]


def test_real_oracle_passes_the_pin_subset(golden_dir):
    for call in PIN_CALLS:
        call(golden_dir)


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(name, old, new, tmp_path, golden_dir, monkeypatch):
    src = open(ORACLE_C).read()
    assert src.count(old) == 1, f"mutation anchor not unique/present: {old!r}"
    mutated = tmp_path / "oracle_mutant.c"
    mutated.write_text(src.replace(old, new))
    so = tmp_path / "liboracle_mutant.so"
    subprocess.check_call(["gcc", "-std=c11", "-O2", "-fPIC", "-shared", "-ffp-contract=off",
                           "-w", "-o", str(so), str(mutated), "-lm"])
    monkeypatch.setattr(oracle, "_lib", oracle.load(str(so)))
    caught = []
    for i, call in enumerate(PIN_CALLS):
        try:
            call(golden_dir)
        except Exception:  # an assertion (or an error raised by the oracle wrapper)
            caught.append(i)
    assert caught, f"no pin catches the planted mistake: {name}"
