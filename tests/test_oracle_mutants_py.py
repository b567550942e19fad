"""Plant plausible mistakes into copies of the oracle's numpy-level functions (query codes,
value norms, selection over the INT8 cache, multi-token decode and selection, block selection)
and check that the pins of tests/test_oracle_pins.py catch each one.

Each mutant is a one-line textual change to oracle/__init__.py, executed as a fresh module
whose functions replace the real oracle's for the duration of the test (the C library is
shared, so only the Python step that the mutant changes differs).
"""
import os
import types

import pytest

import oracle
import test_oracle_pins as pins

ORACLE_PY = oracle.__file__


def pins_golden_dir():
    return os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")

# (name, original text, mutated text)
MUTANTS = [
    ("query codes: per-row scale taken from the whole tensor",
     "scales[b, h] = scale_from_amax(amax(x[b, h]))", "scales[b, h] = scale_from_amax(amax(x))"),
    ("query codes: dequantised with the mean scale",
     "return np.asarray(codes, np.float64) * s[..., None]", "return np.asarray(codes, np.float64) * s.mean()"),
    ("value norms: squared norm", "return np.sqrt(np.sum(x * x, axis=-1))", "return np.sum(x * x, axis=-1)"),
    ("int8 selection: K codes without their scales",
     "khat = dequant_rows(kc[h, s0:e0], k_scale_of_tokens(ks, scheme, h, b, L, cu_parts, part))",
     "khat = dequant_rows(kc[h, s0:e0], np.ones(L))"),
    ("multi-token decode: causal limit one short", "vis = pos <= L - M + m", "vis = pos < L - M + m"),
    ("multi-token decode: causal limit one long", "vis = pos <= L - M + m", "vis = pos <= L - M + m + 1"),
    ("multi-token decode: query tokens reversed",
     "attend(q[b, m, heads], kr[vis], vr[vis])", "attend(q[b, M - 1 - m, heads], kr[vis], vr[vis])"),
    ("multi-token selection: first query token only",
     "qg = _f64(q[b, :, h * G:(h + 1) * G]).reshape(M * G, D)", "qg = _f64(q[b, 0, h * G:(h + 1) * G])"),
    ("block scores: mean instead of max",
     "return np.array([s[j * block:(j + 1) * block].max() for j in range(nb)], np.float64)",
     "return np.array([s[j * block:(j + 1) * block].mean() for j in range(nb)], np.float64)"),
    ("block selection: ties prefer the higher block",
     "blk[h, cu_kept[b]:cu_kept[b + 1]] = topk(bs[(b, h)], int(kept[b]))",
     "blk[h, cu_kept[b]:cu_kept[b + 1]] = np.sort(bs[(b, h)].size - 1 - topk(bs[(b, h)][::-1], int(kept[b])))"),
    ("calibrated quantisation: the given V scale ignored", "    if v_scale is None:\n        v_amax",
     "    if True:\n        v_amax"),
    ("calibrated quantisation: scheme B codes K with the V scale", "ks = np.float32(k_scale)",
     "ks = np.float32(v_scale)"),
    ("block decode: ragged last block not cut at the sequence end",
     "toks = np.concatenate([np.arange(j * block, min((j + 1) * block, L))",
     "toks = np.concatenate([np.arange(j * block, (j + 1) * block)"),
]

PIN_CALLS = [
    lambda: pins.test_calibrated_scales_hand_example(pins_golden_dir()),
    lambda: pins.test_calibrated_with_the_computed_scales_is_the_dynamic_quantisation(),
    lambda: pins.test_query_quantisation_per_row_and_per_tensor(),
    lambda: pins.test_value_norms_closed_form_and_library(),
    lambda: pins.test_int8_selection_with_exact_codes_is_the_plain_selection(),
    lambda: pins.test_multi_token_with_one_token_is_decode(),
    lambda: pins.test_multi_token_query_m_is_decode_over_the_truncated_cache(2),
    lambda: pins.test_multi_token_query_m_is_decode_over_the_truncated_cache(4),
    lambda: pins.test_multi_token_matches_sdpa_with_a_causal_offset_mask(),
    lambda: pins.test_multi_token_over_kept_tokens_masks_by_position(),
    lambda: pins.test_multi_token_scores_are_the_max_over_the_tokens_single_scores(),
    lambda: pins.test_block_scores_brute_force_with_ragged_last_block(),
    lambda: pins.test_block_selection_with_one_token_blocks_is_token_selection(),
    lambda: pins.test_block_selection_hand_example_and_ties(),
    lambda: pins.test_block_selection_brute_force_ranking(),
    lambda: pins.test_decode_over_blocks_is_attention_over_their_tokens(),
]


def test_real_oracle_passes_the_pin_subset():
    for call in PIN_CALLS:
        call()


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(name, old, new, monkeypatch):
    src = open(ORACLE_PY).read()
    assert src.count(old) == 1, f"mutation anchor not unique/present: {old!r}"
    mod = types.ModuleType("oracle_mutant")
    mod.__file__ = ORACLE_PY  # the C library is found beside the real file
    exec(compile(src.replace(old, new), ORACLE_PY, "exec"), mod.__dict__)
    mod._lib = oracle.lib()  # share the loaded C oracle
    for attr, val in vars(mod).items():
        if isinstance(val, types.FunctionType):
            monkeypatch.setattr(oracle, attr, val)
    caught = []
    for i, call in enumerate(PIN_CALLS):
        try:
            call()
        except Exception:  # an assertion (or an error the mutated oracle raises)
            caught.append(i)
    assert caught, f"no pin catches the planted mistake: {name}"
