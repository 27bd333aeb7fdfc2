"""The oracle's pins catch plausible mistakes.  Each case copies the oracle's C
source, plants one mistake in the copy (a dropped term, a wrong sign, an
off-by-one mask, a wrong index, a transposed operand), builds it with gcc and
runs the pin suite against that library in place of the real one: at least
one pin must fail.  The unmodified copy, built the same way, must pass every
pin, so a failure is the planted mistake's doing.  Every planted mistake keeps
all memory accesses in bounds.  The committed oracle is never modified."""
import ctypes
import os

import pytest

import oracle
import tests.test_decode_oracle_pins as dec_pins
import tests.test_gemm_oracle_pins as gemm_pins
import tests.test_oracle_pins as pins

_SRC = os.path.join(os.path.dirname(oracle.__file__), "attention_oracle.c")

# (name, text in the source, replacement, which occurrence)
MUTANTS = [
    ("causal row sees one key too few", "i64 cnt = causal ? i + 1 : N;",
     "i64 cnt = causal ? i : N;", 0),
    ("scale dropped from the scores", "s[j] = scale * acc;\n  }\n  return cnt;",
     "s[j] = acc;\n  }\n  return cnt;", 0),
    ("row maximum not subtracted in the sum", "l += exp(s[j] - m);", "l += exp(s[j]);", 0),
    ("lse without the row maximum", "lse[i] = m + log(l);", "lse[i] = log(l);", 0),
    ("value columns reversed", "oi[c] += p * vj[c];", "oi[c] += p * vj[d - 1 - c];", 0),
    ("dS sign flipped in dQ", "double ds = p * (dp - d_pdp);", "double ds = p * (d_pdp - dp);", 0),
    ("scale dropped from dK", "dkj[c] += scale * ds * qi[c];", "dkj[c] += ds * qi[c];", 0),
    ("dV from the key row's dO (transposed P)", "dvj[c] += p * doi[c];",
     "dvj[c] += p * dO[j * d + c];", 0),
    ("D dropped from dS in dK", "double ds = p * (dp - D[i]);", "double ds = p * dp;", 0),
    ("mask excludes the diagonal", "return !causal || j <= i;", "return !causal || j < i;", 0),
    ("online: sum not rescaled", "l = alpha * l + psum;", "l = l + psum;", 0),
    ("online: output not rescaled", "for (i64 c = 0; c < d; ++c) acc[c] *= alpha;", ";", 0),
    ("online: lse without the running maximum", "lse[i] = m + log(l);", "lse[i] = log(l);", 1),
    ("decode: causal window one key short", "i64 cnt = causal ? len - Nq + i + 1 : len;",
     "i64 cnt = causal ? len - Nq + i : len;", 0),
    ("decode: scale dropped", "s[j] = scale * acc;\n      }\n      double m;",
     "s[j] = acc;\n      }\n      double m;", 0),
    ("gemm: B columns reversed", "ci[j] += a * bk[j];", "ci[j] += a * bk[N - 1 - j];", 0),
]


def _pin_calls():
    calls = []
    for c in (False, True):
        calls += [
            (pins.test_online_softmax_equals_three_pass, (c, 7)),
            (pins.test_probability_rows, (c,)),
            (pins.test_uniform_scores, (c,)),
            (pins.test_key_shift_invariance, (c,)),
            (pins.test_gradient_sum_rules, (c,)),
            (pins.test_dS_rows_sum_to_zero, (c,)),
            (pins.test_finite_differences, (c, 3, 4)),
            (pins.test_against_torch_sdpa_fp64, (c, 129, 64)),
            (dec_pins.test_square_case_is_the_forward, (c,)),
            (dec_pins.test_rows_past_the_length_are_never_read, (c,)),
            (dec_pins.test_against_torch_sdpa_fp64, (c,)),
        ]
    calls += [(f, ()) for f in (
        pins.test_causal_row0_exact, pins.test_closed_form_two_keys,
        pins.test_selected_rows_match_full_forward, pins.test_large_logits_stay_finite,
        dec_pins.test_single_key_returns_its_value, dec_pins.test_identical_keys_average_the_values,
        dec_pins.test_two_keys_closed_form, dec_pins.test_causal_mask_ends_at_the_newest_key,
        dec_pins.test_rows_with_no_visible_key, dec_pins.test_permuting_visible_cache_rows,
        gemm_pins.test_brute_force_tiny, gemm_pins.test_identities,
        gemm_pins.test_rank_one_closed_form, gemm_pins.test_transpose_identity,
        gemm_pins.test_against_numpy)]
    return calls


def _replace_nth(text, old, new, n):
    start = -1
    for _ in range(n + 1):
        start = text.find(old, start + 1)
        assert start >= 0, f"mutation anchor not found: {old!r} (occurrence {n})"
    return text[:start] + new + text[start + len(old):]


def _failing_pins(tmp_path, tag, source):
    src = tmp_path / f"{tag}.c"
    src.write_text(source)
    lib = oracle.bind(ctypes.CDLL(oracle.compile_source(str(src), str(tmp_path / f"{tag}.so"))))
    saved = oracle._load()
    oracle._lib = lib
    failed = []
    try:
        for fn, args in _pin_calls():
            try:
                fn(*args)
            except Exception:  # an assertion, or a NaN the check trips on
                failed.append(f"{fn.__module__.split('.')[-1]}.{fn.__name__}{args}")
    finally:
        oracle._lib = saved
    return failed


def test_unmodified_copy_passes_every_pin(tmp_path):
    assert _failing_pins(tmp_path, "control", open(_SRC).read()) == []


@pytest.mark.filterwarnings("ignore::RuntimeWarning")  # NaN/inf from a planted mistake
@pytest.mark.parametrize("name,old,new,nth", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistake_is_caught(tmp_path, name, old, new, nth):
    text = open(_SRC).read()
    failed = _failing_pins(tmp_path, "mutant", _replace_nth(text, old, new, nth))
    assert failed, f"no pin catches: {name}"
