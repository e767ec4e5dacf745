"""The oracle's pins reject plausible mistakes in the oracle itself.

Each mutant is a build of the oracle's C source with one slip planted (ties
rounded away from zero, a dynamic scale one ulp off or with the wrong
maximum, the weight scale dropped from the forward, the forward's weight
index transposed, dlhs folding the wrong group's weight scale in, the tgmm
reusing the first chunk's scale, the forward's absum without the absolute
value).  The test compiles each mutant, swaps it in for the oracle library
and runs the pins of tests/test_oracle_*.py against it: every mutant must
fail at least one pin.  Nothing here runs on a GPU; every planted read stays
inside its array.
"""
import pytest

import oracle
import oracle.oracle as oracle_module
import test_oracle_e4m3 as E
import test_oracle_gmm as P
import test_oracle_quantize as Q

QS, QD = oracle.Q_STATIC, oracle.Q_DYNAMIC

# (function, text in its body, replacement)
MUTANTS = {
    "encode_ties_away_from_zero": ("gmo_e4m3_encode", "r = (fmod(fl, 2.0) == 0.0) ? fl : fl + 1.0;",
                                   "r = fl + 1.0;"),
    "dynamic_scale_one_ulp_high": ("dyn_scale", "float s = amax / 448.0f;",
                                   "float s = nextafterf(amax / 448.0f, INFINITY);"),
    "dynamic_scale_wrong_maximum": ("dyn_scale", "float s = amax / 448.0f;", "float s = amax / 240.0f;"),
    "fwd_weight_scale_dropped": ("gmo_gmm_fwd", "o[n] *= (double)sr[(int64_t)g * N + n];", "o[n] *= 1.0;"),
    "fwd_weight_index_transposed": ("gmo_gmm_fwd", "double p = x * tab[wrow[n]];",
                                    "double p = x * tab[qr[(int64_t)g * K * N + n * K + k]];"),
    "fwd_absum_without_abs": ("gmo_gmm_fwd", "bab[n] += fabs(p);", "bab[n] += p;"),
    "dlhs_folds_group0_scale": ("gmo_gmm_dlhs", "t[n] = gmo_bf16_to_f32(dout[m * N + n]) * sr[(int64_t)g * N + n];",
                                "t[n] = gmo_bf16_to_f32(dout[m * N + n]) * sr[n];"),
    "drhs_first_chunk_scale_everywhere": ("gmo_tgmm_drhs", "double sxk = (double)sx[(chunk0[g] + c) * K + k];",
                                          "double sxk = (double)sx[chunk0[g] * K + k];"),
}

PINS = [
    ("e4m3 round trip", E.test_encode_round_trip_every_finite_code, ()),
    ("e4m3 midpoints to even", E.test_midpoints_round_to_even, ()),
    ("e4m3 saturation", E.test_clip_saturates_at_448, ()),
    ("e4m3 tiny values", E.test_tiny_values, ()),
    ("e4m3 vs torch cast", E.test_encode_matches_torch_cast_in_range, ()),
    ("amax 448 gives scale 1", Q.test_block_with_amax_448_has_unit_scale, ()),
    ("static 4/448", Q.test_static_scale_4_over_448, ()),
    ("dynamic error bound", Q.test_dynamic_rows_error_bound_and_amax_maps_to_448, ()),
    ("rhs per-column scale", Q.test_rhs_per_column_scale, ()),
    ("fwd vs numpy (static)", P.test_fwd_matches_numpy_matmul, (*P.CASES[0], QS)),
    ("fwd vs numpy (dynamic)", P.test_fwd_matches_numpy_matmul, (*P.CASES[1], QD)),
    ("dlhs vs numpy", P.test_dlhs_matches_numpy_matmul, P.CASES[1]),
    ("drhs vs numpy", P.test_drhs_matches_numpy_matmul, (*P.CASES[1], QD)),
    ("gradients vs autograd", P.test_gradients_match_autograd_of_dequantized_forward, (QD,)),
]


def plant(src: str, func: str, old: str, new: str) -> str:
    start = src.index(f" {func}(")
    start = src.rindex("\n", 0, start) + 1
    end = src.index("\n}\n", start)
    body = src[start:end]
    assert body.count(old) == 1, f"{old!r} occurs {body.count(old)} times in {func}"
    return src[:start] + body.replace(old, new) + src[end:]


@pytest.fixture(scope="module")
def mutant_libs(tmp_path_factory):
    d = str(tmp_path_factory.mktemp("oracle_fp8_mutants"))
    src = oracle.source_text()
    return {name: oracle.load_variant(oracle.build_variant(plant(src, *m), d, name))
            for name, m in MUTANTS.items()}


def failing_pins(L):
    saved = oracle_module._lib
    oracle_module._lib = L
    failed = []
    try:
        for what, fn, args in PINS:
            try:
                fn(*args)
            except AssertionError:
                failed.append(what)
    finally:
        oracle_module._lib = saved
    return failed


def test_the_pins_hold_for_the_oracle():
    assert failing_pins(oracle.lib()) == []


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_every_planted_mistake_fails_a_pin(name, mutant_libs):
    failed = failing_pins(mutant_libs[name])
    assert failed, f"planted mistake {name} passed every pin"
