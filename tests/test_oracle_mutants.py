"""The oracle's pins are sensitive: plant one plausible mistake at a time in a
copy of the oracle's C source (on the CPU), rebuild it, and check that at least
one pin in test_oracle_pins.py fails for every mutant."""
import os
import subprocess

import pytest

import oracle
import test_oracle_pins as pins
import test_oracle_spec as spec_pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "cq_oracle.c")

MUTANTS = {
    "round_half_away": ("nearbyint(w[i] / s)", "round(w[i] / s)"),
    "clip_low_at_minus7": ("if (r < (double)qmin)\n            r = (double)qmin;",
                           "if (r < (double)qmin + 1)\n            r = (double)qmin + 1;"),
    "tie_to_higher_pattern": ("if (f < best) {", "if (f <= best) {"),
    "sum_instead_of_max": ("        if (obj[e] > f)\n            f = obj[e];", "        f = f + obj[e];"),
    "diagonal_dropped": ("obj[e] = obj[e] + (double)d[e][i] * rr;", "obj[e] = obj[e] + rr;"),
    "abs_instead_of_square": ("double rr = r * r;", "double rr = fabs(r);"),
    "subnormal_decode": ("ldexp((double)man, -24)", "ldexp((double)man, -25)"),
    "column_layout_transposed": ("(g % gpr) * jb->n", "((g / gpr) % gpr) * jb->n"),
    "runner_up_not_demoted": ("            runner = best;\n            rb = bb;\n", ""),
    "pack_offset": ("(q[8 * j + t] + 8)", "(q[8 * j + t] + 7)"),
    "domain_skips_first": ("b = CQO_FIRST_SCALE;", "b = CQO_FIRST_SCALE + 1;"),
    "codes_not_clipped_high": ("if (r > (double)qmax)\n            r = (double)qmax;", ""),
    "qmin_fixed_at_minus_8": ("if (r < (double)qmin)\n            r = (double)qmin;",
                              "if (r < -8.0)\n            r = -8.0;"),
    "qmax_fixed_at_7": ("if (r > (double)qmax)\n            r = (double)qmax;",
                        "if (r > 7.0)\n            r = 7.0;"),
}


def _checks():
    g128 = pins.make_groups128()
    yield pins.test_pack_codes_layout
    yield pins.test_all_zero_group
    yield pins.test_pages_solver_example_golden
    yield pins.test_objective_at_rounding_ties_and_clip
    yield pins.test_single_nonzero_closed_form
    yield pins.test_exact_fit_lowest_zero_scale
    yield pins.test_per_column_and_per_group_layouts_agree
    yield pins.test_scale_domain_is_31743_ordered_patterns
    for c in range(12):
        yield lambda c=c: pins.test_oracle_matches_exact_bruteforce(c)
    yield lambda: pins.test_env_duplicate_permute_pow2_invariance(g128)
    yield lambda: pins.test_bounds_absmax_single_env_and_added_env(g128)
    for spec in spec_pins.SPECS:
        yield lambda spec=spec: spec_pins.test_spec_matches_exact_bruteforce(spec)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not unique"
    mut = tmp_path / "cq_oracle_mut.c"
    mut.write_text(src.replace(old, new))
    so = tmp_path / "libmut.so"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fPIC", "-shared",
                           "-pthread", "-o", str(so), str(mut), "-lm"])
    prev = oracle._set_lib(oracle.load(str(so)))
    try:
        caught = None
        for check in _checks():
            try:
                check()
            except AssertionError:
                caught = check
                break
        assert caught is not None, f"no pin caught mutant {name}"
    finally:
        oracle._set_lib(prev)
