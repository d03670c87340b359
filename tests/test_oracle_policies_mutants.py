"""The policy pins are sensitive: plant one plausible mistake at a time in a
copy of oracle/policies.py (on the CPU), load the copy, and check that at
least one pin in test_oracle_policies.py fails for every mutant."""
import os

import pytest

import oracle
import test_oracle_policies as pins
from mutate import apply, first_failure, load_mutant

SRC = os.path.join(os.path.dirname(oracle.__file__), "policies.py")

MUTANTS = {
    "pool_fp32_running_sum": [("acc = np.zeros(D.shape[1:], dtype=np.float64)",
                               "acc = np.zeros(D.shape[1:], dtype=np.float32)"),
                              ("acc = acc + D[e].astype(np.float64)", "acc = acc + D[e]")],
    "pool_drops_last_env": [("for e in range(D.shape[0]):", "for e in range(D.shape[0] - 1):")],
    "pool_divides_by_e_plus_1": [("(acc / float(D.shape[0]))", "(acc / float(D.shape[0] + 1))")],
    "absmax_divides_by_8": [("s = max(absmax_scale(W[g]), 1)", "s = max(absmax_scale(W[g], 8), 1)")],
    "absmax_zero_not_raised": [("s = max(absmax_scale(W[g]), 1)", "s = absmax_scale(W[g])")],
    "absmax_keeps_nonfinite": [("        if not _is_finite_group(W[g]):\n            continue\n", "")],
    "column_block_from_row": [("c = (g % (K // GROUP)) * GROUP", "c = ((g // (K // GROUP)) % (K // GROUP)) * GROUP")],
    "proxy_mean_over_envs": [("module_worst = module_env.max(axis=1)", "module_worst = module_env.mean(axis=1)")],
    "proxy_no_scale": [("/ (b - a) * scale)", "/ (b - a))")],
    "proxy_per_group_not_per_weight": [("scale: float = 1.0 / GROUP):", "scale: float = 1.0):")],
    "pooled_uses_first_env": [("solve(W, pool_diagonals(D), K,", "solve(W, D[:1], K,")],
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_policy_pins_catch_mutant(name, tmp_path):
    mod = load_mutant(apply(open(SRC).read(), MUTANTS[name], name), tmp_path, name)
    assert first_failure(mod, pins.CHECKS) is not None, f"no pin catches mutant {name}"


def test_unmutated_copy_passes(tmp_path):
    mod = load_mutant(open(SRC).read(), tmp_path, "clean")
    for check in pins.CHECKS:
        check(mod)
