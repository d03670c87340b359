"""The diagonal-estimation pins are sensitive: plant one plausible mistake at
a time in a copy of oracle/diagonals.py and check that at least one pin in
test_oracle_diagonals.py fails for every mutant."""
import os

import pytest

import oracle
import test_oracle_diagonals as pins
from mutate import apply, first_failure, load_mutant

SRC = os.path.join(os.path.dirname(oracle.__file__), "diagonals.py")

MUTANTS = {
    "abs_not_square": [("sq = x[a:b] * x[a:b]", "sq = np.abs(x[a:b])")],
    "sample_variance_divisor": [("m[e, k] = math.fsum(sq[:, k]) / (b - a) if b > a else math.nan",
                                 "m[e, k] = math.fsum(sq[:, k]) / max(b - a - 1, 1) if b > a else math.nan")],
    "normalise_by_max": [("mean = math.fsum(m[e]) / m.shape[1]", "mean = max(m[e])")],
    "not_normalised": [("out[e] = m[e] / mean if mean != 0 else math.nan", "out[e] = m[e]")],
    "environments_pooled": [("a, b = offsets[e], offsets[e + 1]", "a, b = offsets[0], offsets[-1]")],
    "bf16_shift": [("<< np.uint32(16)", "<< np.uint32(15)")],
    "fp32_running_sum": [("math.fsum(sq[:, k])", "float(sq[:, k].astype(np.float32).sum(dtype=np.float32))")],
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_diagonal_pins_catch_mutant(name, tmp_path):
    mod = load_mutant(apply(open(SRC).read(), MUTANTS[name], name), tmp_path, name)
    assert first_failure(mod, pins.CHECKS) is not None, f"no pin catches mutant {name}"


def test_unmutated_copy_passes(tmp_path):
    mod = load_mutant(open(SRC).read(), tmp_path, "clean")
    for check in pins.CHECKS:
        check(mod)
