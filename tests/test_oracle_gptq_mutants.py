"""The GPTQ pins are sensitive: plant one plausible mistake at a time in a
copy of oracle/gptq.py and check that at least one pin in test_oracle_gptq.py
fails for every mutant."""
import os

import pytest

import oracle
import test_oracle_gptq as pins
from mutate import apply, first_failure, load_mutant

SRC = os.path.join(os.path.dirname(oracle.__file__), "gptq.py")

MUTANTS = {
    "zero_stored_unshifted": [("np.uint32(ZERO - 1) << np.uint32(4 * (r % 8))",
                               "np.uint32(ZERO) << np.uint32(4 * (r % 8))")],
    "dequant_without_plus_one": [("(u.astype(np.int64) - (z + 1))", "(u.astype(np.int64) - z)")],
    "qweight_nibbles_reversed": [("qweight[i // 8, :] |= u[:, i].astype(np.uint32) << np.uint32(4 * (i % 8))",
                                  "qweight[i // 8, :] |= u[:, i].astype(np.uint32) << np.uint32(4 * (7 - i % 8))")],
    "scales_not_transposed": [(".reshape(R, gpr).T.copy()", ".reshape(gpr, R).copy()")],
    "unpack_shift": [("u[:, i] = (codes[:, i // 8] >> np.uint32(4 * (i % 8)))",
                      "u[:, i] = (codes[:, i // 8] >> np.uint32(4 * (i % 4)))")],
    "g_idx_interleaved": [("g_idx = (np.arange(K) // GROUP)", "g_idx = (np.arange(K) % (K // GROUP))")],
    "groups_along_columns": [("u = unpack_group_codes(codes).reshape(R, gpr, GROUP).reshape(R, K)",
                              "u = unpack_group_codes(codes).reshape(gpr, R, GROUP).transpose(1, 0, 2).reshape(R, K)")],
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_gptq_pins_catch_mutant(name, tmp_path):
    mod = load_mutant(apply(open(SRC).read(), MUTANTS[name], name), tmp_path, name)
    assert first_failure(mod, pins.CHECKS) is not None, f"no pin catches mutant {name}"


def test_unmutated_copy_passes(tmp_path):
    mod = load_mutant(open(SRC).read(), tmp_path, "clean")
    for check in pins.CHECKS:
        check(mod)
