"""Each planted mistake in the oracle (built with -DORACLE_MUTANT=n, on the CPU)
must be caught by at least one pin: a dropped gate term, ties to the wrong
expert, gate and up projections swapped, W2 transposed, one gate for every
slot, an unstable permutation, and a sign error in silu."""
import pytest

import oracle
import oracle_checks as oc

MUTANTS = {1: "dropped softmax term", 2: "ties to the higher id", 3: "silu on the up projection",
           4: "W2 transposed", 5: "slot-0 gate for all slots", 6: "unstable permutation",
           7: "silu exponent sign"}


@pytest.mark.parametrize("mutant", sorted(MUTANTS), ids=lambda m: MUTANTS[m])
def test_mutant_is_caught(mutant, tmp_path_factory):
    d = tmp_path_factory.mktemp(f"mutant{mutant}")
    o = oracle.Oracle(mutant, out_dir=str(d))
    failed = []
    for check in oc.ALL_CHECKS:
        try:
            check(o)
        except AssertionError:
            failed.append(check.__name__)
    assert failed, f"no pin caught mutant {mutant} ({MUTANTS[mutant]})"
