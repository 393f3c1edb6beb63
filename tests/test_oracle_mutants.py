"""Plant one mistake at a time in the oracle (CPU builds with -DKVO_MUTANT=n) and show
that the pins catch each one: a strided group index, a dropped scale, a base-2 lse, a
dropped RoPE term, values read from the key cache, a dropped last position, a flipped
rotary sine, a halved rotary frequency exponent, a multi-token query that cannot see its
own position, a sliding window one token too wide, E4M3 codes decoded without
subnormals or with the wrong exponent bias, E4M3 encoding with ties away from zero."""
import pytest

import oracle
from tests import oracle_pins

MUTANTS = {1: "strided group index", 2: "scale dropped", 3: "base-2 log-sum-exp",
           4: "MLA RoPE score term dropped", 5: "values read from K", 6: "last position dropped",
           7: "rotary sine sign flipped", 8: "rotary frequency exponent halved",
           9: "multi-token: own position hidden", 10: "multi-token: window one too wide",
           11: "E4M3 subnormals decoded as normals", 12: "E4M3 exponent bias 8",
           13: "E4M3 ties rounded away from zero"}


@pytest.mark.parametrize("mutant", sorted(MUTANTS), ids=lambda m: MUTANTS[m])
def test_pins_catch_planted_mistake(mutant, tmp_path):
    lib = oracle.load(mutant=mutant, out_dir=str(tmp_path))
    assert lib.kvo_mutant() == mutant
    caught = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(lib)
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"no pin caught mutant {mutant} ({MUTANTS[mutant]})"
