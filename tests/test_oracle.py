"""CPU oracle against its pins (see oracle_pins.py), plus a mutation check:
each planted mistake in the oracle must be caught by at least one pin."""
import pytest

from tests import oracle_pins

# planted mistakes (switch values inside the oracle) and what they break
FAULTS = {
    1: "ReLU dropped from the indexer score",
    2: "score ties broken towards the later position",
    3: "causal window excludes the query's own position",
    4: "softmax scale dropped",
    5: "V taken from the tail of the latent row instead of its head",
    6: "indexer key written one cache row past the new token's position",
    7: "indexer key map read transposed",
}


@pytest.mark.parametrize("pin", oracle_pins.PINS, ids=lambda f: f.__name__)
def test_oracle_pin(pin, oracle_mod):
    oracle_mod.set_fault(0)
    pin()


@pytest.mark.parametrize("fault", sorted(FAULTS), ids=lambda f: FAULTS[f])
def test_planted_mistake_is_caught(fault, oracle_mod):
    caught = []
    try:
        oracle_mod.set_fault(fault)
        for pin in oracle_pins.PINS:
            try:
                pin()
            except (AssertionError, ValueError, IndexError):
                caught.append(pin.__name__)
    finally:
        oracle_mod.set_fault(0)
    assert caught, f"no pin catches: {FAULTS[fault]}"
