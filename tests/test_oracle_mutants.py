"""Every plausible mistake planted in the oracle (one -DORACLE_MUTANT_* macro each) fails a pin."""
import pytest

import oracle_pins as pins

MUTANTS = ["HALF_BIAS", "SLOT_POS", "WRITE_OFFSET", "COPY_K_ONLY", "CAUSAL", "GQA", "TABLE_INDEX",
           "POOL_STRIDE", "NO_SCALE"]


@pytest.mark.parametrize("mutant", MUTANTS)
def test_mutant_is_caught(mutant):
    failed = []
    for pin in pins.ALL_PINS:
        try:
            pin(mutant=mutant)
        except Exception as e:  # an assertion or an oracle error both count as "caught"
            failed.append((pin.__name__, type(e).__name__))
    assert failed, f"no pin catches mutant {mutant}"
