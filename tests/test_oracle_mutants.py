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


FLATTEN_MUTANTS = ["FLAT_CTX_PRIOR", "FLAT_SORTED_IDS", "FLAT_QSL_SHIFT"]


@pytest.mark.parametrize("mutant", FLATTEN_MUTANTS)
def test_flatten_mutant_is_caught(mutant):
    """Each planted mistake in the oracle's batch flattening fails its pin."""
    with pytest.raises(AssertionError):
        pins.pin_flatten_batch(mutant=mutant)


def test_product_flattening_matches_oracle():
    """The binding's own flattening (paged_kv_cache_446_b200.pkv.flatten_batch, written separately)
    agrees with the pinned oracle on seeded random {request_id: num_tokens} dicts."""
    import numpy as np

    import oracle
    from paged_kv_cache_446_b200 import pkv
    rng = np.random.default_rng(11)
    for _ in range(100):
        R = int(rng.integers(0, 64))
        ids = rng.permutation(10 ** 6)[:R]
        counts = rng.integers(0, 2048, R) * (rng.random(R) < 0.7)
        prior = rng.integers(0, 65536, R)
        batch = {int(i): int(c) for i, c in zip(ids, counts)}
        q1, c1 = pkv.flatten_batch(batch, prior)
        q2, c2 = oracle.flatten_batch(batch, prior)
        assert q1.dtype == q2.dtype == np.int32 and c1.dtype == c2.dtype == np.int32
        assert np.array_equal(q1, q2) and np.array_equal(c1, c2)
