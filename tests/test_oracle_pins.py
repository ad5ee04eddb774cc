"""The CPU oracle against its pins (pages' worked examples, closed forms, invariants, brute force)."""
import pytest

import oracle_pins as pins


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin()


def test_kv_bytes_13b_closed_form():
    """blog.mckayzhao.com/?p=56, "故事要从 KV Cache 说起": ~1.7 GB of KV for one LLaMA-13B request."""
    g = pins.golden("kv_cache_13b.json")
    per_token = 2 * g["layers"] * g["kv_heads"] * g["head_dim"] * g["elem_bytes"]
    total = per_token * g["tokens"]
    assert abs(total - g["stated_bytes_approx"]) / g["stated_bytes_approx"] <= g["relative_tolerance"]
