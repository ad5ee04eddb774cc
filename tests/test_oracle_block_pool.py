"""Pins of the oracle's block-pool model (oracle/block_pool.py) against the pages; no GPU.

Each pin takes `mutant` (None = the real model); test_block_pool_mutant_is_caught plants each named
mistake in the model and asserts that at least one pin fails.
"""
import json
import os

import numpy as np
import pytest

from oracle.block_pool import MUTANTS
from pool_harness import ContentCheck, OracleAdapter, random_script, run_script

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def holders_match_tables(mgr, live):
    """A block's count is the number of live sequences holding it (blog.mckayzhao.com/?p=56,
    "还不止是分页：Copy-on-Write 和内存共享"); blocks nobody holds are free."""
    held = {}
    for s in live:
        for b in set(mgr.table(s)):
            held[b] = held.get(b, 0) + 1
    for b in range(mgr.m.num_blocks):
        assert mgr.holders(b) == held.get(b, 0), f"block {b}: count {mgr.holders(b)}, held by {held.get(b, 0)}"


def pin_contents_and_counts(mutant=None):
    """Random add / fork / append / step / free scripts: every live sequence reads back exactly its
    own tokens (what contiguous storage would hold) and every count equals its holders."""
    for seed, num_blocks in [(0, 40), (1, 64), (2, 200), (3, 24)]:
        mgr = OracleAdapter(num_blocks, 16, mutant)
        cc = ContentCheck(mgr, num_blocks)

        def after(i, op, res):
            cc.check()
            holders_match_tables(mgr, cc.logical)

        run_script(cc, random_script(seed, num_ops=250), after)


def pin_block_accounting(mutant=None):
    """N tokens hold the fewest blocks that fit them and waste at most block_size - 1 slots, whether
    stored at once or one token at a time (blog.mckayzhao.com/?p=56,
    "PagedAttention：操作系统课本里翻出来的灵感")."""
    g = golden("block_accounting.json")
    bs, max_waste = g["block_size"], g["max_wasted_slots"]
    mgr = OracleAdapter(64, bs, mutant)
    mgr.add("grown", 0)
    for n in range(0, 300):
        if n:
            mgr.append("grown", 1)
        mgr.add("direct", n)
        for s in ("grown", "direct"):
            nb = len(mgr.table(s))
            assert nb * bs >= n, "too few blocks to hold the tokens"
            assert n == 0 and nb == 0 or (nb - 1) * bs < n, "more blocks than needed"
            assert nb * bs - n <= max_waste
        mgr.free("direct")


def pin_sharing_figure(mutant=None):
    """The sharing figure: B1, B2 hold a beginning shared by A, B and beam C, stored once; each adds
    its own block (A: B5, B: B6, C: B7)."""
    g = golden("sharing_figure.json")
    mgr = OracleAdapter(16, 16, mutant)
    mgr.add("A", 32)                       # the shared beginning fills B1 and B2 exactly
    mgr.fork("A", "B")
    mgr.fork("A", "C")
    for s in ("A", "B", "C"):
        assert mgr.append(s, 1) == []      # a new block, nothing shared is written
    shared = mgr.table("A")[:2]
    own = {s: mgr.table(s)[2] for s in ("A", "B", "C")}
    for s in ("B", "C"):
        assert mgr.table(s)[:2] == shared
    assert len(set(own.values())) == 3 and not set(own.values()) & set(shared)
    assert [mgr.holders(b) for b in shared] == [3, 3]
    assert all(mgr.holders(b) == 1 for b in own.values())
    st = mgr.stats()
    assert st["used_blocks"] == len(g["shared"]) + len(g["own"])            # 5, not 3 x 3
    assert st["shared_blocks"] == len(g["shared"])
    assert st["logical_tokens"] == 3 * 33 and st["stored_tokens"] == 32 + 3


def pin_copy_on_write(mutant=None):
    """A sequence about to write into a shared block copies it and writes the copy; the original is
    left unchanged for the others; once it has a single holder it is written in place
    (blog.mckayzhao.com/?p=56, "还不止是分页：Copy-on-Write 和内存共享")."""
    mgr = OracleAdapter(16, 16, mutant)
    cc = ContentCheck(mgr, 16)
    cc.add("A", 20)                        # blocks: one full, one holding 4 tokens
    cc.fork("A", "B")
    a_before = mgr.table("A")
    pairs = cc.append("B", 1)
    assert len(pairs) == 1 and pairs[0][0] == a_before[1] and pairs[0][1] not in a_before
    assert mgr.table("A") == a_before and mgr.table("B") == [a_before[0], pairs[0][1]]
    assert mgr.holders(a_before[0]) == 2 and mgr.holders(a_before[1]) == 1
    assert cc.append("A", 1) == []         # A alone holds its last block now
    assert mgr.table("A") == a_before
    assert mgr.stats()["cow_copies"] == 1
    cc.check()
    cc.free("A")
    cc.free("B")
    st = mgr.stats()
    assert st["used_blocks"] == 0 and st["free_blocks"] == 16


def pin_waste_below_claim(mutant=None):
    """Paged storage wastes under 4% of the reserved slots on realistic length mixes
    (blog.mckayzhao.com/?p=56, "PagedAttention：操作系统课本里翻出来的灵感")."""
    bound = golden("block_accounting.json")["waste_after_paging_below"]
    rng = np.random.default_rng(7)
    for lens in (rng.integers(128, 2049, size=64), np.clip(np.rint(rng.lognormal(np.log(1000.0), 1.0, 96)), 16, 8192)):
        mgr = OracleAdapter(int(sum(-(-int(n) // 16) for n in lens)) + 8, 16, mutant)
        for i, n in enumerate(lens):
            mgr.add(i, int(n))
        st = mgr.stats()
        assert st["stored_tokens"] == int(sum(lens))
        assert st["wasted_slots"] / (st["used_blocks"] * 16) < bound


BLOCK_POOL_PINS = [pin_contents_and_counts, pin_block_accounting, pin_sharing_figure, pin_copy_on_write,
                   pin_waste_below_claim]


@pytest.mark.parametrize("pin", BLOCK_POOL_PINS, ids=lambda p: p.__name__)
def test_block_pool_pin(pin):
    pin()


@pytest.mark.parametrize("mutant", MUTANTS)
def test_block_pool_mutant_is_caught(mutant):
    failed = []
    for pin in BLOCK_POOL_PINS:
        try:
            pin(mutant=mutant)
        except Exception as e:  # an assertion or a model error both count as caught
            failed.append((pin.__name__, type(e).__name__))
    assert failed, f"no pin catches mutant {mutant}"


def test_out_of_blocks_changes_nothing():
    mgr = OracleAdapter(4, 16)
    mgr.add(0, 40)                         # 3 blocks
    before = (mgr.table(0), mgr.stats())
    from oracle.block_pool import OutOfBlocks
    with pytest.raises(OutOfBlocks):
        mgr.append(0, 40)                  # needs 3 more
    with pytest.raises(OutOfBlocks):
        mgr.add(1, 17)
    with pytest.raises(OutOfBlocks):
        mgr.step({0: 30})
    assert (mgr.table(0), mgr.stats()) == before
