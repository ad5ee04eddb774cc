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


# ---- prefix cache -------------------------------------------------------------------------------
from oracle.block_pool import CACHE_MUTANTS  # noqa: E402
from pool_harness import PrefixContentCheck, random_cache_script, run_cache_script  # noqa: E402


def pin_prefix_cache_contents(mutant=None):
    """Random serving scripts (shared system prompts, continued conversations, decode appends,
    forks, frees, small pools that evict): every live sequence reads, at every position, the K/V
    of its own prefix -- so every reused block held exactly the prefix it was reused for -- and
    every count equals its holders. The cache must also have been used."""
    hits = 0
    for seed, num_blocks in [(0, 30), (1, 48), (2, 120), (3, 20)]:
        mgr = OracleAdapter(num_blocks, 16, mutant, prefix_cache=True)
        cc = PrefixContentCheck(mgr, num_blocks)

        def after(i, op, res):
            cc.check()
            holders_match_tables(mgr, cc.ids)

        run_cache_script(cc, random_cache_script(seed), after)
        hits += cc.cached_tokens
    assert hits > 0


def pin_shared_system_prompt(mutant=None):
    """Requests that begin with the same system prompt keep one copy of its blocks and every
    table points at it (一文搞懂vLLM, "PagedAttention 是怎么共享内存的")."""
    mgr = OracleAdapter(32, 16, mutant, prefix_cache=True)
    cc = PrefixContentCheck(mgr, 32)
    system = list(range(100, 200))                      # 100 tokens: 6 full blocks + 4
    assert cc.prompt("A", system + [1, 2, 3]) == 0
    assert cc.prompt("B", system + [7, 8]) == 96        # the 6 full blocks of the shared prefix
    a, b = mgr.table("A"), mgr.table("B")
    assert a[:6] == b[:6] and a[6] != b[6]
    assert all(mgr.holders(x) == 2 for x in a[:6])
    cc.check()


def pin_multi_turn(mutant=None):
    """In a multi-turn conversation only the newest message needs computing: every full block of
    the history hits the cache, even after the earlier turn finished (blog.mckayzhao.com/?p=56,
    "进阶特性：让推理再快一点"; vLLM 简介, "自动前缀缓存")."""
    mgr = OracleAdapter(64, 16, mutant, prefix_cache=True)
    cc = PrefixContentCheck(mgr, 64)
    turn1 = list(range(1000, 1070))                     # 70-token first prompt
    cc.prompt(1, turn1)
    answer = list(range(2000, 2041))                    # 41 tokens generated one by one
    for t in answer:
        cc.append(1, 1, [t])
    history = turn1 + answer                            # 111 tokens: 6 full blocks + 15
    cc.free(1)
    cached = cc.prompt(2, history + list(range(3000, 3012)))
    assert cached == 16 * (len(history) // 16) == 96
    cc.check()


def pin_last_token_computed(mutant=None):
    """A prompt wholly in the cache still computes its last token (its block is not reused)."""
    mgr = OracleAdapter(16, 16, mutant, prefix_cache=True)
    cc = PrefixContentCheck(mgr, 16)
    ids = list(range(32))
    cc.prompt("x", ids)
    assert cc.prompt("y", ids) == 16
    cc.check()


def pin_cached_blocks_survive_until_taken(mutant=None):
    """A finished request's blocks stay reusable until the pool needs them; blocks are taken
    least recently released first and a request releases its last block first, so a longer
    prompt loses its tail before its beginning."""
    mgr = OracleAdapter(8, 16, mutant, prefix_cache=True)
    cc = PrefixContentCheck(mgr, 8)
    ids = list(range(64))                               # 4 full blocks
    cc.prompt("a", ids + [999])                         # blocks 0-4
    cc.free("a")                                        # free: 5 6 7 4 3 2 1 0
    assert cc.prompt("b", ids + [5]) == 64              # reuses 0-3, takes 5
    cc.free("b")                                        # free: 6 7 4 5 3 2 1 0
    cc.prompt("filler", list(range(500, 565)))          # takes 6 7 4 5 3: the 4th prompt block goes
    cc.free("filler")
    assert cc.prompt("c", ids + [6]) == 48              # the first three prompt blocks survived
    cc.check()


def pin_whole_prefix_must_match(mutant=None):
    """A block's K/V depend on every token before it, so a block is reused only for the same whole
    prefix: equal tokens after a different beginning are computed again."""
    mgr = OracleAdapter(16, 16, mutant, prefix_cache=True)
    cc = PrefixContentCheck(mgr, 16)
    x, y, z, w = (list(range(k, k + 16)) for k in (0, 100, 200, 300))
    cc.prompt("a", x + w + [1])                         # caches x, then x+w
    cc.prompt("b", z + y + [2])                         # caches z, then z+y
    assert cc.prompt("c", x + y + [3]) == 16            # x hits; y's cached block follows z, not x
    assert cc.prompt("d", x + y + [4]) == 32            # c has cached x+y by now
    cc.check()


CACHE_PINS = [pin_prefix_cache_contents, pin_shared_system_prompt, pin_multi_turn, pin_last_token_computed,
              pin_cached_blocks_survive_until_taken, pin_whole_prefix_must_match]


@pytest.mark.parametrize("pin", CACHE_PINS, ids=lambda p: p.__name__)
def test_prefix_cache_pin(pin):
    pin()


@pytest.mark.parametrize("mutant", CACHE_MUTANTS)
def test_prefix_cache_mutant_is_caught(mutant):
    failed = []
    for pin in CACHE_PINS:
        try:
            pin(mutant=mutant)
        except Exception as e:  # an assertion or a model error both count as caught
            failed.append((pin.__name__, type(e).__name__))
    assert failed, f"no pin catches mutant {mutant}"
