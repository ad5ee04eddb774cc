"""The library's host block manager (pkv_bm_* in include/pkv.h) against the oracle's block-pool model.

No GPU: the manager is host code. Which free block an allocation takes is not fixed by the pages
(any free block will do), so product and oracle are compared op by op under a one-to-one mapping
of block ids that must stay consistent: same outcomes, same lengths, same table shapes, same counts,
same copy-on-write pairs, same statistics. The content simulator checks the product on its own.
"""
import numpy as np
import pytest

from oracle.block_pool import OutOfBlocks
from paged_kv_cache_446_b200 import build as pkv_build
from pool_harness import (ContentCheck, OracleAdapter, PrefixContentCheck, ProductAdapter, random_cache_script,
                          random_script, run_cache_script, run_script)


@pytest.fixture(scope="module")
def pkv():
    pkv_build.build()
    from paged_kv_cache_446_b200 import pkv as mod
    return mod


def block_mapping(prod, orac, live):
    """Product id -> oracle id over all live tables; asserts it is a consistent bijection."""
    fwd, bwd = {}, {}
    for s in live:
        tp, to = prod.table(s), orac.table(s)
        assert prod.length(s) == orac.length(s)
        assert len(tp) == len(to), f"sequence {s}: {len(tp)} blocks vs {len(to)}"
        for a, b in zip(tp, to):
            assert fwd.setdefault(a, b) == b and bwd.setdefault(b, a) == a, f"sharing differs at block {a}"
    return fwd


class Lockstep:
    """Applies each op to product and oracle; both must succeed or both run out of blocks."""

    def __init__(self, num_blocks, prefix_cache=False):
        self.p = ProductAdapter(num_blocks, prefix_cache=prefix_cache)
        self.o = OracleAdapter(num_blocks, prefix_cache=prefix_cache)
        self.last = None

    def _both(self, name, *a):
        outs = []
        for m in (self.p, self.o):
            try:
                outs.append(("ok", getattr(m, name)(*a)))
            except OutOfBlocks:
                outs.append(("oob", None))
        assert outs[0][0] == outs[1][0], f"{name}{a}: product {outs[0][0]}, oracle {outs[1][0]}"
        self.last = (name, outs[0][1], outs[1][1])
        if outs[0][0] == "oob":
            raise OutOfBlocks()
        return outs[0][1]

    def add(self, s, n):
        return self._both("add", s, n)

    def fork(self, p, c):
        return self._both("fork", p, c)

    def append(self, s, n, tokens=None):
        return self._both("append", s, n, tokens)

    def step(self, batch, tokens=None):
        return self._both("step", batch, tokens)

    def prompt(self, s, tokens):
        return self._both("prompt", s, tokens)

    def free(self, s):
        return self._both("free", s)


@pytest.mark.parametrize("seed,num_blocks", [(10, 32), (11, 48), (12, 64), (13, 128), (14, 400), (15, 20)])
def test_matches_oracle_op_by_op(pkv, seed, num_blocks):
    ls = Lockstep(num_blocks)
    live = set()

    def after(i, op, res):
        kind = op[0]
        if res[0] == "ok":
            if kind == "add":
                live.add(op[1])
            elif kind == "fork":
                live.add(op[2])
            elif kind == "free":
                live.discard(op[1])
        fwd = block_mapping(ls.p, ls.o, live)
        for a, b in fwd.items():
            assert ls.p.holders(a) == ls.o.holders(b)
        assert ls.p.stats() == ls.o.stats()
        if res[0] != "ok":
            return
        _, rp, ro = ls.last
        if kind == "append":
            assert [(fwd[a], fwd[b]) for a, b in rp] == ro
        elif kind == "step":
            tp, cp, qp, pp = rp
            to, co, qo, po = ro
            assert cp == co and qp == qo
            assert [[fwd[b] for b in row] for row in tp] == to
            assert [(fwd[a], fwd[b]) for a, b in pp] == po

    outcomes = run_script(ls, random_script(seed, num_ops=400), after)
    kinds = {r[0] for r in outcomes}
    assert "ok" in kinds
    if num_blocks <= 48:
        assert "out_of_blocks" in kinds      # the small pools exercise the failure path


@pytest.mark.parametrize("seed", [20, 21, 22])
def test_contents_read_back(pkv, seed):
    mgr = ProductAdapter(96)
    cc = ContentCheck(mgr, 96)
    run_script(cc, random_script(seed, num_ops=400), lambda i, op, res: cc.check())
    st = mgr.stats()
    assert st["cow_copies"] > 0 and st["shared_blocks"] >= 0


def test_documented_allocation_order(pkv):
    """A new pool hands out 0, 1, 2, ...; released blocks join the back of the free queue, so the
    least recently released block is reused first; a sequence releases its blocks last to first."""
    m = pkv.BlockManager(6)
    m.add(1, 40)
    assert m.sequence(1) == (40, [0, 1, 2])
    m.add(2, 1)
    assert m.sequence(2) == (1, [3])
    m.free(1)                                # queue: 4 5 2 1 0
    m.add(3, 40)
    assert m.sequence(3) == (40, [4, 5, 2])
    m.free(2)                                # queue: 1 0 3
    assert m.append(3, 16) is None
    assert m.sequence(3) == (56, [4, 5, 2, 1])


def test_errors_change_nothing(pkv):
    m = pkv.BlockManager(6)
    m.add(1, 20)                             # 2 blocks, last holds 4 tokens
    m.fork(1, 2)
    snap = (m.sequence(1), m.sequence(2), m.stats())
    cases = [
        (lambda: m.add(3, 16 * 5), pkv.PKV_ERR_OUT_OF_BLOCKS),
        (lambda: m.append(2, 16 * 5), pkv.PKV_ERR_OUT_OF_BLOCKS),          # copy + 5 more
        (lambda: m.step({1: 16 * 3, 2: 16 * 2}, 8), pkv.PKV_ERR_OUT_OF_BLOCKS),
        (lambda: m.add(1, 3), 1),                                         # id already live
        (lambda: m.fork(9, 4), 1),                                        # unknown parent
        (lambda: m.fork(1, 2), 1),                                        # child already live
        (lambda: m.append(9, 1), 1),
        (lambda: m.append(1, -1), 1),
        (lambda: m.free(9), 1),
        (lambda: m.step({1: 1, 9: 1}, 8), 1),                             # unknown id
        (lambda: m.step({1: 1, 2: -1}, 8), 1),
        (lambda: m.step({1: 1, 2: 1}, 1), 1),                             # table row too short
        (lambda: m.block_tables([1, 2], 1), 1),
        (lambda: m.refcount(6), 1),
        (lambda: m.refcount(-1), 1),
    ]
    for fn, status in cases:
        with pytest.raises(pkv.PkvError) as e:
            fn()
        assert e.value.status == status
        assert (m.sequence(1), m.sequence(2), m.stats()) == snap
    # Repeated ids in one step cannot be expressed through a dict; go through the C call.
    import ctypes
    ids = np.array([1, 1], np.int64)
    n = np.array([1, 1], np.int32)
    tables = np.empty((2, 8), np.int32)
    ctx = np.empty(2, np.int32)
    qsl = np.empty(3, np.int32)
    pairs = np.empty((2, 2), np.int32)
    cnt = ctypes.c_int(0)
    assert pkv._bm_step(m._h, pkv._np_ptr(ids), pkv._np_ptr(n), 2, None, pkv._np_ptr(tables), 8, pkv._np_ptr(ctx),
                        pkv._np_ptr(qsl), pkv._np_ptr(pairs), ctypes.byref(cnt)) == 1
    assert (m.sequence(1), m.sequence(2), m.stats()) == snap
    with pytest.raises(pkv.PkvError):
        pkv.BlockManager(-1)
    with pytest.raises(pkv.PkvError):
        pkv.BlockManager(4, 0)


def test_step_outputs(pkv):
    """The step call returns the hot path's inputs: -1 padded tables, lengths after the append,
    the prefix sum of the batch's counts and the copies to make first."""
    m = pkv.BlockManager(64)
    m.add(7, 20)
    m.fork(7, 8)
    m.fork(7, 9)
    m.add(5, 0)
    tables, ctx, qsl, pairs = m.step({8: 1, 9: 3, 7: 1, 5: 40}, 6)
    assert ctx.tolist() == [21, 23, 21, 40]
    assert qsl.tolist() == [0, 1, 4, 5, 45]
    # 8 and 9 each copy the shared partial block; 7 is then its only holder and writes in place.
    src = m.sequence(7)[1][1]
    assert pairs.shape == (2, 2) and pairs[:, 0].tolist() == [src, src]
    assert pairs[0, 1] == tables[0, 1] and pairs[1, 1] == tables[1, 1]
    assert tables[2, :2].tolist() == m.sequence(7)[1] and (tables[:3, 2:] == -1).all()
    assert tables[3, :3].tolist() == m.sequence(5)[1] and (tables[3, 3:] == -1).all()
    assert m.refcount(src) == 1 and m.refcount(tables[0, 0]) == 3
    st = m.stats()
    assert st["cow_copies"] == 2 and st["num_sequences"] == 4
    assert st["logical_tokens"] == 21 + 23 + 21 + 40
    # Empty batch: nothing changes, qsl = [0].
    t2, c2, q2, p2 = m.step({}, 4)
    assert t2.shape == (0, 4) and q2.tolist() == [0] and p2.shape == (0, 2)


def test_batch_step_equals_sequential_appends(pkv):
    """One step over a batch makes the same tables and copies as appending member by member."""
    rng = np.random.default_rng(3)
    a, b = pkv.BlockManager(512), pkv.BlockManager(512)
    lens = rng.integers(0, 50, size=6)
    for m in (a, b):
        for s in range(6):
            m.add(s, int(lens[s]))
        for s in range(6, 18):
            m.fork(s % 6, s)
    batch = {int(s): int(n) for s, n in zip(rng.permutation(18), rng.integers(0, 20, size=18))}
    tables, ctx, qsl, pairs = a.step(batch, 8)
    seq_pairs = [p for p in (b.append(s, n) for s, n in batch.items()) if p is not None]
    assert [tuple(p) for p in pairs.tolist()] == seq_pairs
    assert (tables == b.block_tables(list(batch), 8)).all()
    assert a.stats() == b.stats()


def test_waste_statistics_on_workload_mixes(pkv):
    """Paged storage of the decode workloads' length mixes (64 requests of U[128, 2048] tokens;
    256 of lognormal(ln 1000, 1) clipped to [16, 8192]) wastes under 4% of the reserved slots, the
    figure blog.mckayzhao.com/?p=56 gives in "PagedAttention：操作系统课本里翻出来的灵感"."""
    from paged_kv_cache_446_b200 import workloads as W
    for c in ("c2", "c3"):
        wl = W.make(c, with_tensors=False)
        lens = (wl.prior_lens + 1).astype(np.int64)
        m = pkv.BlockManager(wl.num_blocks)
        for r, n in enumerate(lens):
            m.add(r, int(n))
        st = m.stats()
        assert st["stored_tokens"] == int(lens.sum())
        assert st["wasted_slots"] <= 15 * len(lens)
        assert st["wasted_slots"] / (16 * st["used_blocks"]) < 0.04


@pytest.mark.parametrize("seed,num_blocks", [(30, 24), (31, 40), (32, 64), (33, 200)])
def test_prefix_cache_matches_oracle(pkv, seed, num_blocks):
    """Prefix-caching managers follow the same documented allocation order as the oracle's plain
    model, so block ids, cached-token counts, copies, tables and statistics must be identical."""
    ls = Lockstep(num_blocks, prefix_cache=True)
    live = set()

    def after(i, op, res):
        kind = op[0]
        if res[0] == "ok":
            if kind == "prompt":
                live.add(op[1])
            elif kind == "fork":
                live.add(op[2])
            elif kind == "free":
                live.discard(op[1])
        for s in live:
            assert ls.p.table(s) == ls.o.table(s) and ls.p.length(s) == ls.o.length(s)
        for b in range(num_blocks):
            assert ls.p.holders(b) == ls.o.holders(b)
        assert ls.p.stats() == ls.o.stats()
        if res[0] == "ok" and kind in ("prompt", "append", "step"):
            _, rp, ro = ls.last
            assert rp == ro

    outcomes = run_cache_script(ls, random_cache_script(seed, num_ops=250), after)
    st = ls.p.stats()
    assert st["cache_hits"] > 0
    if num_blocks <= 40:
        assert "out_of_blocks" in {r[0] for r in outcomes}


@pytest.mark.parametrize("seed", [40, 41])
def test_prefix_cache_contents_read_back(pkv, seed):
    mgr = ProductAdapter(48, prefix_cache=True)
    cc = PrefixContentCheck(mgr, 48)
    run_cache_script(cc, random_cache_script(seed, num_ops=300), lambda i, op, res: cc.check())
    assert cc.cached_tokens > 0


def test_prefix_cache_api(pkv):
    m = pkv.BlockManager(32, prefix_cache=True)
    system = list(range(50, 150))
    assert m.add_cached_prefix(1, system + [1]) == 0       # one lookup, a miss
    m.append(1, 101, system + [1])
    assert m.add_cached_prefix(2, system + [2, 3]) == 96
    tables, ctx, qsl, pairs = m.step({2: 6}, 8, system[96:] + [2, 3])
    assert ctx.tolist() == [102] and qsl.tolist() == [0, 6]
    assert tables[0, :6].tolist() == m.sequence(1)[1][:6]
    st = m.stats()
    assert st["cache_hits"] == 6 and st["cache_queries"] == 7 and st["cached_blocks"] == 6
    # Without a prefix cache nothing is looked up; without ids, appends stop tracking.
    n = pkv.BlockManager(8)
    assert n.add_cached_prefix(1, list(range(40))) == 0
    assert n.sequence(1) == (0, [])
    with pytest.raises(ValueError):
        m.append(2, 2, [1])
    with pytest.raises(pkv.PkvError):
        m.add_cached_prefix(2, [1, 2])                         # id already live
